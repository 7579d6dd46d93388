"""sketchssm_decode_static_scratch (the decode whose scratch is the library's static
device array) against sketchssm_decode on the same inputs.

It serves callers that cannot allocate device memory once they are serving (an engine
that has given all free HBM to its own pools, or code that must not take cudaMalloc's
implicit synchronisation); nothing in the call allocates.  The static call runs the
two-launch decode (products through scratch, then the combine); sketchssm_decode runs
the same two launches for GDN / KDA and, for Mamba-2, the one-launch decode, which
sums the same terms in another order.  So y must agree within the parity tolerance
(max |diff| / max |ref| <= 1e-4, the bar of every parity test), and bit for bit where
both calls run the same kernels; the appended buffers are copies and agree bit for bit.
Two decode calls in a row on the static path check that the second call does not
depend on what the first left in the shared array.  This file is collected last so
that it also runs after every other GPU test in the session.
"""
from __future__ import annotations

import pytest

import synth
from gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_state_read_b200 import build
    build.build()


def _layer(cfg, rank, omega, S0):
    import rank_state_read_b200 as rs
    return rs.SketchLayer(cfg.kind, batch=cfg.B, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K,
                          value_dim=cfg.V, window=cfg.W, groups=cfg.G, rank_cap=cfg.cap,
                          rank=rank.tolist(), omega=omega, S0=S0)


def _static_decode(layer, pos, x, y):
    import rank_state_read_b200 as rs
    rs.sketchssm_decode_static_scratch(layer.plan, pos, x["q"], x["k"], x["v"], x["a"], x["beta"],
                                       layer.kbuf, layer.vbuf, layer.abuf, layer.bbuf, layer.Y,
                                       layer.omega, layer.S, y)


def _same_y(kind, y_sta, y_ref):
    import torch
    if kind != "mamba2":
        return torch.equal(y_sta, y_ref)
    return bool(torch.isfinite(y_sta).all()) and rel_err(y_sta.cpu().numpy(), y_ref.cpu().numpy()) <= TOL


def _buffers(layer):
    return [t for t in (layer.kbuf, layer.vbuf, layer.abuf, layer.bbuf) if t is not None]


def _pair(cfg, rank):
    """A layer for each entry point, same state, both flushed to the first sketch."""
    omega, S0 = synth.basis(cfg), synth.init_state(cfg, range(cfg.B))
    ref, sta = _layer(cfg, rank, omega, S0), _layer(cfg, rank, omega, S0)
    ref.flush(0)
    sta.flush(0)
    return ref, sta


CASES = [(1, 8), (3, 6), (4, 4), (1, 256)]


@pytest.mark.parametrize("cid,B", CASES, ids=[f"config{c}-B{b}" for c, b in CASES])
def test_two_calls_in_a_row_match_plan_scratch(cid, B):
    import torch
    cfg = synth.config(cid).replace(B=B)
    rank = synth.layer_rank_table(cfg)
    ref, sta = _pair(cfg, rank)
    for pos in range(2):
        x = synth.device_step_inputs(cfg, 100 + pos, "cuda")
        y_ref = ref.decode(pos, x["q"], x["k"], x["v"], x["a"], x["beta"]).clone()
        y_sta = torch.full_like(y_ref, float("nan"))
        _static_decode(sta, pos, x, y_sta)
        torch.cuda.synchronize()
        assert _same_y(cfg.kind, y_sta, y_ref), f"y differs at pos {pos}"
        for a, b in zip(_buffers(sta), _buffers(ref)):
            assert torch.equal(a, b), f"appended buffers differ at pos {pos}"
    sta.plan.check()
    ref.close()
    sta.close()


def test_plans_of_other_kinds_share_the_array():
    """Calls from plans of different kinds and sizes take turns on the one array; each
    still matches its plan-scratch twin (stale rows of another plan do not leak in)."""
    import torch
    cfgs = [synth.config(4).replace(B=4), synth.config(1).replace(B=16), synth.config(3).replace(B=8)]
    pairs = [_pair(c, synth.layer_rank_table(c)) for c in cfgs]
    for pos in range(3):
        for c, (ref, sta) in zip(cfgs, pairs):
            x = synth.device_step_inputs(c, 300 + pos, "cuda")
            y_ref = ref.decode(pos, x["q"], x["k"], x["v"], x["a"], x["beta"]).clone()
            y_sta = torch.empty_like(y_ref)
            _static_decode(sta, pos, x, y_sta)
            torch.cuda.synchronize()
            assert _same_y(c.kind, y_sta, y_ref), (c.kind, pos)
    for ref, sta in pairs:
        ref.close()
        sta.close()


def test_plan_over_the_limit_is_rejected():
    """A plan whose decode needs more scratch than the static array holds is refused with
    SKETCHSSM_ERR_INVALID_ARG before any tensor is looked at."""
    import rank_state_read_b200 as rs
    cfg = synth.config(3).replace(B=4096)
    plan = rs.Plan(cfg.kind, batch=cfg.B, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K,
                   value_dim=cfg.V, window=cfg.W, groups=cfg.G, basis_rows=cfg.Rb,
                   rank_cap=cfg.cap, rank=synth.layer_rank_table(cfg).tolist())
    lib = rs.load()
    st = lib.sketchssm_decode_static_scratch(plan.handle, 0, *([None] * 14))
    assert st == 1
    msg = lib.sketchssm_last_error().decode()
    assert "static scratch" in msg and str(8 << 20) in msg
    plan.close()
