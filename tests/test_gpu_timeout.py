"""The bounded waits of the decode, flush and prefill kernels, made to run out on purpose.

With the plan's wait limit at a few clock cycles, the CTAs' waits for their own bulk
copies run past it: the kernels record a timeout, which sketchssm_plan_check reports
as SKETCHSSM_ERR_TIMEOUT, and keep waiting (up to the default limit) for the same
copies, so the outputs still equal those of a run at the default limit.  Nothing here
faults or hangs a GPU: the copies are ordinary and land a microsecond later.
"""
from __future__ import annotations

import pytest

import synth

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


@pytest.mark.parametrize("cid", [1, 3])
def test_short_wait_limit_is_reported_and_outputs_complete(cid):
    import torch
    import rank_state_read_b200 as rs
    cfg = synth.config(cid).replace(B=16)
    rank = synth.layer_rank_table(cfg)
    omega, S0 = synth.basis(cfg), synth.init_state(cfg, range(cfg.B))
    ref, short = _layer(cfg, rank, omega, S0), _layer(cfg, rank, omega, S0)
    ref.flush(0)
    short.flush(0)
    ref.plan.check()
    short.plan.check()

    short.plan.set_wait_limit(1)
    for pos in range(cfg.W):
        x = synth.device_step_inputs(cfg, 500 + pos, "cuda")
        y_ref = ref.decode(pos, x["q"], x["k"], x["v"], x["a"], x["beta"]).clone()
        y_short = short.decode(pos, x["q"], x["k"], x["v"], x["a"], x["beta"]).clone()
        torch.cuda.synchronize()
        assert torch.equal(y_short, y_ref), pos
    # a decode CTA whose copies landed before it waited records nothing; over the window
    # cycle (the flush's producer and consumers wait on each other's items) the limit
    # of one cycle is certainly overrun somewhere
    ref.flush(cfg.W)
    short.flush(cfg.W)
    with pytest.raises(rs.SketchSSMError) as err:
        short.plan.check()
    assert err.value.status == 5  # SKETCHSSM_ERR_TIMEOUT
    torch.cuda.synchronize()
    assert torch.equal(short.S, ref.S) and torch.equal(short.Y, ref.Y)

    # back at the default limit nothing is recorded
    short.plan.set_wait_limit(2_000_000_000)
    x = synth.device_step_inputs(cfg, 900, "cuda")
    short.decode(0, x["q"], x["k"], x["v"], x["a"], x["beta"])
    short.plan.check()
    ref.close()
    short.close()


def test_short_wait_limit_in_the_tensor_core_prefill():
    """The Mamba-2 prefill waits for its own tensor-core products: with a one-cycle limit
    the waits overrun, the timeout is reported, and the state and sketch equal those of
    a run at the default limit."""
    import torch
    import rank_state_read_b200 as rs
    cfg = synth.config(1).replace(B=4)
    rank = synth.layer_rank_table(cfg)
    omega, S0 = synth.basis(cfg), synth.init_state(cfg, range(cfg.B))
    ref, short = _layer(cfg, rank, omega, S0), _layer(cfg, rank, omega, S0)
    p = {k: (None if v is None else torch.from_numpy(v).cuda()) for k, v in synth.prompt_inputs(cfg, 40, range(cfg.B)).items()}
    ref.prefill(p["k"], p["v"], p["a"], p["beta"])
    ref.plan.check()
    short.plan.set_wait_limit(1)
    short.prefill(p["k"], p["v"], p["a"], p["beta"])
    with pytest.raises(rs.SketchSSMError) as err:
        short.plan.check()
    assert err.value.status == 5  # SKETCHSSM_ERR_TIMEOUT
    torch.cuda.synchronize()
    assert torch.equal(short.S, ref.S) and torch.equal(short.Y, ref.Y)
    ref.close()
    short.close()


def test_wait_limit_must_be_positive():
    import rank_state_read_b200 as rs
    cfg = synth.config(1).replace(B=1)
    plan = rs.Plan(cfg.kind, batch=1, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K, value_dim=cfg.V,
                   window=cfg.W, groups=cfg.G, basis_rows=cfg.Rb, rank_cap=cfg.cap,
                   rank=synth.layer_rank_table(cfg).tolist())
    with pytest.raises(rs.SketchSSMError):
        plan.set_wait_limit(0)
    plan.close()
