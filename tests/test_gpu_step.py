"""The standard per-step decode (sketchssm_step) against the fp64 oracle's standard
step, and against the sketch path's own state after a window cycle (same recurrence).

Bar: max |gpu - oracle| / max |oracle| <= 1e-4 for y at every step and for S.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_state_read_b200 import build
    build.build()


def _layer(cfg, rank, S0):
    import rank_state_read_b200 as rs
    return rs.SketchLayer(cfg.kind, batch=cfg.B, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K,
                          value_dim=cfg.V, window=cfg.W, groups=cfg.G, rank_cap=cfg.cap,
                          rank=rank.tolist(), omega=synth.basis(cfg), S0=S0)


def step_parity(cfg, T, rows=None):
    import torch
    rows = list(range(cfg.B)) if rows is None else list(rows)
    S0 = synth.init_state(cfg, range(cfg.B))
    gpu = _layer(cfg, synth.layer_rank_table(cfg), S0)
    S_or = np.ascontiguousarray(S0[rows], dtype=np.float64)
    ridx = torch.tensor(rows, device="cuda")
    worst = 0.0
    for t in range(T):
        inp = synth.step_inputs(cfg, t, range(cfg.B))
        d = to_dev(inp)
        y = gpu.standard_step(d["q"], d["k"], d["v"], d["a"], d["beta"])
        yo = oracle.standard_step(cfg.kind, S_or, {k: (None if v is None else v[rows]) for k, v in inp.items()},
                                  cfg.Hqk)
        torch.cuda.synchronize()
        e = rel_err(y.index_select(0, ridx).cpu().numpy(), yo)
        assert e <= TOL, (t, e)
        worst = max(worst, e)
    e = rel_err(gpu.S.index_select(0, ridx).cpu().numpy(), S_or)
    assert e <= TOL, ("S", e)
    gpu.plan.check()
    gpu.close()
    return max(worst, e)


@pytest.mark.parametrize("cid,B,T", [(0, 4, 20), (1, 3, 18), (3, 2, 18), (4, 2, 18)])
def test_standard_step_small(cid, B, T):
    step_parity(synth.config(cid).replace(B=B), T)


@pytest.mark.parametrize("V", [16, 48, 256])
def test_standard_step_other_value_dims(V):
    """Slabs of one, three and four 64-column pieces (V = 256)."""
    cfg = synth.config(3).replace(B=2, V=V, H=4, G=1, Hqk=4, n_dense=1)
    step_parity(cfg, 6)


@pytest.mark.parametrize("cid", [1, 3, 4])
def test_standard_step_full_size_all_rows(cid):
    """The workloads at their full batch, every batch row against the oracle."""
    step_parity(synth.config(cid), 3)


@pytest.mark.parametrize("cid", [1, 3])
def test_matches_sketch_path_state_after_a_window(cid):
    """W standard steps and the sketch path's W decodes + flush apply the same tokens
    in the same order: their states agree."""
    import torch
    cfg = synth.config(cid).replace(B=4)
    rank = synth.layer_rank_table(cfg)
    S0 = synth.init_state(cfg, range(cfg.B))
    std, sk = _layer(cfg, rank, S0), _layer(cfg, rank, S0)
    sk.flush(0)
    for t in range(cfg.W):
        d = to_dev(synth.step_inputs(cfg, t, range(cfg.B)))
        std.standard_step(d["q"], d["k"], d["v"], d["a"], d["beta"])
        sk.decode(t, d["q"], d["k"], d["v"], d["a"], d["beta"])
    sk.flush(cfg.W)
    torch.cuda.synchronize()
    assert rel_err(std.S.cpu().numpy(), sk.S.cpu().numpy().astype(np.float64)) <= TOL
    std.close()
    sk.close()
