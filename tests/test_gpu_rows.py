"""Per-sequence positions (sketchssm_decode_rows / sketchssm_flush_rows) against the
fp64 oracle run row by row: every batch row moves through its own window, and rows
flush early at random (partial windows), so positions drift apart.

Bar: max |gpu - oracle| / max |oracle| <= 1e-4 for y every step and S, Y after flushes.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL, make_layer, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_state_read_b200 import build
    build.build()


def rows_run(cfg, T, seed, rank=None):
    import torch
    B = cfg.B
    rng = np.random.default_rng(seed)
    rank = synth.layer_rank_table(cfg) if rank is None else rank
    omega = synth.basis(cfg)
    S0 = synth.init_state(cfg, range(B))
    gpu = make_layer(cfg, rank, omega, S0)
    orcs = [oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G, rank=rank,
                               omega=omega, S0=S0[b:b + 1]) for b in range(B)]
    gpu.flush(0)
    for o in orcs:
        o.flush(0)
    pos = np.zeros(B, np.int64)
    # start the rows at different points of their windows: a few early partial flushes
    worst = 0.0
    flushes = 0
    for t in range(T):
        inp = synth.step_inputs(cfg, t, range(B))
        d = to_dev(inp)
        y = gpu.decode_rows(torch.tensor(pos, dtype=torch.int32, device="cuda"),
                            d["q"], d["k"], d["v"], d["a"], d["beta"])
        yo = np.concatenate([orcs[b].decode(int(pos[b]), {k: (None if v is None else v[b:b + 1])
                                                             for k, v in inp.items()}) for b in range(B)])
        torch.cuda.synchronize()
        e = rel_err(y.cpu().numpy(), yo)
        assert e <= TOL, (t, e)
        worst = max(worst, e)
        pos += 1
        n = np.where((pos == cfg.W) | (rng.random(B) < 0.2), pos, 0)
        if n.any():
            gpu.flush_rows(torch.tensor(n, dtype=torch.int32, device="cuda"))
            for b in range(B):
                if n[b]:
                    orcs[b].flush(int(n[b]))
                    pos[b] = 0
            torch.cuda.synchronize()
            S_or = np.concatenate([o.S for o in orcs])
            assert rel_err(gpu.S.cpu().numpy(), S_or) <= TOL
            if orcs[0].rtot:
                Y_or = np.concatenate([o.Y for o in orcs])
                assert rel_err(gpu.Y.cpu().numpy(), Y_or) <= TOL
            flushes += 1
    assert flushes > 0 and len(set(pos.tolist())) > 1  # the rows did drift apart
    gpu.plan.check()
    gpu.close()
    return worst


@pytest.mark.parametrize("cid,B", [(1, 5), (3, 4), (4, 3), (0, 4)])
def test_rows_drift_apart(cid, B):
    rows_run(synth.config(cid).replace(B=B), T=40, seed=cid)


def test_rows_per_head_qk_mamba2():
    rows_run(synth.config(1).replace(B=3, Hqk=128), T=24, seed=11)


def test_rows_with_dense_heads_and_rank_cap():
    cfg = synth.config(1).replace(B=3)
    rank = np.full(cfg.H, cfg.cap, np.int32)
    rank[::7] = synth.DENSE
    rows_run(cfg, T=24, seed=12, rank=rank)


def test_out_of_range_rows_are_reported_and_left_alone():
    import torch
    import rank_state_read_b200 as rs
    cfg = synth.config(1).replace(B=3)
    rank = synth.layer_rank_table(cfg)
    gpu = make_layer(cfg, rank, synth.basis(cfg), synth.init_state(cfg, range(cfg.B)))
    gpu.flush(0)
    gpu.plan.check()
    d = to_dev(synth.step_inputs(cfg, 0, range(cfg.B)))
    gpu.y.fill_(7.0)
    pos = torch.tensor([0, cfg.W, 0], dtype=torch.int32, device="cuda")
    y = gpu.decode_rows(pos, d["q"], d["k"], d["v"], d["a"], d["beta"])
    with pytest.raises(rs.SketchSSMError) as err:
        gpu.plan.check()
    assert err.value.status == 1
    assert bool((y[1] == 7.0).all()) and not bool((y[0] == 7.0).all())
    S_before = gpu.S.clone()
    gpu.flush_rows(torch.tensor([0, cfg.W + 1, 0], dtype=torch.int32, device="cuda"))
    with pytest.raises(rs.SketchSSMError):
        gpu.plan.check()
    torch.cuda.synchronize()
    assert torch.equal(gpu.S, S_before)
    gpu.close()
