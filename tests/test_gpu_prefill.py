"""The prefill handoff (sketchssm_prefill) against the fp64 oracle (``oracle.prefill``
followed by the n = 0 flush): the state and the sketch after prompts that span several
token chunks and end in a ragged tail, prompts of 0 and exactly one or two chunks,
Mamba-2 prompts on both sides of the tensor-memory kernel's limits (64 tokens, value
widths up to 128), and the decode steps that follow the handoff from pos = 0.

Bar: max |gpu - oracle| / max |oracle| <= 1e-4 for S, Y and every y.
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


def prefill_parity(cfg, T, rows=None, decode_steps=0):
    import torch
    rows = list(range(cfg.B)) if rows is None else list(rows)
    rank = synth.layer_rank_table(cfg)
    omega = synth.basis(cfg)
    S0 = synth.init_state(cfg, range(cfg.B))
    gpu = make_layer(cfg, rank, omega, S0)
    orc = oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                             rank=rank, omega=omega, S0=S0[rows])
    p = synth.prompt_inputs(cfg, T, range(cfg.B))
    d = to_dev(p)
    gpu.prefill(d["k"], d["v"], d["a"], d["beta"])
    orc.prefill({x: (None if p[x] is None else p[x][rows]) for x in p})
    torch.cuda.synchronize()
    ridx = torch.tensor(rows, device="cuda")
    worst = rel_err(gpu.S.index_select(0, ridx).cpu().numpy(), orc.S)
    assert worst <= TOL, ("S", worst)
    if orc.rtot:
        e = rel_err(gpu.Y.index_select(0, ridx).cpu().numpy(), orc.Y)
        assert e <= TOL, ("Y", e)
        worst = max(worst, e)
    for t in range(decode_steps):  # the decode path picks up at pos = 0
        inp = synth.step_inputs(cfg, 500 + t, range(cfg.B))
        di = to_dev(inp)
        y = gpu.decode(t, di["q"], di["k"], di["v"], di["a"], di["beta"])
        yo = orc.decode(t, {x: (None if inp[x] is None else inp[x][rows]) for x in inp})
        torch.cuda.synchronize()
        e = rel_err(y.index_select(0, ridx).cpu().numpy(), yo)
        assert e <= TOL, ("y", t, e)
        worst = max(worst, e)
    gpu.plan.check()
    gpu.close()
    return worst


@pytest.mark.parametrize("cid,B,T", [(0, 4, 37), (1, 3, 21), (3, 2, 17), (4, 2, 33)])
def test_prefill_small(cid, B, T):
    """Prompts of one or two 16-token chunks plus a ragged tail, every kind."""
    prefill_parity(synth.config(cid).replace(B=B), T)


@pytest.mark.parametrize("T", [0, 1, 16, 32])
@pytest.mark.parametrize("cid", [0, 3])
def test_prefill_edge_lengths(cid, T):
    """No token (Y only), one token, exactly one and two chunks."""
    prefill_parity(synth.config(cid).replace(B=2), T)


@pytest.mark.parametrize("T", [7, 63, 64, 65, 100])
def test_prefill_mamba2_lengths(T):
    """Mamba-2 prompts around the tensor-memory kernel's 64-token limit (a ragged last
    K step, exactly 64, and longer prompts on the chunked kernel)."""
    prefill_parity(synth.config(1).replace(B=3), T)


@pytest.mark.parametrize("V", [16, 48, 112, 128, 160])
def test_prefill_mamba2_value_dims(V):
    """Mamba-2 value widths up to 128 on the tensor-memory kernel (whose 128-row value
    operand reads past the last value row), V = 160 on the chunked one."""
    cfg = synth.config(1).replace(B=2, V=V)
    prefill_parity(cfg, 37)


@pytest.mark.parametrize("V", [16, 48, 256])
def test_prefill_other_value_dims(V):
    """Slabs of 16, 48 and 64 columns (V = 256: four CTAs per state)."""
    cfg = synth.config(4).replace(B=2, V=V, H=4, G=1, Hqk=4, n_dense=1)
    prefill_parity(cfg, 19)


@pytest.mark.parametrize("cid", [1, 3])
def test_prefill_full_size_sampled_rows(cid):
    """The full batch in one launch; the oracle follows three rows."""
    cfg = synth.config(cid)
    prefill_parity(cfg, 18, rows=[0, cfg.B // 2, cfg.B - 1])


@pytest.mark.parametrize("cid", [1, 3, 4])
def test_decode_after_the_handoff(cid):
    """A prompt, the handoff, then W - 1 decode steps from pos = 0."""
    cfg = synth.config(cid).replace(B=3)
    prefill_parity(cfg, 23, decode_steps=cfg.W - 1)


def test_prefill_rejects_a_negative_length():
    import torch
    import rank_state_read_b200 as rs
    cfg = synth.config(0).replace(B=2)
    gpu = make_layer(cfg, synth.layer_rank_table(cfg), synth.basis(cfg), synth.init_state(cfg, range(cfg.B)))
    with pytest.raises(rs.SketchSSMError):
        rs.sketchssm_prefill(gpu.plan, -1, None, None, None, None, gpu.S, gpu.omega, gpu.Y)
    torch.cuda.synchronize()
    gpu.close()


def test_prefill_refused_before_the_state_is_touched():
    """A missing basis (the layer has sketch heads) is refused before the prompt is
    applied: S keeps its values."""
    import torch
    import rank_state_read_b200 as rs
    cfg = synth.config(0).replace(B=2)
    gpu = make_layer(cfg, synth.layer_rank_table(cfg), synth.basis(cfg), synth.init_state(cfg, range(cfg.B)))
    d = to_dev(synth.prompt_inputs(cfg, 5, range(cfg.B)))
    S_before = gpu.S.clone()
    with pytest.raises(rs.SketchSSMError):
        rs.sketchssm_prefill(gpu.plan, 5, d["k"], d["v"], d["a"], d["beta"], gpu.S, None, gpu.Y)
    torch.cuda.synchronize()
    assert torch.equal(gpu.S, S_before)
    gpu.close()
