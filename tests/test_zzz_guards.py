"""Guard bands: every tensor the kernels write (S, Y, the four buffers, y) is placed
inside a larger allocation whose head and tail hold a sentinel; after a run of every
entry point (flush, decode, dense-read decode, the per-row calls, the standard step,
the prefill handoff) the sentinels must be unchanged, i.e. no kernel wrote outside its
tensor.  Small layers of each kind, so that ragged tiles and short slabs are hit.
"""
from __future__ import annotations

import pytest

import synth
from gpu_util import make_layer, to_dev

pytestmark = pytest.mark.gpu

GUARD = 64          # floats on each side (256 bytes: the tensor stays 16-byte aligned)
SENTINEL = 7.5e30   # no kernel produces this from the seeded inputs


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_state_read_b200 import build
    build.build()


def guarded(t):
    import torch
    big = torch.full((t.numel() + 2 * GUARD,), SENTINEL, dtype=torch.float32, device=t.device)
    inner = big[GUARD:GUARD + t.numel()]
    inner.copy_(t.reshape(-1))
    return inner.view(t.shape), big


@pytest.mark.parametrize("cid,B", [(0, 2), (1, 3), (3, 2), (4, 2)])
def test_no_write_outside_the_tensors(cid, B):
    import torch
    cfg = synth.config(cid).replace(B=B)
    layer = make_layer(cfg, synth.layer_rank_table(cfg), synth.basis(cfg), synth.init_state(cfg, range(B)))
    bands = []
    for name in ("S", "Y", "kbuf", "vbuf", "abuf", "bbuf", "y"):
        t = getattr(layer, name)
        if t is None or t.numel() == 0:
            continue
        inner, big = guarded(t)
        setattr(layer, name, inner)
        bands.append((name, big))

    x = [to_dev(synth.step_inputs(cfg, t, range(B))) for t in range(cfg.W + 2)]
    step = lambda f, p, d: f(p, d["q"], d["k"], d["v"], d["a"], d["beta"])
    layer.flush(0)
    for p in range(cfg.W):
        step(layer.decode, p, x[p])
    layer.flush(cfg.W)
    step(layer.dense_decode, 0, x[cfg.W])
    pos = torch.full((B,), 1, dtype=torch.int32, device="cuda")
    layer.decode_rows(pos, x[cfg.W + 1]["q"], x[cfg.W + 1]["k"], x[cfg.W + 1]["v"], x[cfg.W + 1]["a"],
                      x[cfg.W + 1]["beta"])
    n_rows = torch.tensor([2] + [0] * (B - 1), dtype=torch.int32, device="cuda")
    layer.flush_rows(n_rows)
    d = x[0]
    layer.standard_step(d["q"], d["k"], d["v"], d["a"], d["beta"])
    pr = to_dev(synth.prompt_inputs(cfg, 5, range(B)))
    layer.prefill(pr["k"], pr["v"], pr["a"], pr["beta"])
    torch.cuda.synchronize()
    layer.plan.check()
    for name, big in bands:
        assert bool((big[:GUARD] == SENTINEL).all()), f"{name}: write before the tensor"
        assert bool((big[-GUARD:] == SENTINEL).all()), f"{name}: write past the tensor"
        assert bool(torch.isfinite(big[GUARD:-GUARD]).all()), f"{name}: non-finite values inside"
    layer.close()
