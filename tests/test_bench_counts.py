"""bench.py's algorithmic counts (the numerators of its roofline fractions) against
figures worked out by hand from the layer shapes (CPU only).

Per decode step and batch row the sketch decode moves the sketch rows of the sketch
heads, the state of the dense heads, q, the step's token twice (read, then appended),
the buffered tokens (7.5 on average over a window) and y; the dense-read decode moves
the whole state instead of the sketch rows.  Worked out for the Mamba-2 layer at batch
256 (sum of ranks 762, one dense head), the GDN layer at batch 512 and the KDA layer
at batch 1024, these come to 195 / 1465 MB, 276 / 1251 MB and 743 / 2660 MB a step;
the Mamba-2 flush of 16 tokens to 2.93 GB.
"""
from __future__ import annotations

import numpy as np
import pytest

import bench
import synth

HAND = {  # config: (sketch decode MB, dense-read decode MB), mean over the window
    1: (195, 1465),
    3: (276, 1251),
    4: (743, 2660),
}


@pytest.mark.parametrize("cid", sorted(HAND))
def test_decode_bytes_match_the_hand_figures(cid):
    cfg = synth.config(cid)
    rank = synth.layer_rank_table(cfg)
    sk = np.mean([bench.decode_bytes(cfg, rank, p) for p in range(cfg.W)]) / 1e6
    dn = np.mean([bench.dense_decode_bytes(cfg, p) for p in range(cfg.W)]) / 1e6
    assert abs(sk - HAND[cid][0]) / HAND[cid][0] < 5e-3
    assert abs(dn - HAND[cid][1]) / HAND[cid][1] < 5e-3


def test_flush_and_step_bytes_of_the_mamba2_layer():
    cfg = synth.config(1)
    rank = synth.layer_rank_table(cfg)
    assert abs(bench.flush_bytes(cfg, rank, cfg.W) / 1e9 - 2.93) < 0.01
    # the standard step moves the state twice: 2 x 256 x 128 x 128 x 80 x 4 bytes, plus
    # the token (q, k, v, a) and y
    state = 2 * 256 * 128 * 128 * 80 * 4
    extra = 256 * 4 * (2 * 8 * 128 + 2 * 128 * 80 + 128)
    assert bench.step_bytes(cfg) == state + extra


def test_prefill_instruction_counts():
    """One FMA per state element and token (Mamba-2), two (GDN), three (KDA)."""
    for cid, per in ((1, 1), (3, 2), (4, 3)):
        cfg = synth.config(cid)
        assert bench.prefill_instr(cfg, 64) == per * cfg.B * cfg.H * cfg.K * cfg.V * 64


def test_prefill_tensor_work_of_the_mamba2_layer():
    """The 64-token Mamba-2 prompt runs on the tensor cores: 2 K V T FLOPs per head of
    contraction; the kernel issues three tf32 products of 128 x 128 x 64 per head."""
    cfg = synth.config(1)
    assert bench.prefill_tensor_path(cfg, 64) and not bench.prefill_tensor_path(cfg, 65)
    assert not bench.prefill_tensor_path(synth.config(3), 64)
    assert bench.prefill_tensor_path(cfg.replace(V=128), 64)
    assert not bench.prefill_tensor_path(cfg.replace(V=144), 64)
    fl = bench.prefill_flops(cfg, 64)
    heads = 256 * 128
    assert fl["algorithmic"] == heads * 2 * 128 * 80 * 64
    assert fl["issued"] == heads * 3 * 2 * 128 * 128 * 64
    assert bench.prefill_flops(cfg, 61)["issued"] == fl["issued"]  # the prompt padded to 8


def test_prefill_report_carries_the_pipe_of_its_kernel():
    """The prefill line reports the tensor pipe for the tcgen05 (Mamba-2) kernel and the
    FP32 pipe for the others, and its HBM fraction is the algorithmic bytes over the
    kernel time (the handoff minus the sketch-only call)."""
    pf_us = {64: 1200.0, 0: 350.0}
    clocks = {"sm_max_mhz": 1965.0}
    m2 = bench.prefill_report(synth.config(1), pf_us, clocks, 6541.5, "measured")
    assert "tensor" in m2 and "fp32_pipe" not in m2
    assert m2["kernel_us"] == 850.0
    gbs = bench.prefill_bytes(synth.config(1), 64) / 850e-6 / 1e9
    assert abs(m2["roofline"]["frac"] - gbs / 6541.5) < 1e-4
    assert m2["tensor"]["flops_per_launch"] == bench.prefill_flops(synth.config(1), 64)
    gdn = bench.prefill_report(synth.config(3), pf_us, clocks, 6541.5, "measured")
    assert "fp32_pipe" in gdn and "tensor" not in gdn


def test_prefill_bytes_of_the_mamba2_layer():
    """The prefill reads and writes the state once and reads every prompt token:
    2 x 256 x 128 x 128 x 80 x 4 bytes + 64 tokens x 256 rows x (8 x 128 + 128 x 80 + 128) x 4."""
    cfg = synth.config(1)
    state = 2 * 256 * 128 * 128 * 80 * 4
    toks = 64 * 256 * 4 * (8 * 128 + 128 * 80 + 128)
    assert bench.prefill_bytes(cfg, 64) == state + toks


def test_state_traffic_ratio_of_the_shapes():
    """The state-only bytes per token of the standard step over those of the sketch path
    (the analytic reconstruction of the pages' figure: 10.4x at rank 8, W = 16, K = 128,
    V = 80, no dense head)."""
    cfg = synth.config(1).replace(n_dense=0)
    rank = np.full(cfg.H, 8, np.int32)
    r = bench.state_traffic(cfg, rank)["analytic_state_bytes_per_token"]
    assert abs(r["ratio"] - 10.4) < 0.05
