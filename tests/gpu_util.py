"""Shared driver of the GPU-vs-oracle parity tests (imported by tests only)."""
from __future__ import annotations

from typing import Iterable, List, Optional, Sequence

import numpy as np

import oracle
import synth

TOL = 1e-4  # max |gpu - oracle| / max |oracle| per tensor, per step / flush


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    diff = float(np.max(np.abs(np.asarray(gpu, np.float64) - ref))) if ref.size else 0.0
    return diff / den if den > 0 else diff


def to_dev(inp: dict, device="cuda") -> dict:
    import torch
    return {k: (None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(device))
            for k, v in inp.items()}


def make_layer(cfg: synth.Config, rank: np.ndarray, omega: np.ndarray, S0: np.ndarray):
    import rank_state_read_b200 as rs
    return rs.SketchLayer(cfg.kind, batch=cfg.B, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K,
                          value_dim=cfg.V, window=cfg.W, groups=cfg.G, rank_cap=cfg.cap,
                          rank=rank.tolist(), omega=omega, S0=S0)


def parity_run(cfg: synth.Config, T: int, *, rank: Optional[np.ndarray] = None,
               rows: Optional[Sequence[int]] = None, dense: bool = False,
               flush_at: Optional[Iterable[int]] = None, tol: float = TOL) -> dict:
    """Run the GPU layer over T decode steps of seeded inputs beside the fp64 oracle
    on batch rows ``rows`` (all rows if None); compare y every step and S, Y after
    every flush.  ``flush_at`` lists the step counts after which a flush of the
    buffered tokens happens (default: every W steps).  Returns the worst errors."""
    import torch
    rank = synth.layer_rank_table(cfg) if rank is None else np.asarray(rank, np.int32)
    rows = list(range(cfg.B)) if rows is None else list(rows)
    omega = synth.basis(cfg)
    S0 = synth.init_state(cfg, range(cfg.B))
    gpu = make_layer(cfg, rank, omega, S0)
    orc = oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                             rank=rank, omega=omega, S0=S0[rows])
    ridx = torch.tensor(rows, device="cuda")
    flush_at = set(range(cfg.W, T + 1, cfg.W)) if flush_at is None else set(flush_at)
    worst = {"y": 0.0, "S": 0.0, "Y": 0.0}

    def cmp_state():
        torch.cuda.synchronize()
        worst["S"] = max(worst["S"], rel_err(gpu.S.index_select(0, ridx).cpu().numpy(), orc.S))
        if orc.rtot:
            worst["Y"] = max(worst["Y"], rel_err(gpu.Y.index_select(0, ridx).cpu().numpy(), orc.Y))

    gpu.flush(0)
    orc.flush(0)
    cmp_state()
    pos = 0
    for t in range(1, T + 1):
        inp = synth.step_inputs(cfg, t - 1, range(cfg.B))
        d = to_dev(inp)
        if dense:
            y = gpu.dense_decode(pos, d["q"], d["k"], d["v"], d["a"], d["beta"])
        else:
            y = gpu.decode(pos, d["q"], d["k"], d["v"], d["a"], d["beta"])
        yo = orc.decode(pos, {k: (None if v is None else v[rows]) for k, v in inp.items()},
                        dense_all=dense)
        worst["y"] = max(worst["y"], rel_err(y.index_select(0, ridx).cpu().numpy(), yo))
        pos += 1
        if t in flush_at:
            gpu.flush(pos)
            orc.flush(pos)
            cmp_state()
            pos = 0
        assert pos < cfg.W, "flush schedule leaves more than W tokens buffered"
    torch.cuda.synchronize()
    gpu.close()
    for k, v in worst.items():
        assert v <= tol, f"{k}: max relative error {v:.3e} > {tol:.0e} ({cfg.name})"
    return worst
