"""Shared driver of the GPU-vs-oracle parity tests (imported by tests only).

Error measures, per compared tensor (y at every step; S and Y after every flush):
  * ``rel``      max |gpu - oracle| / max |oracle| over the tensor (the bar: <= TOL);
  * ``rel_head`` the same ratio taken per (batch row, head) slab -- y[b][h], S[b][h],
                 and head h's rows of Y[b] -- and maximised over the slabs (also <= TOL,
                 so that a head of small magnitude cannot hide behind a large one);
  * ``elem``     max |gpu - oracle| / |oracle| over the elements with
                 |oracle| >= 1e-3 max |oracle| (reported, not a bar: an element a
                 thousand times below the tensor's largest carries the rounding of the
                 large terms it is summed from).
"""
from __future__ import annotations

import json
import os
from typing import Iterable, List, Optional, Sequence

import numpy as np

import oracle
import synth

TOL = 1e-4  # bar of ``rel`` and ``rel_head``
ELEM_FLOOR = 1e-3

REPORT: List[dict] = []  # one record per parity run of the session


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    diff = float(np.max(np.abs(np.asarray(gpu, np.float64) - ref))) if ref.size else 0.0
    return diff / den if den > 0 else diff


def _slab_errors(gpu: np.ndarray, ref: np.ndarray, seg: Optional[np.ndarray] = None):
    """(rel, rel_head, elem) of one tensor whose leading axes are (batch row, head) --
    or, with ``seg``, (batch row, sketch row) with head segments starting at ``seg``."""
    B = ref.shape[0]
    gmax = float(np.max(np.abs(ref))) if ref.size else 0.0
    dmax = head = elem = 0.0
    for b0 in range(0, B, 16):  # row chunks bound the host memory of full-size states
        r = np.asarray(ref[b0:b0 + 16], np.float64)
        d = np.abs(np.asarray(gpu[b0:b0 + 16], np.float64) - r)
        ar = np.abs(r)
        if r.size == 0:
            continue
        dmax = max(dmax, float(d.max()))
        if seg is None:
            dh = d.reshape(r.shape[0], r.shape[1], -1).max(axis=2)
            rh = ar.reshape(r.shape[0], r.shape[1], -1).max(axis=2)
        else:
            dh = np.maximum.reduceat(d.max(axis=2), seg, axis=1)
            rh = np.maximum.reduceat(ar.max(axis=2), seg, axis=1)
        head = max(head, float(np.max(np.where(rh > 0, dh / np.where(rh > 0, rh, 1.0), dh))))
        m = ar >= ELEM_FLOOR * gmax
        if m.any():
            elem = max(elem, float((d[m] / ar[m]).max()))
    rel = dmax / gmax if gmax > 0 else dmax
    return rel, head, elem


def to_dev(inp: dict, device="cuda") -> dict:
    import torch
    return {k: (None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(device))
            for k, v in inp.items()}


def make_layer(cfg: synth.Config, rank: np.ndarray, omega: np.ndarray, S0):
    import rank_state_read_b200 as rs
    return rs.SketchLayer(cfg.kind, batch=cfg.B, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K,
                          value_dim=cfg.V, window=cfg.W, groups=cfg.G, rank_cap=cfg.cap,
                          rank=rank.tolist(), omega=omega, S0=S0)


def parity_run(cfg: synth.Config, T: int, *, rank: Optional[np.ndarray] = None,
               rows: Optional[Sequence[int]] = None, dense: bool = False,
               flush_at: Optional[Iterable[int]] = None, tol: float = TOL, layer: int = 0,
               init: str = "numpy", name: Optional[str] = None) -> dict:
    """Run the GPU layer over T decode steps of seeded inputs beside the fp64 oracle
    on batch rows ``rows`` (all rows if None); compare y every step and S, Y after
    every flush.  ``flush_at`` lists the step counts after which a flush of the
    buffered tokens happens (default: every W steps).  ``layer`` selects the stack
    layer whose basis and inputs are drawn.  ``init="sampled"`` draws the initial state
    of the rows the oracle does not check on the device (fast, other numbers) and that of
    the checked rows with the host generator, as everywhere else.  Returns the worst
    errors (``y``, ``S``, ``Y``: rel; ``*_head``, ``*_elem``: the other measures)."""
    import torch
    rank = synth.layer_rank_table(cfg) if rank is None else np.asarray(rank, np.int32)
    rows = list(range(cfg.B)) if rows is None else list(rows)
    omega = synth.basis(cfg, layer)
    S0_rows = synth.init_state(cfg, rows, layer)
    if init == "numpy" and len(rows) == cfg.B and rows == list(range(cfg.B)):
        S0 = S0_rows
    elif init == "numpy":
        S0 = synth.init_state(cfg, range(cfg.B), layer)
    else:
        S0 = synth.device_state(cfg, 4242 + layer, "cuda")
        S0[torch.tensor(rows, device="cuda")] = torch.from_numpy(S0_rows).to("cuda")
    gpu = make_layer(cfg, rank, omega, S0)
    del S0
    orc = oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                             rank=rank, omega=omega, S0=S0_rows)
    del S0_rows
    ridx = torch.tensor(rows, device="cuda")
    flush_at = set(range(cfg.W, T + 1, cfg.W)) if flush_at is None else set(flush_at)
    worst = {k: 0.0 for k in ("y", "S", "Y", "y_head", "S_head", "Y_head", "y_elem", "S_elem", "Y_elem")}
    sk_heads = [h for h in range(cfg.H) if rank[h] > 0]
    seg = np.asarray([int(orc.off[h]) for h in sk_heads], np.int64)

    def note(key, errs):
        for suffix, e in zip(("", "_head", "_elem"), errs):
            worst[key + suffix] = max(worst[key + suffix], e)

    def cmp_state():
        torch.cuda.synchronize()
        note("S", _slab_errors(gpu.S.index_select(0, ridx).cpu().numpy(), orc.S))
        if orc.rtot:
            note("Y", _slab_errors(gpu.Y.index_select(0, ridx).cpu().numpy(), orc.Y, seg))

    gpu.flush(0)
    orc.flush(0)
    cmp_state()
    pos = 0
    for t in range(1, T + 1):
        inp = synth.step_inputs(cfg, t - 1, range(cfg.B), layer)
        d = to_dev(inp)
        if dense:
            y = gpu.dense_decode(pos, d["q"], d["k"], d["v"], d["a"], d["beta"])
        else:
            y = gpu.decode(pos, d["q"], d["k"], d["v"], d["a"], d["beta"])
        yo = orc.decode(pos, {k: (None if v is None else v[rows]) for k, v in inp.items()},
                        dense_all=dense)
        note("y", _slab_errors(y.index_select(0, ridx).cpu().numpy(), yo))
        pos += 1
        if t in flush_at:
            gpu.flush(pos)
            orc.flush(pos)
            cmp_state()
            pos = 0
        assert pos < cfg.W, "flush schedule leaves more than W tokens buffered"
    torch.cuda.synchronize()
    gpu.close()
    REPORT.append({"name": name or cfg.name, "workload": cfg.name, "kind": cfg.kind, "batch": cfg.B,
                   "rows_checked": len(rows), "steps": T, "dense_read": dense, "layer": layer,
                   **{k: float(f"{v:.3e}") for k, v in worst.items()}})
    for k in ("y", "S", "Y", "y_head", "S_head", "Y_head"):
        assert worst[k] <= tol, f"{k}: max relative error {worst[k]:.3e} > {tol:.0e} ({cfg.name})"
    return worst


def write_report(path: str) -> None:
    """Write the session's parity records (JSON) to ``path``."""
    os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
    with open(path, "w") as f:
        json.dump(REPORT, f, indent=1)
