#!/usr/bin/env python
"""Benchmark of the SketchSSM decode hot path ("write full, read sketch") on B200.

Workload: the Nemotron-Nano-9B-v2-shaped Mamba-2 layer (128 heads, K=128, V=80,
8 basis groups, rank cap 49, mean rank 6, one dense-fallback head, W=16) at batch
256 per GPU, synthetic seeded inputs.  One step = one window cycle of the whole hot
path on every layer replica: W=16 sketch-decode launches, each followed on the last
position by the flush (state update + sketch projection), i.e. B*W tokens per
replica.  Layer replicas (default 8, about 1.8 GB each) rotate so that no decode
finds its layer's data in the 126 MB L2 from the previous step.

Printed JSON line (rank 0): value = tokens per second per SSM layer over all ranks,
device time (CUDA events, max over ranks), plus the per-kernel roofline of the
dominant kernel, the dense-read decode baseline, an end-to-end number through the
C ABI with host-resident inputs, the fp64 CPU oracle timed on the host cores, and
the prefill handoff (a 64-token prompt applied to the state, then its sketch) with the
prefill kernel's rate against the FP32 pipe's peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode tok/s per SSM layer at batch 256; HBM GB/s vs peak; speedup vs dense read"
UNIT = "tok/s"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------- bytes

def token_bytes(cfg) -> int:
    """Bytes of one buffered token of one batch row: k (per q/k head), v, a, beta."""
    da = cfg.K if cfg.kda else 1
    return 4 * (cfg.Hqk * cfg.K + cfg.H * cfg.V + cfg.H * da + (cfg.H if cfg.has_beta else 0))


def omega_bytes(cfg, rank) -> int:
    Hg = cfg.H // cfg.G
    rmax = [max([int(r) for r in rank[g * Hg:(g + 1) * Hg] if r > 0], default=0) for g in range(cfg.G)]
    return 4 * cfg.K * sum(rmax)


def decode_bytes(cfg, rank, pos: int) -> int:
    """Algorithmic HBM bytes of one sketch-decode launch at buffer position pos:
    per row the sketch rows of the sketch heads, the state of the dense heads, q, the
    step's token (read, then appended), the pos earlier buffered tokens and y; plus
    the basis rows once per launch."""
    sk = [int(r) for r in rank if r > 0]
    nd = sum(1 for r in rank if r <= 0)
    row = (4 * cfg.V * sum(sk) + 4 * nd * cfg.K * cfg.V + 4 * cfg.Hqk * cfg.K
           + (2 + pos) * token_bytes(cfg) + 4 * cfg.H * cfg.V)
    return cfg.B * row + omega_bytes(cfg, rank)


def dense_decode_bytes(cfg, pos: int) -> int:
    """Same for the dense-read decode: the full state of every head instead of the sketch."""
    row = (4 * cfg.H * cfg.K * cfg.V + 4 * cfg.Hqk * cfg.K + (2 + pos) * token_bytes(cfg)
           + 4 * cfg.H * cfg.V)
    return cfg.B * row


def step_bytes(cfg) -> int:
    """Algorithmic HBM bytes of one standard per-step decode launch: the state read and
    written, plus q, k (per q/k head), v, a, beta read and y written, per batch row."""
    da = cfg.K if cfg.kda else 1
    per_row = (2 * cfg.H * cfg.K * cfg.V + 2 * cfg.Hqk * cfg.K + 2 * cfg.H * cfg.V + cfg.H * da
               + (cfg.H if cfg.has_beta else 0))
    return 4 * cfg.B * per_row


PREFILL_T = 64        # prompt tokens of the timed prefill handoff
FP32_LANES_PER_SM = 128
SMS = 148


def prefill_instr(cfg, T: int) -> int:
    """Algorithmic FP32 lane instructions of one prefill launch: the fewest FMA-pipe
    instructions per state element and prompt token of the forms of the recurrence
    written out here.  Mamba-2 1: over a chunk S <- P S + sum_i (w_i k_i) v_i^T, one
    FMA per element and token (the per-chunk scale and key scaling are extra).  GDN 2:
    with the decay carried as a running scale, k^T S is one FMA and the rank-one write
    another.  KDA 3: its decay differs per key row, so the write takes two FMAs (the
    erase term and the new value) besides the k^T S one."""
    per = {"mamba2": 1, "gdn": 2, "kda": 3}[cfg.kind]
    return per * cfg.B * cfg.H * cfg.K * cfg.V * T


def flush_bytes(cfg, rank, n: int) -> int:
    """One flush of n buffered tokens: the state read and written once, the n tokens
    read, the sketch written; plus the basis rows once per launch."""
    sk = sum(int(r) for r in rank if r > 0)
    row = 2 * 4 * cfg.H * cfg.K * cfg.V + n * token_bytes(cfg) + 4 * cfg.V * sk
    return cfg.B * row + omega_bytes(cfg, rank)


def decode_launches(cfg) -> int:
    """Kernel launches of one sketch-decode call: the products kernel (Mamba-2) or the
    coefficient kernel (GDN / KDA), then the combine."""
    return 2


# ----------------------------------------------------------------------------- environment

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s)"


def kernel_traffic(kernel: str, workload: str = "nemotron-nano-mamba2-layer"):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary,
    if the kernel's source is unchanged since the counters were taken (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[f"{kernel}@{workload}"]
        for src_rel, sha in rec["sources"].items():
            src = os.path.join(ROOT, src_rel)
            if hashlib.sha256(open(src, "rb").read()).hexdigest() != sha:
                return None
        return rec
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = ["-i", str(self.device_index)]
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.out.read())) if len(r) >= 9]
        self.out.close()
        os.unlink(self.out.name)
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle

def oracle_cycles(cfg, rank, omega, rows, min_s: float, max_cycles: int):
    """Time whole window cycles (W decodes + the flush) of the fp64 oracle on `rows`."""
    import oracle
    S0 = synth.init_state(cfg, rows)
    layer = oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                               rank=rank, omega=omega, S0=S0)
    steps = [synth.step_inputs(cfg, t, rows) for t in range(cfg.W)]
    layer.flush(0)
    cycles, t0 = 0, time.perf_counter()
    while True:
        for p in range(cfg.W):
            layer.decode(p, steps[p])
        layer.flush(cfg.W)
        cycles += 1
        el = time.perf_counter() - t0
        if el >= min_s or cycles >= max_cycles:
            return cycles, el, oracle.num_threads()


def cpu_baseline(cfg, rank, omega) -> dict:
    """The oracle on every host core over the whole batch (about 10 s), then on one
    core over 8 batch rows (about 4 s; rows are independent, so tok/s compares)."""
    import oracle
    rows = list(range(cfg.B))
    cycles, el, threads = oracle_cycles(cfg, rank, omega, rows, min_s=10.0, max_cycles=64)
    tok = cfg.B * cfg.W * cycles
    oracle.set_num_threads(1)
    try:
        rows1 = rows[:8]
        c1, el1, _ = oracle_cycles(cfg, rank, omega, rows1, min_s=4.0, max_cycles=64)
    finally:
        oracle.set_num_threads(threads)
    return {"value": tok / el, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{cycles} window cycle(s) ({cycles * cfg.W} decode steps + {cycles} flushes) "
                      f"of one layer at batch {cfg.B}, fp64, {el:.1f} s",
            "value_1_core": len(rows1) * cfg.W * c1 / el1,
            "sample_1_core": f"{c1} window cycle(s) of {len(rows1)} batch rows on one core, {el1:.1f} s"}


# ----------------------------------------------------------------------------- ranks

def replica_seed(rank_id: int, replica: int) -> int:
    """Seed of one layer replica on one rank: every rank owns its own batch rows."""
    return 1_000_003 * (rank_id + 1) + 7919 * replica


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a group)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


# ----------------------------------------------------------------------------- GPU arm

class Replicas:
    """L independent layer replicas of one workload on one GPU (each more than 1 GB, so
    that no launch finds its layer's data in the 126 MB L2), with W steps of inputs
    each, and the timing loops of the hot path and its baselines.  Every loop records a
    CUDA event pair around every launch it times, on the launching stream."""

    def __init__(self, cfg, L: int, rank_id: int, dev, seed_base: int = 0):
        import torch
        import rank_state_read_b200 as rs
        self.cfg, self.dev = cfg, dev
        self.stream = torch.cuda.current_stream()
        self.rank = synth.layer_rank_table(cfg)
        self.omega = synth.basis(cfg)
        self.layers, self.inputs = [], []
        for l in range(L):
            seed = replica_seed(rank_id, seed_base + l)
            S0 = synth.device_state(cfg, seed, dev)
            self.layers.append(rs.SketchLayer(cfg.kind, batch=cfg.B, heads=cfg.H, qk_heads=cfg.Hqk,
                                              key_dim=cfg.K, value_dim=cfg.V, window=cfg.W, groups=cfg.G,
                                              rank_cap=cfg.cap, rank=self.rank.tolist(), omega=self.omega,
                                              S0=S0, device=dev))
            self.inputs.append([synth.device_step_inputs(cfg, seed + 1 + p, dev) for p in range(cfg.W)])
            del S0
        for lay in self.layers:
            lay.flush(0)
        torch.cuda.synchronize()

    def _ev(self):
        import torch
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    def cycle(self, dense=False, events=None):
        """One window cycle on every replica: W decodes (the sketch decode, or the
        dense-read decode), the last followed by the flush (sketch decode only)."""
        cfg = self.cfg
        for p in range(cfg.W):
            for l, lay in enumerate(self.layers):
                x = self.inputs[l][p]
                e0 = self._ev() if events is not None else None
                if dense:
                    lay.dense_decode(p, x["q"], x["k"], x["v"], x["a"], x["beta"])
                else:
                    lay.decode(p, x["q"], x["k"], x["v"], x["a"], x["beta"])
                if events is not None:
                    events["decode"].append((p, e0, self._ev()))
                if p == cfg.W - 1 and not dense:
                    e2 = self._ev() if events is not None else None
                    lay.flush(cfg.W)
                    if events is not None:
                        events["flush"].append((cfg.W, e2, self._ev()))

    def dense_cycles(self, k: int):
        """k dense-read cycles; their buffered tokens are then applied (untimed)."""
        import torch
        ev = {"decode": [], "flush": []}
        for _ in range(k):
            self.cycle(dense=True, events=ev)
        for lay in self.layers:
            lay.flush(self.cfg.W)
        torch.cuda.synchronize()
        return [(p, a, b) for p, a, b in ev["decode"]]

    def standard_steps(self, k: int):
        """k x W standard per-step decodes on every replica (same tokens)."""
        import torch
        out = []
        for _ in range(k):
            for p in range(self.cfg.W):
                for l, lay in enumerate(self.layers):
                    x = self.inputs[l][p]
                    e0 = self._ev()
                    lay.standard_step(x["q"], x["k"], x["v"], x["a"], x["beta"])
                    out.append((e0, self._ev()))
        torch.cuda.synchronize()
        return out

    def close(self):
        for lay in self.layers:
            lay.close()
        self.layers, self.inputs = [], []


def _mean_ms(pairs):
    return sum(a.elapsed_time(b) for a, b in pairs) / len(pairs)


def kernel_roof(kernel, achieved, nbytes_per_launch, peak, peak_src, workload):
    tr = kernel_traffic(kernel, workload)
    return {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": peak_src,
            "algorithmic_bytes_per_launch": int(nbytes_per_launch),
            "traffic": None if tr is None else tr["dram_bytes_per_launch_full_size"]}


def family_record(reps: Replicas, cycles: int, peak: float, peak_src: str, barrier) -> dict:
    """Decode, flush, dense-read decode and standard step of one workload: mean device
    time per launch (CUDA events), algorithmic GB/s and fraction of the HBM peak, DRAM
    traffic per launch from the committed ncu record when its source is unchanged."""
    cfg, rank = reps.cfg, reps.rank
    ev = {"decode": [], "flush": []}
    barrier()
    for _ in range(cycles):
        reps.cycle(events=ev)
    barrier()
    dec = [(p, a.elapsed_time(b)) for p, a, b in ev["decode"]]
    fl = [a.elapsed_time(b) for _, a, b in ev["flush"]]
    dd = [(p, a.elapsed_time(b)) for p, a, b in reps.dense_cycles(max(1, cycles // 2))]
    barrier()
    st = reps.standard_steps(1)
    barrier()
    dec_us = 1e3 * sum(t for _, t in dec) / len(dec)
    fl_us = 1e3 * sum(fl) / len(fl)
    dd_us = 1e3 * sum(t for _, t in dd) / len(dd)
    st_us = 1e3 * _mean_ms(st)
    dec_b = sum(decode_bytes(cfg, rank, p) for p, _ in dec) / len(dec)
    dd_b = sum(dense_decode_bytes(cfg, p) for p, _ in dd) / len(dd)
    fl_b = flush_bytes(cfg, rank, cfg.W)
    gbs = lambda nbytes, us: nbytes / (us * 1e-6) / 1e9
    w = cfg.name
    return {
        "workload": w, "kind": cfg.kind, "batch": cfg.B, "heads": cfg.H, "K": cfg.K, "V": cfg.V,
        "groups": cfg.G, "qk_heads": cfg.Hqk, "mean_rank": cfg.mean_rank,
        "dense_heads": int((rank < 0).sum()), "layer_replicas": len(reps.layers), "window_cycles": cycles,
        "decode": {"us": round(dec_us, 2), **kernel_roof("sketchssm_decode", gbs(dec_b, dec_us), dec_b, peak,
                                                         peak_src, w),
                   "launches_per_call": decode_launches(cfg)},
        "flush": {"us": round(fl_us, 2), **kernel_roof("sketchssm_flush", gbs(fl_b, fl_us), fl_b, peak, peak_src, w)},
        "dense_read": {"us": round(dd_us, 2), **kernel_roof("sketchssm_dense_decode", gbs(dd_b, dd_us), dd_b, peak,
                                                             peak_src, w)},
        "standard_step": {"us": round(st_us, 2), **kernel_roof("sketchssm_step", gbs(step_bytes(cfg), st_us),
                                                                step_bytes(cfg), peak, peak_src, w)},
        "window_tok_s": round(cfg.B * cfg.W / ((cfg.W * dec_us + fl_us) * 1e-6), 1),
        "speedup_vs_dense_read": round(dd_us / dec_us, 3),
        "traffic_ratio_dense_over_sketch": round(dd_b / dec_b, 3),
        "speedup_vs_standard_step": round(cfg.W * st_us / (cfg.W * dec_us + fl_us), 3),
        "state_traffic": state_traffic(cfg, rank),
    }


def state_traffic(cfg, rank) -> dict:
    """DRAM bytes per token of the sketch path (W decodes + the flush, over W tokens)
    against the standard per-step decode, from the committed ncu record (all bytes the
    kernels moved, the token buffers included), beside the same ratio for the state
    alone counted from the shapes (the pages' figure is about 10x)."""
    B, H, K, V, W = cfg.B, cfg.H, cfg.K, cfg.V, cfg.W
    sk_rows = int(rank[rank > 0].sum())
    nd = int((rank <= 0).sum())
    st_state = 2 * H * K * V * 4
    sk_state = (sk_rows * V + nd * K * V) * 4 + (2 * H * K * V + sk_rows * V) * 4 / W
    out = {"analytic_state_bytes_per_token": {"standard_step": st_state, "sketch_path": round(sk_state, 1),
                                              "ratio": round(st_state / sk_state, 2)},
           "pages_ratio": "about 10x (mean sketch rank 8)"}
    dec = kernel_traffic("sketchssm_decode", cfg.name)
    fl = kernel_traffic("sketchssm_flush", cfg.name)
    st = kernel_traffic("sketchssm_step", cfg.name)
    if dec and fl and st:
        sk = (W * dec["dram_bytes_per_launch_full_size"] + fl["dram_bytes_per_launch_full_size"]) / (W * B)
        std = st["dram_bytes_per_launch_full_size"] / B
        out["measured_dram_bytes_per_token"] = {"standard_step": round(std, 1), "sketch_path": round(sk, 1),
                                                "ratio": round(std / sk, 2),
                                                "source": "profiles/ncu_traffic.json"}
    else:
        out["measured_dram_bytes_per_token"] = None
    return out


def run_ours(args, cfg) -> None:
    import torch
    import torch.distributed as dist
    import rank_state_read_b200 as rs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank_id = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    reps = Replicas(cfg, args.replicas, rank_id, dev)
    stream = reps.stream
    rank, omega, layers, inputs = reps.rank, reps.omega, reps.layers, reps.inputs
    L = len(layers)

    for _ in range(args.warmup):
        reps.cycle()
    barrier()

    # ---- timed region: K steps of the hot path
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ev = {"decode": [], "flush": []}
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        reps.cycle(events=ev)
    t_end.record(stream)
    barrier()
    clocks = sampler.stop()
    ms = t_start.elapsed_time(t_end)
    dec = [(p, a.elapsed_time(b)) for p, a, b in ev["decode"]]
    fl = [b_.elapsed_time(c_) for _, b_, c_ in ev["flush"]]
    launches = decode_launches(cfg) * len(ev["decode"]) + len(ev["flush"])

    # ---- dense-read baseline decode (same positions, same replicas)
    kd = max(1, min(args.steps, 10))
    barrier()
    dd = [(p, a.elapsed_time(b)) for p, a, b in reps.dense_cycles(kd)]
    # ---- standard per-step decode (full state read and updated every token), the
    # baseline the pages' speedups are quoted against: same replicas, same tokens
    barrier()
    st = [a.elapsed_time(b) for a, b in reps.standard_steps(kd)]
    barrier()

    # ---- prefill handoff on replica 0: a prompt of PREFILL_T tokens applied to the state,
    # then the sketch formed (sketchssm_prefill); the kernel alone = the call with the
    # prompt minus the call with none (which only forms the sketch)
    prompt = synth.device_prompt_inputs(cfg, PREFILL_T, replica_seed(rank_id, 99), dev)
    pf_ev = {PREFILL_T: [], 0: []}
    barrier()
    for it in range(4):
        for T in (PREFILL_T, 0):
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if T:
                layers[0].prefill(prompt["k"], prompt["v"], prompt["a"], prompt["beta"])
            else:
                rs.sketchssm_prefill(layers[0].plan, 0, None, None, None, None, layers[0].S, layers[0].omega,
                                     layers[0].Y)
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(stream)
            if it:  # the first round warms up
                pf_ev[T].append((e0, e1))
    barrier()
    pf_us = {T: 1e3 * sum(a.elapsed_time(b) for a, b in ev_) / len(ev_) for T, ev_ in pf_ev.items()}
    del prompt

    # ---- end to end through the C ABI: every decode's inputs copied in from pinned host
    # memory on one stream, its y copied out to pinned host memory on another (PCIe
    # carries both directions at once), ordered by events; two device input slots
    cin = torch.cuda.Stream(device=dev)
    cout = torch.cuda.Stream(device=dev)
    host_in = [{k: (None if v is None else v.cpu().pin_memory()) for k, v in inputs[0][p].items()}
               for p in range(cfg.W)]
    slots = [{k: (None if v is None else torch.empty_like(v)) for k, v in inputs[0][0].items()} for _ in range(2)]
    ready = [torch.cuda.Event() for _ in range(2)]   # a slot's inputs have landed
    used = [torch.cuda.Event() for _ in range(2)]    # the decode that read a slot has run
    ydone = [torch.cuda.Event() for _ in layers]     # a layer's y has been copied out
    host_y = [torch.empty(layers[0].y.shape, dtype=torch.float32).pin_memory() for _ in layers]
    ke = max(1, min(args.steps, 5))
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    cin.wait_event(e_start)
    cout.wait_event(e_start)
    h2d = d2h = 0
    s = 0
    for _ in range(ke):
        for p in range(cfg.W):
            for l, lay in enumerate(layers):
                slot = s & 1
                cin.wait_event(used[slot])
                with torch.cuda.stream(cin):
                    for k, v in host_in[p].items():
                        if v is not None:
                            slots[slot][k].copy_(v, non_blocking=True)
                            h2d += v.numel() * 4
                ready[slot].record(cin)
                stream.wait_event(ready[slot])
                stream.wait_event(ydone[l])
                x = slots[slot]
                y = lay.decode(p, x["q"], x["k"], x["v"], x["a"], x["beta"])
                used[slot].record(stream)
                cout.wait_stream(stream)
                with torch.cuda.stream(cout):
                    host_y[l].copy_(y, non_blocking=True)
                ydone[l].record(cout)
                d2h += y.numel() * 4
                if p == cfg.W - 1:
                    lay.flush(cfg.W)
                s += 1
    stream.wait_stream(cin)
    stream.wait_stream(cout)
    e_end.record(stream)
    barrier()
    e2e_ms = e_start.elapsed_time(e_end)
    reps.close()
    del reps, layers, inputs, slots

    # ---- the other families (GDN, KDA layers) under the same clock, smaller loops
    families = {}
    if not args.no_families:
        peak, peak_src = hbm_peak()
        for cid, key in ((3, "gdn"), (4, "kda")):
            fcfg = synth.config(cid)
            fr = Replicas(fcfg, args.family_replicas, rank_id, dev, seed_base=200 + cid)
            for _ in range(2):
                fr.cycle()
            families[key] = family_record(fr, args.family_cycles, peak, peak_src, barrier)
            fr.close()
            del fr
            torch.cuda.empty_cache()

    # ---- max over ranks
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)

    tokens = cfg.B * cfg.W * L * args.steps * world
    value = tokens / (ms / 1e3)
    e2e_value = cfg.B * cfg.W * L * ke * world / (e2e_ms / 1e3)

    peak, peak_src = hbm_peak()
    dec_ms = sum(t for _, t in dec)
    dec_bytes = sum(decode_bytes(cfg, rank, p) for p, _ in dec)
    fl_ms = sum(fl)
    fl_bytes = len(fl) * flush_bytes(cfg, rank, cfg.W)
    dd_ms = sum(t for _, t in dd)
    dd_bytes = sum(dense_decode_bytes(cfg, p) for p, _ in dd)
    dec_gbs = dec_bytes / (dec_ms / 1e3) / 1e9
    fl_gbs = fl_bytes / (fl_ms / 1e3) / 1e9
    dd_gbs = dd_bytes / (dd_ms / 1e3) / 1e9
    mean_dec_us = 1e3 * dec_ms / len(dec)
    mean_fl_us = 1e3 * fl_ms / len(fl)
    mean_dd_us = 1e3 * dd_ms / len(dd)
    mean_st_us = 1e3 * sum(st) / len(st)
    st_gbs = step_bytes(cfg) / (mean_st_us * 1e-6) / 1e9

    share_dec = dec_ms / (dec_ms + fl_ms)
    r_dec = kernel_roof("sketchssm_decode", dec_gbs, dec_bytes / len(dec), peak, peak_src, cfg.name)
    r_fl = kernel_roof("sketchssm_flush", fl_gbs, fl_bytes / len(fl), peak, peak_src, cfg.name)
    dominant, other = (r_dec, r_fl) if share_dec >= 0.5 else (r_fl, r_dec)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; shapes of the Nemotron Nano 9B v2 calibration card)",
        "config": {"workload": cfg.name, "kind": cfg.kind, "batch_per_gpu": cfg.B, "heads": cfg.H,
                   "K": cfg.K, "V": cfg.V, "groups": cfg.G, "qk_heads": cfg.Hqk, "window": cfg.W,
                   "rank_cap": cfg.cap, "mean_rank": cfg.mean_rank, "dense_heads": int((rank < 0).sum()),
                   "sketch_rows": int(rank[rank > 0].sum()), "layer_replicas": L,
                   "step": f"{cfg.W} sketch decodes + 1 flush per replica",
                   "l2": f"inputs larger than L2: {L} rotating layer replicas "
                         f"({L * 1.8:.0f} GB), no L2 flush",
                   "parallelism": f"batch sharded, {world} independent rank(s), no collective"},
        "roofline": dominant,
        "roofline_other": other,
        "kernel_share": {"sketchssm_decode": round(share_dec, 4), "sketchssm_flush": round(1 - share_dec, 4)},
        "decode_us": round(mean_dec_us, 2), "flush_us": round(mean_fl_us, 2),
        "decode_launches_per_call": decode_launches(cfg),
        "decode_only_tok_s": round(cfg.B * world / (mean_dec_us / 1e6), 1),
        "dense_read": {"decode_us": round(mean_dd_us, 2), "hbm_gbs": round(dd_gbs, 1),
                       "frac": round(dd_gbs / peak, 4),
                       "decode_only_tok_s": round(cfg.B * world / (mean_dd_us / 1e6), 1),
                       "traffic": (lambda tr: None if tr is None else tr["dram_bytes_per_launch_full_size"])(
                           kernel_traffic("sketchssm_dense_decode", cfg.name))},
        "speedup_vs_dense_read": round(mean_dd_us / mean_dec_us, 3),
        "traffic_ratio_dense_over_sketch": round(dd_bytes / len(dd) / (dec_bytes / len(dec)), 3),
        "standard_step": {"step_us": round(mean_st_us, 2), "hbm_gbs": round(st_gbs, 1),
                          "frac": round(st_gbs / peak, 4), "tok_s": round(cfg.B / (mean_st_us * 1e-6), 1),
                          "algorithmic_bytes_per_launch": step_bytes(cfg),
                          "traffic": (lambda tr: None if tr is None else tr["dram_bytes_per_launch_full_size"])(
                              kernel_traffic("sketchssm_step", cfg.name))},
        "speedup_vs_standard_step": round(cfg.W * mean_st_us / (cfg.W * mean_dec_us + mean_fl_us), 3),
        "state_traffic": state_traffic(cfg, rank),
        "prefill": prefill_report(cfg, pf_us, clocks, peak, peak_src),
        "configs": families,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d // ke,
                "d2h_bytes_per_step": d2h // ke,
                "note": "every decode: its inputs copied in from pinned host memory (torch copies on one "
                        "stream) before the C-ABI decode call on device pointers, y copied out to pinned "
                        "host memory on another stream; two input slots, event-ordered"},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank_id == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(cfg, rank, omega)
    if world > 1:
        dist.destroy_process_group()
    if rank_id == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- reference arm

def prefill_bytes(cfg, T: int) -> int:
    """Algorithmic HBM bytes of one prefill launch: the state read and written once, and
    the prompt's T tokens (k per q/k head, v, a, beta) read, per batch row."""
    da = cfg.K if cfg.kda else 1
    tok = 4 * (cfg.Hqk * cfg.K + cfg.H * cfg.V + cfg.H * da + (cfg.H if cfg.has_beta else 0))
    return cfg.B * (2 * 4 * cfg.H * cfg.K * cfg.V + T * tok)


def prefill_tensor_path(cfg, T: int) -> bool:
    """Whether the library applies this prompt on the tensor cores (the tcgen05 kernel:
    Mamba-2, at most 64 tokens, V a multiple of 16 up to 128)."""
    return cfg.kind == "mamba2" and 1 <= T <= 64 and cfg.V % 16 == 0 and cfg.V <= 128


def prefill_flops(cfg, T: int) -> dict:
    """Tensor-core work of one Mamba-2 prefill launch: the contraction's algorithmic
    FLOPs, 2 K V T per head, and the FLOPs the kernel issues, three tf32 products (hi/lo
    split) of M = 128 value rows (V padded) x N = K state rows x the prompt padded to 8."""
    heads = cfg.B * cfg.H
    tp = (T + 7) // 8 * 8
    return {"algorithmic": 2 * heads * cfg.K * cfg.V * T, "issued": 3 * 2 * heads * 128 * cfg.K * tp}


def tf32_peak():
    """Dense tf32 tensor peak: the measured bf16 burst figure x the nominal tf32/bf16
    ratio (1.1 / 2.25 PFLOP/s)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]) * 1.1 / 2.25, "measured bf16 burst x nominal tf32/bf16 ratio"
    except Exception:
        return 1590.0 * 1.1 / 2.25, "fallback bf16 (1.59 PFLOP/s) x nominal tf32/bf16 ratio"


def prefill_report(cfg, pf_us: dict, clocks: dict, peak: float, peak_src: str) -> dict:
    """The prefill handoff's line: its time, prompt tok/s, the prefill kernel's rate of
    algorithmic bytes against the HBM peak (its bound once its arithmetic keeps up), and
    the rate of its arithmetic: for the tensor-core (Mamba-2) kernel its FLOP rate
    against the tf32 tensor peak; otherwise its FP32 lane-instruction rate against the
    FP32 pipe's peak (148 SMs x 128 lanes x the SM clock)."""
    T = PREFILL_T
    k_us = max(pf_us[T] - pf_us[0], 1e-3)
    gbs = prefill_bytes(cfg, T) / (k_us * 1e-6) / 1e9
    rep = {"prompt_tokens": T, "handoff_us": round(pf_us[T], 2), "sketch_only_us": round(pf_us[0], 2),
           "kernel_us": round(k_us, 2), "prompt_tok_s": round(cfg.B * T / (pf_us[T] * 1e-6), 1),
           "roofline": {"kernel": "sketchssm_prefill", "bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                        "unit": "GB/s", "frac": round(gbs / peak, 4), "peak_source": peak_src,
                        "algorithmic_bytes_per_launch": prefill_bytes(cfg, T),
                        "traffic": (lambda tr: None if tr is None else tr["dram_bytes_per_launch_full_size"])(
                            kernel_traffic("sketchssm_prefill", cfg.name))}}
    if prefill_tensor_path(cfg, T):
        fl = prefill_flops(cfg, T)
        tp, tsrc = tf32_peak()
        rep["tensor"] = {"achieved": round(fl["algorithmic"] / (k_us * 1e-6) / 1e12, 2),
                         "issued": round(fl["issued"] / (k_us * 1e-6) / 1e12, 2), "peak": round(tp, 1),
                         "unit": "TFLOP/s", "frac_issued": round(fl["issued"] / (k_us * 1e-6) / 1e12 / tp, 4),
                         "peak_source": tsrc, "flops_per_launch": fl}
    else:
        mhz = clocks.get("sm_max_mhz") or 1965.0
        alu_peak = SMS * FP32_LANES_PER_SM * mhz * 1e6 / 1e12
        ach = prefill_instr(cfg, T) / (k_us * 1e-6) / 1e12
        rep["fp32_pipe"] = {"achieved": round(ach, 2), "peak": round(alu_peak, 2), "unit": "T FP32 lane-instr/s",
                            "frac": round(ach / alu_peak, 4), "algorithmic_instr_per_launch": prefill_instr(cfg, T)}
    return rep


def run_reference(args, cfg) -> None:
    """The reference arm of this pipeline is the fp64 CPU oracle as it stands: each
    step is one window cycle of the same layer on a bounded sample of batch rows."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    rank = synth.layer_rank_table(cfg)
    omega = synth.basis(cfg)
    rows = list(range(args.ref_rows))
    import oracle
    S0 = synth.init_state(cfg, rows)
    layer = oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                               rank=rank, omega=omega, S0=S0)
    steps = [synth.step_inputs(cfg, t, rows) for t in range(cfg.W)]
    layer.flush(0)

    def cycle():
        for p in range(cfg.W):
            layer.decode(p, steps[p])
        layer.flush(cfg.W)

    for _ in range(args.warmup):
        cycle()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cycle()
    el = time.perf_counter() - t0
    value = len(rows) * cfg.W * args.steps / el
    threads = oracle.num_threads()
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT,
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * el / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; shapes of the Nemotron Nano 9B v2 calibration card)",
            "config": {"workload": cfg.name, "kind": cfg.kind, "batch_per_gpu": cfg.B,
                       "rows_per_step": len(rows), "step": f"{cfg.W} decodes + 1 flush"},
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{len(rows)} of {cfg.B} batch rows per step, "
                                       f"{args.steps} window cycles"},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_case(args, cfg) -> None:
    """A small single-layer run for a profiler (ncu -k <kernel> -s <skip> -c <count>):
    flush(0), then `--steps` window cycles of W sketch decodes and a flush, then W
    dense-read decodes and a flush, then two standard per-step decodes and a prefill
    handoff of 32 tokens, with no timing and no JSON line.  Launch order: the initial
    flush; per cycle W sketch decodes (Mamba-2: one kernel each; GDN / KDA: the
    coefficient kernel and the combine) and the flush; W dense-read decodes (two
    kernels each) and the flush; the two step kernels; the prefill kernel and its flush."""
    import torch
    import rank_state_read_b200 as rs
    rank = synth.layer_rank_table(cfg)
    layer = rs.SketchLayer(cfg.kind, batch=cfg.B, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K,
                           value_dim=cfg.V, window=cfg.W, groups=cfg.G, rank_cap=cfg.cap,
                           rank=rank.tolist(), omega=synth.basis(cfg),
                           S0=synth.device_state(cfg, replica_seed(0, 0), "cuda"), device="cuda")
    xs = [synth.device_step_inputs(cfg, 1000 + p, "cuda") for p in range(cfg.W)]
    layer.flush(0)
    for _ in range(args.steps):
        for p in range(cfg.W):
            x = xs[p]
            layer.decode(p, x["q"], x["k"], x["v"], x["a"], x["beta"])
        layer.flush(cfg.W)
    for p in range(cfg.W):  # a window of dense-read decodes
        x = xs[p]
        layer.dense_decode(p, x["q"], x["k"], x["v"], x["a"], x["beta"])
    layer.flush(cfg.W)
    for p in range(2):  # then two standard per-step decodes (step_kernel)
        x = xs[p]
        layer.standard_step(x["q"], x["k"], x["v"], x["a"], x["beta"])
    pr = synth.device_prompt_inputs(cfg, 32, 7, "cuda")  # then a prefill handoff of 32 tokens
    layer.prefill(pr["k"], pr["v"], pr["a"], pr["beta"])
    torch.cuda.synchronize()
    layer.plan.check()
    layer.close()
    print(f"profile case done: config {args.config}, {args.steps} window cycle(s)", flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", type=int, default=1, choices=(0, 1, 3, 4))
    ap.add_argument("--replicas", type=int, default=8)
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-families", action="store_true", help="skip the GDN / KDA sub-records")
    ap.add_argument("--family-replicas", type=int, default=4)
    ap.add_argument("--family-cycles", type=int, default=6)
    ap.add_argument("--profile", action="store_true",
                    help="small single-layer run for a profiler: no timing, no JSON line")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args, synth.config(args.config))
        return
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    cfg = synth.config(args.config)
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
