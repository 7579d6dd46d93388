"""Seeded synthetic workloads shaped like the SketchSSM pages' layers.

Shapes and structure come from the pages:

* Nemotron-Nano-9B-v2 calibration card ("Contents" table): 27 recurrent layers,
  128 state heads per layer, K=128, V=80, 8 basis groups per layer, window W=16,
  rank cap 49, basis omega float32 of shape (27, 8, 79, 128).
* Same card, "Verified mean ranks" table: dense / sketch head counts over the
  3456 heads of the stack for mean ranks 4, 6, 10, 21.
* SketchSSM abstract: Mamba-2, Gated DeltaNet and KDA layers, fp32 state.

The pages publish no calibrated basis, rank table or activations, so every value
here is drawn from a seeded generator (numpy PCG64 through ``default_rng`` with a
list seed).  Each batch row of each step has its own stream, so any subset of rows
can be regenerated exactly without generating the others.

Nothing in this module computes any part of the method (no flush, no sketch, no
read); it only produces inputs.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional

import numpy as np

DENSE = -1  # rank-table value of a dense-fallback head

# stream tags (second element of every list seed)
_TAG_BASIS = 1
_TAG_INIT = 2
_TAG_RANKS = 3
_TAG_STEP = 4
_TAG_PROMPT = 5

KINDS = ("mamba2", "gdn", "kda")

# Dense heads per mean rank over the 27-layer, 3456-head Nemotron-Nano stack
# (calibration card, "Verified mean ranks" table).
STACK_DENSE_HEADS = {4: 12, 6: 30, 10: 230, 21: 775}


@dataclasses.dataclass(frozen=True)
class Config:
    cid: int
    name: str
    kind: str          # "mamba2" | "gdn" | "kda"
    B: int             # batch rows
    H: int             # state heads per layer
    G: int             # basis groups per layer (contiguous, H/G heads each)
    Hqk: int           # heads carrying q/k (G for group-shared Mamba-2 B/C, H per head)
    K: int             # key dim
    V: int             # value dim
    W: int             # buffer window
    Rb: int            # basis rows stored per group
    cap: int           # rank cap
    mean_rank: Optional[int]
    n_dense: int       # dense heads (over all layers)
    steps: int         # decode steps of the workload
    fixed_rank: Optional[int] = None  # every head has this rank (no draw)
    layers: int = 1
    seed: int = 0

    @property
    def kda(self) -> bool:
        return self.kind == "kda"

    @property
    def has_beta(self) -> bool:
        return self.kind in ("gdn", "kda")

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[int, Config] = {
    # tiny Mamba-2-style layer, every head rank 6, one group with a full 128x128 basis
    0: Config(0, "tiny-mamba2", "mamba2", B=4, H=8, G=1, Hqk=1, K=128, V=80, W=16,
              Rb=128, cap=128, mean_rank=6, n_dense=0, steps=64, fixed_rank=6,
              seed=10_000),
    # Nemotron-Nano-9B-v2-shaped Mamba-2 layer at batch 256
    1: Config(1, "nemotron-nano-mamba2-layer", "mamba2", B=256, H=128, G=8, Hqk=8,
              K=128, V=80, W=16, Rb=79, cap=49, mean_rank=6, n_dense=1, steps=1024,
              seed=10_001),
    # Gated DeltaNet-style layer
    3: Config(3, "gdn-layer", "gdn", B=512, H=32, G=4, Hqk=32, K=128, V=128, W=16,
              Rb=64, cap=64, mean_rank=8, n_dense=1, steps=1024, seed=10_003),
    # KDA-style layer (per-key-channel decay)
    4: Config(4, "kda-layer", "kda", B=1024, H=32, G=4, Hqk=32, K=128, V=128, W=16,
              Rb=64, cap=64, mean_rank=10, n_dense=1, steps=2048, seed=10_004),
}


def config(cid: int, *, mean_rank: int = 6, batch: int = 256) -> Config:
    """Return workload ``cid``.  ``cid == 2`` is one point of the 27-layer stack sweep
    (mean rank in {4, 6, 10, 21}, batch in {64, 256, 1024}, 256 steps)."""
    if cid == 2:
        if mean_rank not in STACK_DENSE_HEADS:
            raise ValueError(f"stack sweep has mean ranks {sorted(STACK_DENSE_HEADS)}")
        return Config(2, f"nemotron-nano-stack-r{mean_rank}-b{batch}", "mamba2", B=batch,
                      H=128, G=8, Hqk=8, K=128, V=80, W=16, Rb=79, cap=49,
                      mean_rank=mean_rank, n_dense=STACK_DENSE_HEADS[mean_rank],
                      steps=256, layers=27, seed=10_002 * 100 + mean_rank)
    return CONFIGS[cid]


# ----------------------------------------------------------------------------- ranks

def rank_table(seed: int, n_heads: int, mean_rank: int, n_dense: int, cap: int,
               fixed_rank: Optional[int] = None) -> np.ndarray:
    """Per-head rank table (int32, DENSE for dense-fallback heads).

    Sketch ranks are log-normal, r = clip(round(exp(N(ln m - 0.32, 0.8^2))), 1, cap)
    (exp(-0.32 + 0.8^2/2) = 1, so the draw has mean m before clipping), then a seeded
    +-1 repair on random heads makes the sum over sketch heads exactly m * (#sketch).
    Dense heads are a seeded choice of ``n_dense`` head indices.
    """
    rng = np.random.default_rng([seed, _TAG_RANKS])
    ranks = np.empty(n_heads, dtype=np.int32)
    dense = rng.choice(n_heads, size=n_dense, replace=False) if n_dense else np.empty(0, int)
    is_dense = np.zeros(n_heads, dtype=bool)
    is_dense[dense] = True
    sk = np.flatnonzero(~is_dense)
    if fixed_rank is not None:
        r = np.full(sk.size, fixed_rank, dtype=np.int64)
    else:
        z = rng.standard_normal(sk.size)
        r = np.clip(np.rint(np.exp(math.log(mean_rank) - 0.32 + 0.8 * z)), 1, cap).astype(np.int64)
        target = int(mean_rank) * sk.size
        if not (sk.size <= target <= cap * sk.size):
            raise ValueError("mean rank outside [1, cap]")
        total = int(r.sum())
        while total != target:
            i = int(rng.integers(sk.size))
            if total < target and r[i] < cap:
                r[i] += 1
                total += 1
            elif total > target and r[i] > 1:
                r[i] -= 1
                total -= 1
    ranks[sk] = r
    ranks[is_dense] = DENSE
    return ranks


def layer_rank_table(cfg: Config) -> np.ndarray:
    """Rank table of a one-layer config, int32 [H]."""
    if cfg.layers != 1:
        raise ValueError("use stack_rank_tables for multi-layer configs")
    return rank_table(cfg.seed, cfg.H, cfg.mean_rank, cfg.n_dense, cfg.cap, cfg.fixed_rank)


def stack_rank_tables(cfg: Config) -> np.ndarray:
    """Rank tables of every layer, int32 [layers][H]; drawn over the whole stack so that
    the dense-head count and the rank sum hold for the stack, as on the card."""
    t = rank_table(cfg.seed, cfg.layers * cfg.H, cfg.mean_rank, cfg.n_dense, cfg.cap,
                   cfg.fixed_rank)
    return t.reshape(cfg.layers, cfg.H)


# ----------------------------------------------------------------------------- basis

def basis(cfg: Config, layer: int = 0) -> np.ndarray:
    """Group-shared basis omega, float32 [G][Rb][K]: row i of group g is basis vector i.

    For each group, Q from the QR factorisation (fp64) of a seeded K x K Gaussian
    matrix; the rows of omega_g are the first Rb columns of Q, so they are orthonormal
    in fp64 and ordered.
    """
    return basis_fp64(cfg, layer).astype(np.float32)


def basis_fp64(cfg: Config, layer: int = 0) -> np.ndarray:
    out = np.empty((cfg.G, cfg.Rb, cfg.K), dtype=np.float64)
    for g in range(cfg.G):
        rng = np.random.default_rng([cfg.seed, _TAG_BASIS, layer, g])
        q, _ = np.linalg.qr(rng.standard_normal((cfg.K, cfg.K)))
        out[g] = q.T[: cfg.Rb]
    return out


# ----------------------------------------------------------------------------- state

def init_state(cfg: Config, rows: Iterable[int], layer: int = 0) -> np.ndarray:
    """Initial state S0 = 0.1 * N(0, 1), float32 [len(rows)][H][K][V]."""
    rows = list(rows)
    out = np.empty((len(rows), cfg.H, cfg.K, cfg.V), dtype=np.float32)
    for j, b in enumerate(rows):
        rng = np.random.default_rng([cfg.seed, _TAG_INIT, layer, b])
        out[j] = (0.1 * rng.standard_normal((cfg.H, cfg.K, cfg.V))).astype(np.float32)
    return out


# ----------------------------------------------------------------------------- tokens

def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def _unit_rows(z: np.ndarray) -> np.ndarray:
    return z / np.linalg.norm(z, axis=-1, keepdims=True)


def step_inputs(cfg: Config, step: int, rows: Iterable[int], layer: int = 0) -> dict:
    """Inputs of decode step ``step`` for the given batch rows (float32).

    q, k: [n][Hqk][K], L2-normalised Gaussian.   v: [n][H][V] ~ N(0, 1).
    a:    Mamba-2 / GDN: [n][H], exp(-softplus(N(0,1)) * 0.05);
          KDA: [n][H][K], 0.9 + 0.1 * U(0,1) kept strictly inside (0.9, 1) in fp32.
    beta: GDN / KDA: [n][H], sigmoid(N(0,1)); Mamba-2: None.
    """
    rows = list(rows)
    n = len(rows)
    q = np.empty((n, cfg.Hqk, cfg.K), np.float32)
    k = np.empty((n, cfg.Hqk, cfg.K), np.float32)
    v = np.empty((n, cfg.H, cfg.V), np.float32)
    a = np.empty((n, cfg.H, cfg.K) if cfg.kda else (n, cfg.H), np.float32)
    beta = np.empty((n, cfg.H), np.float32) if cfg.has_beta else None
    lo = np.nextafter(np.float32(0.9), np.float32(1.0))
    hi = np.nextafter(np.float32(1.0), np.float32(0.0))
    for j, b in enumerate(rows):
        rng = np.random.default_rng([cfg.seed, _TAG_STEP, layer, step, b])
        q[j] = _unit_rows(rng.standard_normal((cfg.Hqk, cfg.K)))
        k[j] = _unit_rows(rng.standard_normal((cfg.Hqk, cfg.K)))
        v[j] = rng.standard_normal((cfg.H, cfg.V))
        if cfg.kda:
            a[j] = np.clip((0.9 + 0.1 * rng.uniform(size=(cfg.H, cfg.K))).astype(np.float32), lo, hi)
        else:
            a[j] = np.exp(-_softplus(rng.standard_normal(cfg.H)) * 0.05)
        if beta is not None:
            beta[j] = 1.0 / (1.0 + np.exp(-rng.standard_normal(cfg.H)))
    return {"q": q, "k": k, "v": v, "a": a, "beta": beta}


def prompt_inputs(cfg: Config, T: int, rows: Iterable[int], layer: int = 0) -> dict:
    """A prompt of ``T`` tokens for the given batch rows (float32, token-major).

    k: [n][T][Hqk][K], v: [n][T][H][V], a: [n][T][H] (KDA [n][T][H][K]),
    beta: [n][T][H] (None for Mamba-2); every token drawn with the distributions of
    ``step_inputs`` (no query: a prompt only writes the state), from its own stream
    per (row, token).
    """
    rows = list(rows)
    n = len(rows)
    k = np.empty((n, T, cfg.Hqk, cfg.K), np.float32)
    v = np.empty((n, T, cfg.H, cfg.V), np.float32)
    a = np.empty((n, T, cfg.H, cfg.K) if cfg.kda else (n, T, cfg.H), np.float32)
    beta = np.empty((n, T, cfg.H), np.float32) if cfg.has_beta else None
    lo = np.nextafter(np.float32(0.9), np.float32(1.0))
    hi = np.nextafter(np.float32(1.0), np.float32(0.0))
    for j, b in enumerate(rows):
        for t in range(T):
            rng = np.random.default_rng([cfg.seed, _TAG_PROMPT, layer, t, b])
            k[j, t] = _unit_rows(rng.standard_normal((cfg.Hqk, cfg.K)))
            v[j, t] = rng.standard_normal((cfg.H, cfg.V))
            if cfg.kda:
                a[j, t] = np.clip((0.9 + 0.1 * rng.uniform(size=(cfg.H, cfg.K))).astype(np.float32), lo, hi)
            else:
                a[j, t] = np.exp(-_softplus(rng.standard_normal(cfg.H)) * 0.05)
            if beta is not None:
                beta[j, t] = 1.0 / (1.0 + np.exp(-rng.standard_normal(cfg.H)))
    return {"k": k, "v": v, "a": a, "beta": beta}


# ----------------------------------------------------------------------------- device draws

def device_state(cfg: Config, seed: int, device) -> "torch.Tensor":
    """S0 with the distribution of ``init_state`` drawn by torch's generator on
    ``device`` (other numbers than the numpy streams; for timing runs, where a
    full-batch state of several GB would take minutes to draw on the host)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    S = torch.empty((cfg.B, cfg.H, cfg.K, cfg.V), dtype=torch.float32, device=device)
    S.normal_(0.0, 0.1, generator=g)
    return S


def device_prompt_inputs(cfg: Config, T: int, seed: int, device) -> dict:
    """A prompt of ``T`` tokens with the distributions of ``prompt_inputs``, drawn on
    ``device`` (token-major, as ``prompt_inputs``)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    f32 = dict(dtype=torch.float32, device=device)
    z = torch.randn((cfg.B, T, cfg.Hqk, cfg.K), generator=g, **f32)
    out = {"k": z / z.norm(dim=-1, keepdim=True),
           "v": torch.randn((cfg.B, T, cfg.H, cfg.V), generator=g, **f32)}
    if cfg.kda:
        lo = float(np.nextafter(np.float32(0.9), np.float32(1.0)))
        hi = float(np.nextafter(np.float32(1.0), np.float32(0.0)))
        out["a"] = (0.9 + 0.1 * torch.rand((cfg.B, T, cfg.H, cfg.K), generator=g, **f32)).clamp_(lo, hi)
    else:
        out["a"] = torch.exp(-torch.nn.functional.softplus(torch.randn((cfg.B, T, cfg.H), generator=g, **f32)) * 0.05)
    out["beta"] = (torch.sigmoid(torch.randn((cfg.B, T, cfg.H), generator=g, **f32))
                   if cfg.has_beta else None)
    return out


def device_step_inputs(cfg: Config, seed: int, device) -> dict:
    """One step's inputs with the distributions of ``step_inputs``, drawn on ``device``."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    f32 = dict(dtype=torch.float32, device=device)

    def unit(shape):
        z = torch.randn(shape, generator=g, **f32)
        return z / z.norm(dim=-1, keepdim=True)

    out = {"q": unit((cfg.B, cfg.Hqk, cfg.K)), "k": unit((cfg.B, cfg.Hqk, cfg.K)),
           "v": torch.randn((cfg.B, cfg.H, cfg.V), generator=g, **f32)}
    if cfg.kda:
        lo = float(np.nextafter(np.float32(0.9), np.float32(1.0)))
        hi = float(np.nextafter(np.float32(1.0), np.float32(0.0)))
        out["a"] = (0.9 + 0.1 * torch.rand((cfg.B, cfg.H, cfg.K), generator=g, **f32)).clamp_(lo, hi)
    else:
        z = torch.randn((cfg.B, cfg.H), generator=g, **f32)
        out["a"] = torch.exp(-torch.nn.functional.softplus(z) * 0.05)
    out["beta"] = (torch.sigmoid(torch.randn((cfg.B, cfg.H), generator=g, **f32))
                   if cfg.has_beta else None)
    return out
