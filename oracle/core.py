"""ctypes front end of the C oracle (test infrastructure only).

``OracleLayer`` keeps one layer's fp64 state, sketch and key/value buffers and runs
the decode / flush protocol of the SketchSSM paper abstract: tokens are buffered
for W steps (ReplaySSM), every decode step reads the sketch plus the buffer, and a
flush applies the buffer to the full state and re-forms the sketch.
"""
from __future__ import annotations

import ctypes
from typing import Iterable, Iterator, Optional

import numpy as np

from . import build as _build

KIND_ID = {"mamba2": 0, "gdn": 1, "kda": 2}

_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in ("kind", "B", "H", "Hqk", "K", "V", "W", "G", "Rb")]


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        lib.oracle_layout.restype = ctypes.c_int64
        lib.oracle_layout.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P, P]
        lib.oracle_flush.restype = None
        lib.oracle_flush.argtypes = [ctypes.POINTER(_Dims), P, P, ctypes.c_int64, P, P, P, P,
                                     P, P, ctypes.c_int32, P]
        lib.oracle_decode.restype = None
        lib.oracle_decode.argtypes = [ctypes.POINTER(_Dims), P, P, ctypes.c_int64,
                                      ctypes.c_int32, P, P, P, P, P, P, P, P, P, P, P, P,
                                      ctypes.c_int32, P]
        lib.oracle_step.restype = None
        lib.oracle_step.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P, P, P]
        lib.oracle_prefill.restype = None
        lib.oracle_prefill.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int32, P, P, P, P, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.restype = None
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Host threads of the oracle's loops from now on."""
    _load().oracle_set_num_threads(int(n))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def load_library(path: str):
    """Load an oracle build from ``path`` (the tests load mutated copies this way)."""
    global _lib
    saved = _lib
    try:
        _lib = None
        _build_path = _build.build
        _build.build = lambda: path
        return _load()
    finally:
        _build.build = _build_path
        _lib = saved


def layout(rank: np.ndarray, G: int, lib=None):
    """(off [H+1], rmax [G], Rtot) of a rank table; raises on an invalid rank."""
    rank = np.ascontiguousarray(rank, dtype=np.int32)
    H = rank.size
    off = np.zeros(H + 1, np.int32)
    rmax = np.zeros(G, np.int32)
    rtot = (lib or _load()).oracle_layout(H, G, _p(rank), _p(off), _p(rmax))
    if rtot < 0:
        raise ValueError("rank table holds a value that is neither DENSE nor >= 1")
    return off, rmax, int(rtot)


class OracleLayer:
    """One recurrent layer for a set of batch rows, all in fp64."""

    def __init__(self, kind: str, *, H: int, Hqk: int, K: int, V: int, W: int, G: int,
                 rank: np.ndarray, omega: np.ndarray, S0: np.ndarray, lib=None):
        self._lib = lib or _load()
        S0 = _f64(S0)
        B = S0.shape[0]
        assert S0.shape == (B, H, K, V)
        omega = _f64(omega)
        assert omega.ndim == 3 and omega.shape[0] == G and omega.shape[2] == K
        self.kind = kind
        self.dims = _Dims(KIND_ID[kind], B, H, Hqk, K, V, W, G, omega.shape[1])
        self.rank = np.ascontiguousarray(rank, dtype=np.int32)
        assert self.rank.shape == (H,)
        if (self.rank > omega.shape[1]).any():
            raise ValueError("rank above the stored basis rows")
        self.off, self.rmax, self.rtot = layout(self.rank, G, self._lib)
        self.omega = omega
        self.S = S0.copy()
        self.Y = np.zeros((B, self.rtot, V))
        self.kbuf = np.zeros((B, Hqk, W, K))
        self.vbuf = np.zeros((B, H, W, V))
        self.abuf = np.zeros((B, H, W, K) if kind == "kda" else (B, H, W))
        self.bbuf = np.zeros((B, H, W))

    @property
    def B(self) -> int:
        return self.dims.B

    def flush(self, n: int) -> None:
        """Apply buffer slots 0..n-1 to S, then re-form Y from the new S."""
        assert 0 <= n <= self.dims.W
        self._lib.oracle_flush(ctypes.byref(self.dims), _p(self.rank), _p(self.off), self.rtot,
                             _p(self.S), _p(self.omega), _p(self.kbuf), _p(self.vbuf),
                             _p(self.abuf), _p(self.bbuf), n, _p(self.Y))

    def prefill(self, prompt: dict) -> None:
        """Prefill handoff: apply the prompt's tokens to S in order (``prefill``), then
        form Y from the new state (the n = 0 flush).  The buffer is left alone."""
        prefill(self.kind, self.S, prompt, self.dims.Hqk, lib=self._lib)
        self.flush(0)

    def decode(self, pos: int, inp: dict, dense_all: bool = False) -> np.ndarray:
        """Append the step's token at slot ``pos`` and return y [B][H][V]."""
        assert 0 <= pos < self.dims.W
        d = self.dims
        q, k, v, a = (_f64(inp[x]) for x in ("q", "k", "v", "a"))
        beta = None if inp.get("beta") is None else _f64(inp["beta"])
        assert q.shape == (d.B, d.Hqk, d.K) and k.shape == q.shape and v.shape == (d.B, d.H, d.V)
        if self.kind != "mamba2":
            assert beta is not None and beta.shape == (d.B, d.H)
        y = np.empty((d.B, d.H, d.V))
        self._lib.oracle_decode(ctypes.byref(d), _p(self.rank), _p(self.off), self.rtot, pos,
                              _p(q), _p(k), _p(v), _p(a), _p(beta), _p(self.kbuf),
                              _p(self.vbuf), _p(self.abuf), _p(self.bbuf), _p(self.Y),
                              _p(self.omega), _p(self.S), int(dense_all), _p(y))
        return y


def standard_step(kind: str, S: np.ndarray, inp: dict, Hqk: int, lib=None) -> np.ndarray:
    """The per-step recurrent decode (no buffer, no sketch): apply the step's token to
    the fp64 state ``S`` [B][H][K][V] in place and return y = S^T q [B][H][V]."""
    assert S.dtype == np.float64 and S.flags.c_contiguous
    B, H, K, V = S.shape
    q, k, v, a = (_f64(inp[x]) for x in ("q", "k", "v", "a"))
    beta = None if inp.get("beta") is None else _f64(inp["beta"])
    assert q.shape == (B, Hqk, K) and k.shape == q.shape and v.shape == (B, H, V)
    if kind != "mamba2":
        assert beta is not None and beta.shape == (B, H)
    dims = _Dims(KIND_ID[kind], B, H, Hqk, K, V, 1, 1, 1)
    y = np.empty((B, H, V))
    (lib or _load()).oracle_step(ctypes.byref(dims), _p(S), _p(q), _p(k), _p(v), _p(a), _p(beta), _p(y))
    return y


def prefill(kind: str, S: np.ndarray, prompt: dict, Hqk: int, lib=None) -> None:
    """Apply a prompt's tokens to the fp64 state ``S`` [B][H][K][V] in place, in order.

    ``prompt`` is token-major: k [B][T][Hqk][K], v [B][T][H][V], a [B][T][H]
    (KDA [B][T][H][K]), beta [B][T][H] (None for Mamba-2)."""
    assert S.dtype == np.float64 and S.flags.c_contiguous
    B, H, K, V = S.shape
    k, v, a = (_f64(prompt[x]) for x in ("k", "v", "a"))
    beta = None if prompt.get("beta") is None else _f64(prompt["beta"])
    T = k.shape[1]
    assert k.shape == (B, T, Hqk, K) and v.shape == (B, T, H, V)
    assert a.shape == ((B, T, H, K) if kind == "kda" else (B, T, H))
    if kind != "mamba2":
        assert beta is not None and beta.shape == (B, T, H)
    dims = _Dims(KIND_ID[kind], B, H, Hqk, K, V, 1, 1, 1)
    (lib or _load()).oracle_prefill(ctypes.byref(dims), T, _p(S), _p(k), _p(v), _p(a), _p(beta))


def trajectory(layer: OracleLayer, inputs: Iterable[dict], *, dense_all: bool = False,
               initial_flush: bool = True) -> Iterator[tuple]:
    """Drive the decode / flush protocol over a sequence of step inputs.

    Yields ("flush", t, S, Y) after the initial n=0 flush (t = 0) and after every
    flush of W tokens (t = step count so far), and ("decode", t, y) for step t
    (1-based).  A flush follows the decode that fills slot W-1.
    """
    W = layer.dims.W
    if initial_flush:
        layer.flush(0)
        yield ("flush", 0, layer.S.copy(), layer.Y.copy())
    pos = 0
    for t, inp in enumerate(inputs, start=1):
        y = layer.decode(pos, inp, dense_all=dense_all)
        yield ("decode", t, y)
        pos += 1
        if pos == W:
            layer.flush(W)
            yield ("flush", t, layer.S.copy(), layer.Y.copy())
            pos = 0
