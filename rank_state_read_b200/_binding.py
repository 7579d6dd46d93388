"""ctypes binding of libsketchssm (include/sketchssm.h): argument marshalling only.

Every step of the flush and decode runs in the library's CUDA kernels; this module
only turns torch tensors into device pointers and status codes into exceptions.
PyTorch supplies the device memory and the stream.  If the library has not been
built, loading fails loudly: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libsketchssm.so")

DENSE = -1
KINDS = {"mamba2": 0, "gdn": 1, "kda": 2}
STATUS = {0: "SKETCHSSM_OK", 1: "SKETCHSSM_ERR_INVALID_ARG", 2: "SKETCHSSM_ERR_ALIGNMENT",
          3: "SKETCHSSM_ERR_UNSUPPORTED", 4: "SKETCHSSM_ERR_CUDA", 5: "SKETCHSSM_ERR_TIMEOUT"}

# every symbol include/sketchssm.h declares
EXPORTS = ("sketchssm_plan_create", "sketchssm_plan_query", "sketchssm_plan_check",
           "sketchssm_plan_set_wait_limit", "sketchssm_plan_destroy", "sketchssm_flush", "sketchssm_decode", "sketchssm_dense_decode",
           "sketchssm_decode_static_scratch", "sketchssm_step", "sketchssm_decode_rows",
           "sketchssm_flush_rows", "sketchssm_prefill", "sketchssm_status_string", "sketchssm_last_error")


class SketchSSMError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")


class Desc(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in
                ("kind", "batch", "heads", "qk_heads", "key_dim", "value_dim", "window", "groups",
                 "basis_rows", "rank_cap")]


_lib = None


def load():
    """Load libsketchssm.so (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m rank_state_read_b200.build` "
                           "(nvcc, sm_100a); there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.sketchssm_plan_create.argtypes = [ctypes.POINTER(Desc), P, P, P, ctypes.POINTER(P)]
    lib.sketchssm_plan_query.argtypes = [P, ctypes.POINTER(I64), P, P, I32, P, ctypes.POINTER(I32)]
    lib.sketchssm_plan_check.argtypes = [P, P]
    lib.sketchssm_plan_set_wait_limit.argtypes = [P, I64]
    lib.sketchssm_plan_destroy.argtypes = [P]
    lib.sketchssm_flush.argtypes = [P, P, P, P, P, P, P, I32, P, P]
    lib.sketchssm_decode.argtypes = [P, I32, P, P, P, P, P, P, P, P, P, P, P, P, P, P]
    lib.sketchssm_dense_decode.argtypes = [P, I32, P, P, P, P, P, P, P, P, P, P, P, P]
    lib.sketchssm_decode_static_scratch.argtypes = [P, I32, P, P, P, P, P, P, P, P, P, P, P, P, P, P]
    lib.sketchssm_step.argtypes = [P, P, P, P, P, P, P, P, P]
    lib.sketchssm_decode_rows.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P]
    lib.sketchssm_flush_rows.argtypes = [P, P, P, P, P, P, P, P, P, P]
    lib.sketchssm_prefill.argtypes = [P, I32, P, P, P, P, P, P, P, P]
    for f in EXPORTS[:13]:
        getattr(lib, f).restype = ctypes.c_int
    lib.sketchssm_status_string.argtypes = [ctypes.c_int]
    lib.sketchssm_status_string.restype = ctypes.c_char_p
    lib.sketchssm_last_error.argtypes = []
    lib.sketchssm_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise SketchSSMError(status, where, load().sketchssm_last_error().decode())


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], name: str, numel: Optional[int] = None):
    if t is None or (numel == 0 and t.numel() == 0):
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return t.data_ptr()


class Plan:
    """A layer shape at a fixed batch plus its rank table (sketchssm_plan)."""

    def __init__(self, kind: str, *, batch: int, heads: int, qk_heads: int, key_dim: int,
                 value_dim: int, window: int, groups: int, basis_rows: int, rank_cap: int,
                 rank: Sequence[int], group: Optional[Sequence[int]] = None, stream=None):
        lib = load()
        self.kind = kind
        self.desc = Desc(KINDS[kind], batch, heads, qk_heads, key_dim, value_dim, window, groups,
                         basis_rows, rank_cap)
        if len(rank) != heads:
            raise ValueError("rank table must have one entry per head")
        rank_arr = (ctypes.c_int32 * heads)(*[int(r) for r in rank])
        group_arr = None
        if group is not None:
            if len(group) != heads:
                raise ValueError("group table must have one entry per head")
            group_arr = (ctypes.c_int32 * heads)(*[int(g) for g in group])
        handle = ctypes.c_void_p()
        _check(lib.sketchssm_plan_create(ctypes.byref(self.desc), ctypes.cast(rank_arr, ctypes.c_void_p),
                                         None if group_arr is None else ctypes.cast(group_arr, ctypes.c_void_p),
                                         _stream(stream), ctypes.byref(handle)), "sketchssm_plan_create")
        self.handle = handle
        self.rank = [int(r) for r in rank]
        rt = ctypes.c_int64()
        off = (ctypes.c_int32 * (heads + 1))()
        rmax = (ctypes.c_int32 * groups)()
        _check(lib.sketchssm_plan_query(handle, ctypes.byref(rt), ctypes.cast(off, ctypes.c_void_p),
                                        ctypes.cast(rmax, ctypes.c_void_p), 1, None, None),
               "sketchssm_plan_query")
        self.r_total = int(rt.value)
        self.offsets = list(off)
        self.rmax = list(rmax)
        self.work = {}
        for n in range(1, window + 1):
            nw = ctypes.c_int32()
            work = (ctypes.c_int32 * (groups + heads))()
            _check(lib.sketchssm_plan_query(handle, None, None, None, n,
                                            ctypes.cast(work, ctypes.c_void_p), ctypes.byref(nw)),
                   "sketchssm_plan_query")
            self.work[n] = list(work)[: nw.value]

    # shapes of the caller-owned tensors (include/sketchssm.h, "Layouts")
    @property
    def shapes(self) -> dict:
        d = self.desc
        B, H, Q, K, V, W, G = d.batch, d.heads, d.qk_heads, d.key_dim, d.value_dim, d.window, d.groups
        kda = self.kind == "kda"
        return {"S": (B, H, K, V), "omega": (G, d.basis_rows, K), "Y": (B, self.r_total, V),
                "q": (B, Q, K), "k": (B, Q, K), "v": (B, H, V), "a": (B, H, K) if kda else (B, H),
                "beta": (B, H), "kbuf": (B, Q, W, K), "vbuf": (B, H, W, V),
                "abuf": (B, H, W, K) if kda else (B, H, W), "bbuf": (B, H, W), "y": (B, H, V)}

    def numel(self, name: str) -> int:
        n = 1
        for x in self.shapes[name]:
            n *= x
        return n

    def check(self, stream=None) -> None:
        """Synchronise and raise if a kernel recorded a timeout (sketchssm_plan_check)."""
        _check(load().sketchssm_plan_check(self.handle, _stream(stream)), "sketchssm_plan_check")

    def set_wait_limit(self, cycles: int) -> None:
        """Cycles a CTA waits for its own copies before it records a timeout
        (sketchssm_plan_set_wait_limit; default 2e9)."""
        _check(load().sketchssm_plan_set_wait_limit(self.handle, int(cycles)), "sketchssm_plan_set_wait_limit")

    def close(self) -> None:
        if getattr(self, "handle", None) is not None and self.handle.value:
            load().sketchssm_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def sketchssm_plan_create(kind: str, rank: Sequence[int], stream=None, **shape) -> Plan:
    return Plan(kind, rank=rank, stream=stream, **shape)


def sketchssm_plan_destroy(plan: Plan) -> None:
    plan.close()


def sketchssm_flush(plan: Plan, S, omega, kbuf, vbuf, abuf, bbuf, n_tokens: int, Y, stream=None) -> None:
    n = plan.numel
    _check(load().sketchssm_flush(
        plan.handle, _ptr(S, "S", n("S")), _ptr(omega, "omega", n("omega")),
        _ptr(kbuf, "kbuf", n("kbuf")), _ptr(vbuf, "vbuf", n("vbuf")), _ptr(abuf, "abuf", n("abuf")),
        _ptr(bbuf, "bbuf", n("bbuf")), int(n_tokens), _ptr(Y, "Y", n("Y")), _stream(stream)),
        "sketchssm_flush")


def sketchssm_decode(plan: Plan, pos: int, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, Y, omega, S, y,
                     stream=None) -> None:
    n = plan.numel
    _check(load().sketchssm_decode(
        plan.handle, int(pos), _ptr(q, "q", n("q")), _ptr(k, "k", n("k")), _ptr(v, "v", n("v")),
        _ptr(a, "a", n("a")), _ptr(beta, "beta", n("beta")), _ptr(kbuf, "kbuf", n("kbuf")),
        _ptr(vbuf, "vbuf", n("vbuf")), _ptr(abuf, "abuf", n("abuf")), _ptr(bbuf, "bbuf", n("bbuf")),
        _ptr(Y, "Y", n("Y")), _ptr(omega, "omega", n("omega")), _ptr(S, "S", n("S")),
        _ptr(y, "y", n("y")), _stream(stream)), "sketchssm_decode")


def sketchssm_dense_decode(plan: Plan, pos: int, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, S, y,
                           stream=None) -> None:
    n = plan.numel
    _check(load().sketchssm_dense_decode(
        plan.handle, int(pos), _ptr(q, "q", n("q")), _ptr(k, "k", n("k")), _ptr(v, "v", n("v")),
        _ptr(a, "a", n("a")), _ptr(beta, "beta", n("beta")), _ptr(kbuf, "kbuf", n("kbuf")),
        _ptr(vbuf, "vbuf", n("vbuf")), _ptr(abuf, "abuf", n("abuf")), _ptr(bbuf, "bbuf", n("bbuf")),
        _ptr(S, "S", n("S")), _ptr(y, "y", n("y")), _stream(stream)), "sketchssm_dense_decode")


def sketchssm_decode_static_scratch(plan: Plan, pos: int, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, Y, omega,
                                    S, y, stream=None) -> None:
    """sketchssm_decode with its scratch in the library's static device array (no allocation)."""
    n = plan.numel
    _check(load().sketchssm_decode_static_scratch(
        plan.handle, int(pos), _ptr(q, "q", n("q")), _ptr(k, "k", n("k")), _ptr(v, "v", n("v")),
        _ptr(a, "a", n("a")), _ptr(beta, "beta", n("beta")), _ptr(kbuf, "kbuf", n("kbuf")),
        _ptr(vbuf, "vbuf", n("vbuf")), _ptr(abuf, "abuf", n("abuf")), _ptr(bbuf, "bbuf", n("bbuf")),
        _ptr(Y, "Y", n("Y")), _ptr(omega, "omega", n("omega")), _ptr(S, "S", n("S")),
        _ptr(y, "y", n("y")), _stream(stream)), "sketchssm_decode_static_scratch")


def sketchssm_step(plan: Plan, q, k, v, a, beta, S, y, stream=None) -> None:
    """The standard per-step decode (sketchssm_step): S updated in place, y = S^T q."""
    n = plan.numel
    _check(load().sketchssm_step(
        plan.handle, _ptr(q, "q", n("q")), _ptr(k, "k", n("k")), _ptr(v, "v", n("v")), _ptr(a, "a", n("a")),
        _ptr(beta, "beta", n("beta")), _ptr(S, "S", n("S")), _ptr(y, "y", n("y")), _stream(stream)),
        "sketchssm_step")


def sketchssm_prefill(plan: Plan, T: int, k, v, a, beta, S, omega, Y, stream=None) -> None:
    """Prefill handoff (sketchssm_prefill): the prompt's T tokens applied to S in place,
    then Y formed from the new state.  k [B][T][Hqk][K], v [B][T][H][V], a [B][T][H]
    (KDA [B][T][H][K]), beta [B][T][H] (None for Mamba-2)."""
    d, n = plan.desc, plan.numel
    T = int(T)
    per_tok = {"k": d.batch * d.qk_heads * d.key_dim, "v": d.batch * d.heads * d.value_dim,
               "a": n("a"), "beta": d.batch * d.heads}
    if T == 0:
        k = v = a = beta = None
    _check(load().sketchssm_prefill(
        plan.handle, T, _ptr(k, "k", T * per_tok["k"]), _ptr(v, "v", T * per_tok["v"]),
        _ptr(a, "a", T * per_tok["a"]), _ptr(beta, "beta", T * per_tok["beta"]),
        _ptr(S, "S", n("S")), _ptr(omega, "omega", n("omega")), _ptr(Y, "Y", n("Y")), _stream(stream)),
        "sketchssm_prefill")


def _rows(t, name: str, B: int):
    if not isinstance(t, torch.Tensor) or t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous int32 CUDA tensor")
    if t.numel() != B:
        raise ValueError(f"{name} has {t.numel()} elements, expected {B}")
    return t.data_ptr()


def sketchssm_decode_rows(plan: Plan, pos, q, k, v, a, beta, kbuf, vbuf, abuf, bbuf, Y, omega, S, y,
                          stream=None) -> None:
    """sketchssm_decode with a buffer position per batch row (pos: int32 [B] on the device)."""
    n = plan.numel
    _check(load().sketchssm_decode_rows(
        plan.handle, _rows(pos, "pos", plan.desc.batch), _ptr(q, "q", n("q")), _ptr(k, "k", n("k")),
        _ptr(v, "v", n("v")), _ptr(a, "a", n("a")), _ptr(beta, "beta", n("beta")), _ptr(kbuf, "kbuf", n("kbuf")),
        _ptr(vbuf, "vbuf", n("vbuf")), _ptr(abuf, "abuf", n("abuf")), _ptr(bbuf, "bbuf", n("bbuf")),
        _ptr(Y, "Y", n("Y")), _ptr(omega, "omega", n("omega")), _ptr(S, "S", n("S")), _ptr(y, "y", n("y")),
        _stream(stream)), "sketchssm_decode_rows")


def sketchssm_flush_rows(plan: Plan, S, omega, kbuf, vbuf, abuf, bbuf, n_tokens, Y, stream=None) -> None:
    """sketchssm_flush with a token count per batch row (n_tokens: int32 [B] on the device)."""
    n = plan.numel
    _check(load().sketchssm_flush_rows(
        plan.handle, _ptr(S, "S", n("S")), _ptr(omega, "omega", n("omega")), _ptr(kbuf, "kbuf", n("kbuf")),
        _ptr(vbuf, "vbuf", n("vbuf")), _ptr(abuf, "abuf", n("abuf")), _ptr(bbuf, "bbuf", n("bbuf")),
        _rows(n_tokens, "n_tokens", plan.desc.batch), _ptr(Y, "Y", n("Y")), _stream(stream)),
        "sketchssm_flush_rows")
