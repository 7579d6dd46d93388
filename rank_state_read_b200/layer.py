"""One recurrent layer on the GPU: a plan plus the caller-owned device tensors.

Plumbing only (allocation with torch, the decode / flush call order of the C ABI);
the arithmetic runs in libsketchssm's kernels.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np
import torch

from ._binding import (Plan, sketchssm_decode, sketchssm_decode_rows, sketchssm_dense_decode, sketchssm_flush,
                       sketchssm_flush_rows, sketchssm_prefill, sketchssm_step)


def _dev(x, device) -> torch.Tensor:
    if isinstance(x, torch.Tensor):
        return x.to(device=device, dtype=torch.float32).contiguous()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


class SketchLayer:
    """State S, sketch Y, key/value buffers and output y of one layer at a fixed batch.

    Protocol (include/sketchssm.h): flush(0) once to form the first sketch, then
    decode(pos) for pos = 0 .. W-1, flush(W), and again from pos = 0.
    """

    def __init__(self, kind: str, *, batch: int, heads: int, qk_heads: int, key_dim: int,
                 value_dim: int, window: int, groups: int, rank_cap: int, rank: Sequence[int],
                 omega, S0=None, device="cuda", stream=None):
        omega_t = _dev(omega, device)
        self.plan = Plan(kind, batch=batch, heads=heads, qk_heads=qk_heads, key_dim=key_dim,
                         value_dim=value_dim, window=window, groups=groups,
                         basis_rows=omega_t.shape[1], rank_cap=rank_cap, rank=rank, stream=stream)
        sh = self.plan.shapes
        z = lambda name: torch.zeros(sh[name], dtype=torch.float32, device=device)
        self.kind = kind
        self.omega = omega_t
        self.S = z("S") if S0 is None else _dev(S0, device)
        self.Y = z("Y")
        self.kbuf, self.vbuf, self.abuf = z("kbuf"), z("vbuf"), z("abuf")
        self.bbuf = None if kind == "mamba2" else z("bbuf")
        self.y = z("y")
        self.window = window

    def flush(self, n: int, stream=None) -> None:
        sketchssm_flush(self.plan, self.S, self.omega, self.kbuf, self.vbuf, self.abuf, self.bbuf, n,
                        self.Y, stream)

    def decode(self, pos: int, q, k, v, a, beta: Optional[torch.Tensor] = None, out=None,
               stream=None) -> torch.Tensor:
        y = self.y if out is None else out
        sketchssm_decode(self.plan, pos, q, k, v, a, beta, self.kbuf, self.vbuf, self.abuf, self.bbuf,
                         self.Y, self.omega, self.S, y, stream)
        return y

    def dense_decode(self, pos: int, q, k, v, a, beta: Optional[torch.Tensor] = None, out=None,
                     stream=None) -> torch.Tensor:
        y = self.y if out is None else out
        sketchssm_dense_decode(self.plan, pos, q, k, v, a, beta, self.kbuf, self.vbuf, self.abuf,
                               self.bbuf, self.S, y, stream)
        return y

    def decode_rows(self, pos: torch.Tensor, q, k, v, a, beta: Optional[torch.Tensor] = None, out=None,
                    stream=None) -> torch.Tensor:
        """Decode with a buffer position per batch row (pos: int32 [B] on the device)."""
        y = self.y if out is None else out
        sketchssm_decode_rows(self.plan, pos, q, k, v, a, beta, self.kbuf, self.vbuf, self.abuf, self.bbuf,
                              self.Y, self.omega, self.S, y, stream)
        return y

    def flush_rows(self, n_tokens: torch.Tensor, stream=None) -> None:
        """Flush each batch row's first n_tokens[b] buffered tokens (int32 [B] on the device)."""
        sketchssm_flush_rows(self.plan, self.S, self.omega, self.kbuf, self.vbuf, self.abuf, self.bbuf,
                             n_tokens, self.Y, stream)

    def standard_step(self, q, k, v, a, beta: Optional[torch.Tensor] = None, out=None,
                      stream=None) -> torch.Tensor:
        """The per-step recurrent decode (no buffer): S updated in place, y = S^T q."""
        y = self.y if out is None else out
        sketchssm_step(self.plan, q, k, v, a, beta, self.S, y, stream)
        return y

    def prefill(self, k, v, a, beta: Optional[torch.Tensor] = None, stream=None) -> None:
        """Prefill handoff: the prompt (token-major k [B][T][Hqk][K], v [B][T][H][V],
        a [B][T][H] or KDA [B][T][H][K], beta [B][T][H]) applied to S, then Y formed
        from the new state; decoding continues at pos = 0."""
        sketchssm_prefill(self.plan, int(k.shape[1]), k, v, a, beta, self.S, self.omega, self.Y, stream)

    def close(self) -> None:
        self.plan.close()
