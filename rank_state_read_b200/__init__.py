"""SketchSSM decode path on B200 (sm_100a): write the full state, read a compact sketch.

The work runs in libsketchssm.so (hand-written CUDA kernels behind the C ABI of
include/sketchssm.h); this package is its thin Python binding.  Importing it does
not touch the GPU; the first call loads the library and fails loudly if it has not
been built (``python -m rank_state_read_b200.build``).

One layer at batch B (tensors fp32 on the GPU; layouts in include/sketchssm.h)::

    import rank_state_read_b200 as rs
    layer = rs.SketchLayer("mamba2", batch=B, heads=128, qk_heads=8, key_dim=128,
                           value_dim=80, window=16, groups=8, rank_cap=49,
                           rank=ranks, omega=omega, S0=S0)
    layer.prefill(k_p, v_p, a_p)         # a prompt, then its sketch (or layer.flush(0))
    for t in range(steps):
        y = layer.decode(t % 16, q, k, v, a)   # never reads S for sketch heads
        if t % 16 == 15:
            layer.flush(16)              # the buffered tokens reach S; Y is re-formed
"""
from ._binding import (  # noqa: F401
    DENSE,
    EXPORTS,
    KINDS,
    LIB_PATH,
    Desc,
    Plan,
    SketchSSMError,
    load,
    sketchssm_decode,
    sketchssm_decode_rows,
    sketchssm_decode_static_scratch,
    sketchssm_dense_decode,
    sketchssm_flush,
    sketchssm_flush_rows,
    sketchssm_plan_create,
    sketchssm_plan_destroy,
    sketchssm_prefill,
    sketchssm_step,
)
from .layer import SketchLayer  # noqa: F401
