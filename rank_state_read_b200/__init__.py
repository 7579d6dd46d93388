"""SketchSSM decode path on B200 (sm_100a): write the full state, read a compact sketch.

The work runs in libsketchssm.so (hand-written CUDA kernels behind the C ABI of
include/sketchssm.h); this package is its thin Python binding.  Importing it does
not touch the GPU; the first call loads the library and fails loudly if it has not
been built (``python -m rank_state_read_b200.build``).
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
