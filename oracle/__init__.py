"""fp64 CPU oracle of the SketchSSM decode path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The product path (``rank_state_read_b200``) never imports
it and shares no code with it.

* ``sketch_oracle.c`` : the algorithm in its steps (flush, sketch, replay, read),
  plain fp64 loops, compiled by ``oracle/build.py``; also the standard per-step
  recurrent decode (``standard_step``), the baseline the paper compares against,
  and the prefill handoff (``prefill``: a prompt's tokens applied to the state in
  order, after which ``OracleLayer.prefill`` forms the sketch with the n = 0 flush).
* ``brute``           : the plain definitions on tiny inputs (explicit matrices).

Parity is pinned by the ``-m "not gpu"`` tests in ``tests/test_oracle_pins.py``;
nothing here is "parity unpinned" except the accuracy of a rank-r sketch against the
exact read on real models (that needs a calibrated basis the pages do not publish).
"""
from .core import (OracleLayer, layout, load_library, num_threads, prefill, set_num_threads,  # noqa: F401
                   standard_step, trajectory)
