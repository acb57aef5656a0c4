"""fp64 CPU oracle of the PACE decode path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  It shares no code with the CUDA
library and imports nothing from it.
"""
from .pace_oracle import *  # noqa: F401,F403
from .pace_oracle import (QMAX, FLAG_NONFINITE, FLAG_SCALE_OVERFLOW, PoolState,  # noqa: F401
                          quantize, dequantize, pack_codes, unpack_codes, gdn_step,
                          gdn_step_delta, sequential, chunk_form, commit, pace_run,
                          per_token_rounding, commit_ratios, period_reference,
                          relative_error)
