"""fp64 CPU oracle for Lightning Attention (test infrastructure only).

Only the test suite, the entry module's smoke check and the benchmark's
CPU-baseline leg import this package; the product package never does.
"""
from .oracle import (backward, blocked, build, decode_step, max_threads, quadratic,  # noqa: F401
                     recurrent, segmented)
