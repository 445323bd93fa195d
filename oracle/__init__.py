"""fp64 CPU oracle for Lightning Attention (test infrastructure only).

Only the test suite, the entry module's smoke check and the benchmark's
CPU-baseline leg import this package; the product package never does.
"""
from .oracle import (backward, blocked, blocked_decay, build, decode_step, decode_step_decay,  # noqa: F401
                     max_threads, quadratic, quadratic_decay, recurrent, recurrent_decay, segmented,
                     segmented_decay)
