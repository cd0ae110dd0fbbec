"""CPU oracle for the DSA forward path (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path never does.
"""
from .oracle import (  # noqa: F401
    F32, BF16, E4M3, build, lib_path, num_threads,
    e4m3_decode, e4m3_encode, bf16_decode,
    fold, scores, topk, topk_dyn, attention, forward_rows,
)
