"""MPQ row-batched post-training-quantisation solver for B200 (sm_100a).

The solver itself is libmpq.so (CUDA kernels behind a C ABI declared in
include/mpq.h); this package only binds it.  Importing the package loads the
library and raises ImportError if it has not been built.
"""
from ._lib import (Gram, MPQError, Plan, idx_to_numpy, kernel_launch_count, lib,  # noqa: F401
                   profile_start, profile_stop, rht)

__all__ = ["Plan", "Gram", "rht", "MPQError", "idx_to_numpy", "kernel_launch_count", "lib",
           "profile_start", "profile_stop"]
