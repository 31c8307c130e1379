"""B200-native gated delta-rule linear attention (DeltaNet, Gated DeltaNet,
KDA, Gated DeltaNet-2, KLA): chunked forward, recurrent decode, and the
chunked backward of the scalar-decay variants.

The compute lives in libgdr.so (hand-written CUDA for sm_100a, C ABI in
include/gdr.h); this package is its thin Python binding.  Importing the
package does not load the library; the first call does, and raises if the
library is missing.
"""
from .ops import (VARIANTS, backward, decode_step, device_status, forward, forward_kernel_name,  # noqa: F401
                  forward_launches, forward_plan)
from ._lib import GdrError  # noqa: F401

__all__ = ["forward", "backward", "decode_step", "device_status", "forward_launches", "forward_kernel_name", "forward_plan",
           "VARIANTS", "GdrError"]
