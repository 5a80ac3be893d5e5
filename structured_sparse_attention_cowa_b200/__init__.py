"""CoWindow Attention (CoWA) for NVIDIA B200 (sm_100a).

The compute lives in libcowa.so (hand-written CUDA: TMA + tcgen05 forward and
backward kernels, a split-KV decode kernel); `cowa` is its ctypes binding.
"""

from .cowa import (CowaError, Pattern, cowa_bwd, cowa_decode, cowa_fwd, cowa_fwd_chunk, lib,  # noqa: F401
                   plan_debug, visible_counts, workspace_status)

__all__ = ["Pattern", "CowaError", "cowa_fwd", "cowa_fwd_chunk", "cowa_bwd", "cowa_decode", "lib", "plan_debug",
           "visible_counts", "workspace_status"]
