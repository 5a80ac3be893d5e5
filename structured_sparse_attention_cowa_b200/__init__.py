"""CoWindow Attention (CoWA) for NVIDIA B200 (sm_100a).

The compute lives in libcowa.so (hand-written CUDA: TMA + tcgen05 forward and
backward kernels, a split-KV decode kernel); `cowa` is its ctypes binding.
"""

from .cowa import (CowaError, Pattern, compact_append, compact_cache, compact_rows, cowa_bwd,  # noqa: F401
                   cowa_bwd_varlen,
                   cowa_decode, cowa_decode_compact, cowa_fwd, cowa_fwd_chunk, cowa_fwd_varlen, lib, plan_debug, visible_counts,
                   workspace_status)

__all__ = ["Pattern", "CowaError", "cowa_fwd", "cowa_fwd_chunk", "cowa_fwd_varlen", "cowa_bwd", "cowa_bwd_varlen", "cowa_decode", "cowa_decode_compact",
           "compact_rows", "compact_cache", "compact_append", "lib", "plan_debug", "visible_counts",
           "workspace_status"]
