"""Python binding of libcowa.so: argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
turns torch tensors into the C ABI's pointers and strides, allocates the
caller-owned outputs and workspace with torch, and raises on any non-OK
status.  There is no fallback: if libcowa.so is missing or fails to load,
every call raises.

Calls are asynchronous on the stream, as in the C ABI.  A kernel whose bounded wait
runs out records COWA_ERR_TIMEOUT in its workspace's status word instead of hanging;
reading that word needs a stream synchronisation, so no call reads it on its own:
pass `workspace=` and call `workspace_status(workspace)` at a point where a sync is
acceptable (a workspace the binding allocates itself is not checked).

Function names follow the C ABI (include/cowa.h): cowa_fwd, cowa_fwd_chunk,
cowa_fwd_varlen, cowa_bwd, cowa_bwd_varlen, cowa_decode, cowa_decode_compact (with compact_cache /
compact_append), the E4M3-cache decodes (cowa_decode_fp8, cowa_decode_fp8_compact, with
quantize_e4m3, compact_cache_fp8, compact_append_fp8), cowa_decode_noalloc, plus the planner
introspection helpers.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# COWA_DEBUG=1 selects the self-checking build (`python -m structured_sparse_attention_cowa_b200.build
# --debug`); it computes the same bits and reports a failed check as COWA_ERR_CHECK
LIB_PATH = os.path.join(_HERE, "libcowa_debug.so" if os.environ.get("COWA_DEBUG") == "1" else "libcowa.so")

COWA_OK = 0
_STATUS = {0: "COWA_OK", 1: "COWA_ERR_INVALID_ARG", 2: "COWA_ERR_UNSUPPORTED", 3: "COWA_ERR_ALIGNMENT",
           4: "COWA_ERR_WORKSPACE", 5: "COWA_ERR_CUDA", 6: "COWA_ERR_TIMEOUT", 7: "COWA_ERR_CHECK"}

BWD_PREPROCESS, BWD_DKDV, BWD_DQ = 1, 2, 4


class CowaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {_STATUS.get(status, status)} ({msg})")
        self.status = status


class c_pattern(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int32), ("L", ctypes.c_int32), ("T", ctypes.c_int32), ("D", ctypes.c_int32),
                ("kv_head_base", ctypes.c_int32), ("h_kv_global", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float)]


class c_tensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride_b", ctypes.c_int64), ("stride_t", ctypes.c_int64),
                ("stride_h", ctypes.c_int64)]


@dataclasses.dataclass(frozen=True)
class Pattern:
    """CoWA window parameters (see include/cowa.h, cowa_pattern)."""

    S: int
    L: int
    T: int
    D: int
    kv_head_base: int = 0
    h_kv_global: int = 0
    softmax_scale: float = 0.0

    def c(self) -> c_pattern:
        return c_pattern(self.S, self.L, self.T, self.D, self.kv_head_base, self.h_kv_global, self.softmax_scale)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libcowa.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{os.path.basename(LIB_PATH)} not found at {LIB_PATH}; build it with "
                           "`python -m structured_sparse_attention_cowa_b200.build`"
                           + (" --debug" if LIB_PATH.endswith("_debug.so") else ""))
    L = ctypes.CDLL(LIB_PATH)
    P, T, vp, i, sz = ctypes.POINTER(c_pattern), c_tensor, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.cowa_fwd_workspace_size.argtypes = [P, i, i, i, i, i]
    L.cowa_fwd_workspace_size.restype = sz
    L.cowa_fwd.argtypes = [P, i, i, i, i, i, T, T, T, T, vp, vp, sz, vp]
    L.cowa_fwd.restype = i
    L.cowa_fwd_chunk.argtypes = [P, i, i, i, i, i, i, i, T, T, T, T, vp, vp, sz, vp]
    L.cowa_fwd_chunk.restype = i
    L.cowa_fwd_varlen_workspace_size.argtypes = [P, i, i, i, i, i]
    L.cowa_fwd_varlen_workspace_size.restype = sz
    L.cowa_fwd_varlen.argtypes = [P, i, i, i, i, i, vp, T, T, T, T, vp, vp, sz, vp]
    L.cowa_fwd_varlen.restype = i
    L.cowa_bwd_workspace_size.argtypes = [P, i, i, i, i, i]
    L.cowa_bwd_workspace_size.restype = sz
    L.cowa_bwd.argtypes = [P, i, i, i, i, i, T, T, T, T, vp, T, T, T, T, vp, sz, vp]
    L.cowa_bwd.restype = i
    L.cowa_bwd_stages.argtypes = [P, i, i, i, i, i, T, T, T, T, vp, T, T, T, T, i, vp, sz, vp]
    L.cowa_bwd_stages.restype = i
    L.cowa_bwd_varlen_workspace_size.argtypes = [P, i, i, i, i, i]
    L.cowa_bwd_varlen_workspace_size.restype = sz
    L.cowa_bwd_varlen.argtypes = [P, i, i, i, i, i, vp, T, T, T, T, vp, T, T, T, T, vp, sz, vp]
    L.cowa_bwd_varlen.restype = i
    L.cowa_decode_workspace_size.argtypes = [P, i, i, i, i, i]
    L.cowa_decode_workspace_size.restype = sz
    L.cowa_decode.argtypes = [P, i, i, i, i, i, vp, T, T, vp, vp, vp, vp, sz, vp]
    L.cowa_decode.restype = i
    L.cowa_decode_noalloc.argtypes = [P, i, i, i, i, i, vp, T, T, vp, vp, vp, vp]
    L.cowa_decode_noalloc.restype = i
    L.cowa_decode_noalloc_status.argtypes = [vp]
    L.cowa_decode_noalloc_status.restype = i
    L.cowa_compact_rows.argtypes = [P, i]
    L.cowa_compact_rows.restype = i
    L.cowa_compact_build.argtypes = [P, i, i, i, i, T, T, vp, vp, vp]
    L.cowa_compact_build.restype = i
    L.cowa_compact_append.argtypes = [P, i, i, i, vp, vp, vp, vp, vp, vp]
    L.cowa_compact_append.restype = i
    L.cowa_decode_compact_workspace_size.argtypes = [P, i, i, i, i]
    L.cowa_decode_compact_workspace_size.restype = sz
    L.cowa_decode_compact.argtypes = [P, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.cowa_decode_compact.restype = i
    f = ctypes.c_float
    L.cowa_decode_fp8_workspace_size.argtypes = [P, i, i, i, i, i]
    L.cowa_decode_fp8_workspace_size.restype = sz
    L.cowa_decode_fp8.argtypes = [P, i, i, i, i, i, vp, T, T, f, f, vp, vp, vp, vp, sz, vp]
    L.cowa_decode_fp8.restype = i
    L.cowa_quantize_e4m3.argtypes = [vp, vp, ctypes.c_int64, f, vp]
    L.cowa_quantize_e4m3.restype = i
    L.cowa_compact_build_fp8.argtypes = [P, i, i, i, i, T, T, vp, vp, vp]
    L.cowa_compact_build_fp8.restype = i
    L.cowa_compact_append_fp8.argtypes = [P, i, i, i, vp, vp, vp, vp, vp, vp]
    L.cowa_compact_append_fp8.restype = i
    L.cowa_decode_fp8_compact_workspace_size.argtypes = [P, i, i, i, i]
    L.cowa_decode_fp8_compact_workspace_size.restype = sz
    L.cowa_decode_fp8_compact.argtypes = [P, i, i, i, i, vp, vp, vp, f, f, vp, vp, vp, vp, sz, vp]
    L.cowa_decode_fp8_compact.restype = i
    L.cowa_workspace_status.argtypes = [vp, vp]
    L.cowa_workspace_status.restype = i
    L.cowa_status_string.argtypes = [i]
    L.cowa_status_string.restype = ctypes.c_char_p
    L.cowa_visible_counts.argtypes = [P, i, i, vp]
    L.cowa_visible_counts.restype = i
    L.cowa_plan_debug.argtypes = [P, i, i, i, i, i, vp, sz, ctypes.POINTER(sz), vp]
    L.cowa_plan_debug.restype = i
    L.cowa_debug_wait_timeout.argtypes = [vp, sz, ctypes.c_int64, vp]
    L.cowa_debug_wait_timeout.restype = i
    L.cowa_version.argtypes = []
    L.cowa_version.restype = i
    _lib = L
    return L


def _check(fn: str, status: int):
    if status != COWA_OK:
        raise CowaError(fn, status, lib().cowa_status_string(status).decode())


def _t4(x) -> c_tensor:
    """[B, N, H, d] tensor (d contiguous) -> cowa_tensor."""
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("expected a [B, N, H, d] tensor with the last dim contiguous")
    return c_tensor(x.data_ptr(), x.stride(0), x.stride(1), x.stride(2))


def _stream(stream):
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _workspace(nbytes: int, device):
    import torch

    return torch.zeros(max(256, nbytes), dtype=torch.uint8, device=device)


def _bf16_cuda(name, x):
    import torch

    if not (x.is_cuda and x.dtype == torch.bfloat16):
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")


def cowa_fwd(q, k, v, pattern: Pattern, out=None, lse=None, workspace=None, stream=None):
    """o [B,N,H_q,d] bf16 and lse [B,H_q,N] fp32 of CoWA attention over q, k, v."""
    import torch

    for n_, x_ in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n_, x_)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    pat = pattern.c()
    L = lib()
    ws_bytes = L.cowa_fwd_workspace_size(ctypes.byref(pat), B, N, Hq, Hkv, d)
    if workspace is None:
        workspace = _workspace(ws_bytes, q.device)
    _check("cowa_fwd", L.cowa_fwd(ctypes.byref(pat), B, N, Hq, Hkv, d, _t4(q), _t4(k), _t4(v), _t4(out),
                                  lse.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out, lse


def cowa_fwd_chunk(q, k, v, pattern: Pattern, q_offset: int, n_k=None, kv_layout: str = "bthd", out=None,
                   lse=None, workspace=None, stream=None):
    """Chunked prefill: o [B,N_q,H_q,d] bf16 and lse [B,H_q,N_q] fp32 for the query rows at
    positions q_offset .. q_offset+N_q-1 against the keys 0 .. n_k-1 of k, v.  k, v are
    [B, N_k, H_kv, d] (kv_layout "bthd") or a cache [B, H_kv, T_cap, d] ("bhtd"); n_k defaults
    to their full length and must cover q_offset + N_q."""
    import torch

    for n_, x_ in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n_, x_)
    B, Nq, Hq, d = q.shape
    if kv_layout == "bthd":
        kt, vt = k, v
    elif kv_layout == "bhtd":
        kt, vt = k.transpose(1, 2), v.transpose(1, 2)  # strided views [B, T, H, d]
    else:
        raise ValueError("kv_layout is 'bthd' or 'bhtd'")
    Hkv = kt.shape[2]
    if n_k is None:
        n_k = kt.shape[1]
    if not 0 < n_k <= kt.shape[1]:
        raise ValueError("n_k out of range")
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    pat = pattern.c()
    L = lib()
    ws_bytes = L.cowa_fwd_workspace_size(ctypes.byref(pat), B, Nq, Hq, Hkv, d)
    if workspace is None:
        workspace = _workspace(ws_bytes, q.device)
    _check("cowa_fwd_chunk", L.cowa_fwd_chunk(ctypes.byref(pat), B, Nq, int(n_k), int(q_offset), Hq, Hkv, d, _t4(q),
                                              _t4(kt), _t4(vt), _t4(out), lse.data_ptr(), workspace.data_ptr(),
                                              workspace.numel(), _stream(stream)))
    return out, lse


def cowa_fwd_varlen(q, k, v, cu_seqlens, pattern: Pattern, out=None, lse=None, workspace=None, stream=None):
    """Packed variable-length batch: q [total, H_q, d], k, v [total, H_kv, d], cu_seqlens CUDA int32
    [n_seq + 1]; returns o [total, H_q, d] bf16 and lse [H_q, total] fp32, each sequence attending
    over its own rows at positions 0.. ."""
    import torch

    for n_, x_ in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n_, x_)
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D CUDA int32 tensor")
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    n_seq = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if lse is None:
        lse = torch.empty((Hq, total), dtype=torch.float32, device=q.device)
    pat = pattern.c()
    L = lib()
    ws_bytes = L.cowa_fwd_varlen_workspace_size(ctypes.byref(pat), n_seq, total, Hq, Hkv, d)
    if workspace is None:
        workspace = _workspace(ws_bytes, q.device)
    t4 = lambda x: _t4(x.unsqueeze(0))
    _check("cowa_fwd_varlen", L.cowa_fwd_varlen(ctypes.byref(pat), n_seq, total, Hq, Hkv, d, cu_seqlens.data_ptr(),
                                                t4(q), t4(k), t4(v), t4(out), lse.data_ptr(), workspace.data_ptr(),
                                                workspace.numel(), _stream(stream)))
    return out, lse


def cowa_bwd(q, k, v, o, lse, do, pattern: Pattern, dq=None, dk=None, dv=None, workspace=None, stream=None,
             stages: int = 7):
    """(dq, dk, dv) bf16: gradients of sum(do * o) for the forward with the same inputs.
    `stages` selects BWD_PREPROCESS | BWD_DKDV | BWD_DQ (all by default)."""
    import torch

    for n_, x_ in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _bf16_cuda(n_, x_)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    pat = pattern.c()
    L = lib()
    ws_bytes = L.cowa_bwd_workspace_size(ctypes.byref(pat), B, N, Hq, Hkv, d)
    if workspace is None:
        workspace = _workspace(ws_bytes, q.device)
    if stages == 7:
        _check("cowa_bwd", L.cowa_bwd(ctypes.byref(pat), B, N, Hq, Hkv, d, _t4(q), _t4(k), _t4(v), _t4(o),
                                      lse.data_ptr(), _t4(do), _t4(dq), _t4(dk), _t4(dv),
                                      workspace.data_ptr(), workspace.numel(), _stream(stream)))
    else:
        _check("cowa_bwd_stages", L.cowa_bwd_stages(ctypes.byref(pat), B, N, Hq, Hkv, d, _t4(q), _t4(k), _t4(v),
                                                    _t4(o), lse.data_ptr(), _t4(do), _t4(dq), _t4(dk), _t4(dv),
                                                    stages, workspace.data_ptr(), workspace.numel(),
                                                    _stream(stream)))
    return dq, dk, dv


def cowa_bwd_varlen(q, k, v, o, lse, do, cu_seqlens, pattern: Pattern, dq=None, dk=None, dv=None, workspace=None,
                    stream=None):
    """Gradients of cowa_fwd_varlen: q, o, do [total, H_q, d], k, v [total, H_kv, d], lse [H_q, total],
    cu_seqlens a CUDA int32 tensor of n_seq + 1 offsets (as for cowa_fwd_varlen); returns dq, dk, dv.
    One launch per backward kernel over all sequences (see cowa_bwd_varlen in cowa.h)."""
    import torch

    for n_, x_ in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _bf16_cuda(n_, x_)
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D CUDA int32 tensor")
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    n_seq = cu_seqlens.numel() - 1
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    pat = pattern.c()
    L = lib()
    ws_bytes = L.cowa_bwd_varlen_workspace_size(ctypes.byref(pat), n_seq, total, Hq, Hkv, d)
    if workspace is None:
        workspace = _workspace(ws_bytes, q.device)
    t4 = lambda x: _t4(x.unsqueeze(0))
    _check("cowa_bwd_varlen", L.cowa_bwd_varlen(ctypes.byref(pat), n_seq, total, Hq, Hkv, d, cu_seqlens.data_ptr(),
                                                t4(q), t4(k), t4(v), t4(o), lse.data_ptr(), t4(do), t4(dq), t4(dk),
                                                t4(dv), workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return dq, dk, dv


def _cache_tensor(x, layout: str) -> c_tensor:
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("cache must be 4-D with the head dim contiguous")
    if layout == "bhtd":   # [B, H_kv, T_cap, d]
        return c_tensor(x.data_ptr(), x.stride(0), x.stride(2), x.stride(1))
    if layout == "bthd":   # [B, T_cap, H_kv, d]
        return c_tensor(x.data_ptr(), x.stride(0), x.stride(1), x.stride(2))
    raise ValueError("layout must be 'bhtd' or 'bthd'")


def cowa_decode(q_t, k_cache, v_cache, pos, pattern: Pattern, layout: str = "bhtd", out=None, lse=None,
                workspace=None, stream=None, want_lse: bool = True):
    """o [B,H_q,d] bf16 (and lse [B,H_q] fp32) for one new token per sequence at pos[b]."""
    import torch

    for n_, x_ in (("q_t", q_t), ("k_cache", k_cache), ("v_cache", v_cache)):
        _bf16_cuda(n_, x_)
    B, Hq, d = q_t.shape
    if layout == "bhtd":
        Hkv, T_cap = k_cache.shape[1], k_cache.shape[2]
    else:
        T_cap, Hkv = k_cache.shape[1], k_cache.shape[2]
    if not q_t.is_contiguous():
        raise ValueError("q_t must be contiguous [B, H_q, d]")
    if pos.dtype != torch.int32 or not pos.is_cuda:
        raise TypeError("pos must be a CUDA int32 tensor [B]")
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q_t.device) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q_t.device)
    pat = pattern.c()
    L = lib()
    ws_bytes = L.cowa_decode_workspace_size(ctypes.byref(pat), B, Hq, Hkv, d, T_cap)
    if workspace is None:
        workspace = _workspace(ws_bytes, q_t.device)
    _check("cowa_decode", L.cowa_decode(ctypes.byref(pat), B, Hq, Hkv, d, T_cap, q_t.data_ptr(),
                                        _cache_tensor(k_cache, layout), _cache_tensor(v_cache, layout),
                                        pos.data_ptr(), out.data_ptr(), lse.data_ptr() if lse is not None else None,
                                        workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out, lse


def compact_rows(pattern: Pattern, h_kv: int) -> int:
    """Rows per (b, KV head) of the compacted decode cache."""
    n = lib().cowa_compact_rows(ctypes.byref(pattern.c()), h_kv)
    if n <= 0:
        raise CowaError("invalid pattern for the compacted cache")
    return n


def compact_cache(k, v, pattern: Pattern, out=None, stream=None):
    """Compacted caches (k_c, v_c), [B, H_kv, rows, d] bf16, built from k, v [B, N, H_kv, d] of
    positions 0..N-1."""
    import torch

    for n_, x_ in (("k", k), ("v", v)):
        _bf16_cuda(n_, x_)
    B, N, Hkv, d = k.shape
    rows = compact_rows(pattern, Hkv)
    if out is None:
        out = (torch.zeros((B, Hkv, rows, d), dtype=torch.bfloat16, device=k.device),
               torch.zeros((B, Hkv, rows, d), dtype=torch.bfloat16, device=k.device))
    kc, vc = out
    _check("cowa_compact_build", lib().cowa_compact_build(ctypes.byref(pattern.c()), B, N, Hkv, d, _t4(k), _t4(v),
                                                          kc.data_ptr(), vc.data_ptr(), _stream(stream)))
    return kc, vc


def compact_append(kc, vc, k_new, v_new, pos, pattern: Pattern, stream=None):
    """Appends the token at pos[b] (k_new, v_new [B, H_kv, d]) to the compacted caches in place."""
    import torch

    B, Hkv, _, d = kc.shape
    if pos.dtype != torch.int32 or not pos.is_cuda:
        raise ValueError("pos must be a CUDA int32 tensor")
    k_new, v_new = k_new.contiguous(), v_new.contiguous()
    _check("cowa_compact_append", lib().cowa_compact_append(ctypes.byref(pattern.c()), B, Hkv, d, k_new.data_ptr(),
                                                            v_new.data_ptr(), pos.data_ptr(), kc.data_ptr(),
                                                            vc.data_ptr(), _stream(stream)))


def cowa_decode_compact(q_t, kc, vc, pos, pattern: Pattern, out=None, lse=None, workspace=None, stream=None):
    """cowa_decode over the compacted caches kc, vc [B, H_kv, rows, d]."""
    import torch

    for n_, x_ in (("q_t", q_t), ("k_compact", kc), ("v_compact", vc)):
        _bf16_cuda(n_, x_)
    if not (q_t.is_contiguous() and kc.is_contiguous() and vc.is_contiguous()):
        raise ValueError("q_t and the compacted caches must be contiguous")
    if pos.dtype != torch.int32 or not pos.is_cuda:
        raise ValueError("pos must be a CUDA int32 tensor")
    B, Hq, d = q_t.shape
    Hkv = kc.shape[1]
    if kc.shape[2] != compact_rows(pattern, Hkv):
        raise ValueError("compacted cache has the wrong number of rows for this pattern")
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q_t.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q_t.device)
    pat = pattern.c()
    L = lib()
    ws_bytes = L.cowa_decode_compact_workspace_size(ctypes.byref(pat), B, Hq, Hkv, d)
    if workspace is None:
        workspace = _workspace(ws_bytes, q_t.device)
    _check("cowa_decode_compact", L.cowa_decode_compact(ctypes.byref(pat), B, Hq, Hkv, d, q_t.data_ptr(), kc.data_ptr(),
                                                        vc.data_ptr(), pos.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                                        workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out, lse


def cowa_decode_noalloc(q_t, k_cache, v_cache, pos, pattern: Pattern, out, lse=None, layout: str = "bhtd",
                        stream=None):
    """cowa_decode without a workspace: the library's static per-device scratch holds the split
    partials (see include/cowa.h).  `out` [B,H_q,d] bf16 (and `lse` [B,H_q] fp32, optional) are
    the caller's; nothing is allocated by this call."""
    for n_, x_ in (("q_t", q_t), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out)):
        _bf16_cuda(n_, x_)
    B, Hq, d = q_t.shape
    if layout == "bhtd":
        Hkv, T_cap = k_cache.shape[1], k_cache.shape[2]
    else:
        T_cap, Hkv = k_cache.shape[1], k_cache.shape[2]
    pat = pattern.c()
    _check("cowa_decode_noalloc", lib().cowa_decode_noalloc(
        ctypes.byref(pat), B, Hq, Hkv, d, T_cap, q_t.data_ptr(), _cache_tensor(k_cache, layout),
        _cache_tensor(v_cache, layout), pos.data_ptr(), out.data_ptr(),
        lse.data_ptr() if lse is not None else None, _stream(stream)))
    return out, lse


# ---------------------------------------------------------------------------- E4M3 cache
def _u8_cuda(name, x):
    import torch

    if not (x.is_cuda and x.dtype == torch.uint8):
        raise TypeError(f"{name} must be a CUDA uint8 tensor of E4M3 codes")


def quantize_e4m3(x, scale: float, out=None, stream=None):
    """E4M3 codes (uint8, same shape) of the bf16 tensor x divided by scale: a float32 multiply by
    the float32 reciprocal of scale, round to nearest even, saturating at +-448."""
    import torch

    _bf16_cuda("x", x)
    if not x.is_contiguous() or x.numel() % 8 != 0:
        raise ValueError("x must be contiguous with a multiple of 8 elements")
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device) if out is None else out
    _check("cowa_quantize_e4m3", lib().cowa_quantize_e4m3(x.data_ptr(), out.data_ptr(), x.numel(), float(scale),
                                                          _stream(stream)))
    return out


def cowa_decode_fp8(q_t, k_codes, v_codes, pos, pattern: Pattern, k_scale: float, v_scale: float,
                    layout: str = "bhtd", out=None, lse=None, workspace=None, stream=None):
    """cowa_decode over an E4M3 cache: keys k_scale * e4m3(k_codes), values v_scale * e4m3(v_codes);
    codes uint8 [B, H_kv, T_cap, 128] ("bhtd") or [B, T_cap, H_kv, 128] ("bthd")."""
    import torch

    _bf16_cuda("q_t", q_t)
    _u8_cuda("k_codes", k_codes)
    _u8_cuda("v_codes", v_codes)
    if not q_t.is_contiguous():
        raise ValueError("q_t must be contiguous [B, H_q, d]")
    if pos.dtype != torch.int32 or not pos.is_cuda:
        raise TypeError("pos must be a CUDA int32 tensor [B]")
    B, Hq, d = q_t.shape
    Hkv, T_cap = (k_codes.shape[1], k_codes.shape[2]) if layout == "bhtd" else (k_codes.shape[2], k_codes.shape[1])
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q_t.device) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q_t.device) if lse is None else lse
    pat = pattern.c()
    L = lib()
    if workspace is None:
        workspace = _workspace(L.cowa_decode_fp8_workspace_size(ctypes.byref(pat), B, Hq, Hkv, d, T_cap), q_t.device)
    _check("cowa_decode_fp8", L.cowa_decode_fp8(ctypes.byref(pat), B, Hq, Hkv, d, T_cap, q_t.data_ptr(),
                                                _cache_tensor(k_codes, layout), _cache_tensor(v_codes, layout),
                                                float(k_scale), float(v_scale), pos.data_ptr(), out.data_ptr(),
                                                lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                                _stream(stream)))
    return out, lse


def compact_cache_fp8(k_codes, v_codes, pattern: Pattern, out=None, stream=None):
    """Compacted E4M3 caches [B, H_kv, rows, 128] (uint8) built from codes [B, N, H_kv, 128]."""
    import torch

    _u8_cuda("k_codes", k_codes)
    _u8_cuda("v_codes", v_codes)
    B, N, Hkv, d = k_codes.shape
    rows = compact_rows(pattern, Hkv)
    if out is None:
        out = (torch.zeros((B, Hkv, rows, d), dtype=torch.uint8, device=k_codes.device),
               torch.zeros((B, Hkv, rows, d), dtype=torch.uint8, device=k_codes.device))
    kc, vc = out
    _check("cowa_compact_build_fp8", lib().cowa_compact_build_fp8(ctypes.byref(pattern.c()), B, N, Hkv, d,
                                                                  _t4(k_codes), _t4(v_codes), kc.data_ptr(),
                                                                  vc.data_ptr(), _stream(stream)))
    return kc, vc


def compact_append_fp8(kc, vc, k_new, v_new, pos, pattern: Pattern, stream=None):
    """Appends one token's codes (k_new, v_new uint8 [B, H_kv, 128]) at pos[b] to compacted E4M3 caches."""
    import torch

    _u8_cuda("k_new", k_new)
    _u8_cuda("v_new", v_new)
    if pos.dtype != torch.int32 or not pos.is_cuda:
        raise ValueError("pos must be a CUDA int32 tensor")
    B, Hkv, _, d = kc.shape
    k_new, v_new = k_new.contiguous(), v_new.contiguous()
    _check("cowa_compact_append_fp8", lib().cowa_compact_append_fp8(ctypes.byref(pattern.c()), B, Hkv, d,
                                                                    k_new.data_ptr(), v_new.data_ptr(), pos.data_ptr(),
                                                                    kc.data_ptr(), vc.data_ptr(), _stream(stream)))


def cowa_decode_fp8_compact(q_t, kc, vc, pos, pattern: Pattern, k_scale: float, v_scale: float, out=None,
                            lse=None, workspace=None, stream=None):
    """cowa_decode_fp8 over compacted E4M3 caches kc, vc [B, H_kv, rows, 128] (uint8)."""
    import torch

    _bf16_cuda("q_t", q_t)
    _u8_cuda("k_compact", kc)
    _u8_cuda("v_compact", vc)
    if not (q_t.is_contiguous() and kc.is_contiguous() and vc.is_contiguous()):
        raise ValueError("q_t and the compacted caches must be contiguous")
    if pos.dtype != torch.int32 or not pos.is_cuda:
        raise ValueError("pos must be a CUDA int32 tensor")
    B, Hq, d = q_t.shape
    Hkv = kc.shape[1]
    if kc.shape[2] != compact_rows(pattern, Hkv):
        raise ValueError("compacted cache has the wrong number of rows for this pattern")
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q_t.device) if out is None else out
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q_t.device) if lse is None else lse
    pat = pattern.c()
    L = lib()
    if workspace is None:
        workspace = _workspace(L.cowa_decode_fp8_compact_workspace_size(ctypes.byref(pat), B, Hq, Hkv, d), q_t.device)
    _check("cowa_decode_fp8_compact", L.cowa_decode_fp8_compact(ctypes.byref(pat), B, Hq, Hkv, d, q_t.data_ptr(),
                                                                kc.data_ptr(), vc.data_ptr(), float(k_scale),
                                                                float(v_scale), pos.data_ptr(), out.data_ptr(),
                                                                lse.data_ptr(), workspace.data_ptr(),
                                                                workspace.numel(), _stream(stream)))
    return out, lse


def decode_noalloc_status(stream=None) -> int:
    """Synchronize the stream, read (and clear) the status word of cowa_decode_noalloc's scratch
    on the current device; returns the cowa_status code."""
    return lib().cowa_decode_noalloc_status(_stream(stream))


def workspace_status(workspace, stream=None) -> int:
    """Read (and clear) the device status word of a workspace; returns the cowa_status code."""
    return lib().cowa_workspace_status(ctypes.c_void_p(workspace.data_ptr()), _stream(stream))


# ---------------------------------------------------------------------------- introspection
def visible_counts(pattern: Pattern, h_kv: int, N: int) -> np.ndarray:
    out = np.zeros((h_kv, N), dtype=np.int64)
    pat = pattern.c()
    _check("cowa_visible_counts", lib().cowa_visible_counts(ctypes.byref(pat), h_kv, N,
                                                            out.ctypes.data_as(ctypes.c_void_p)))
    return out


def plan_debug(pattern: Pattern, h_kv: int, N: int, BM: int, BN: int, which: int, dev_scratch=None) -> np.ndarray:
    """Tile-plan records, int32 [n, 4]; which = 0 fwd (host), 1 bwd (host), 2 fwd (device kernel)."""
    pat = pattern.c()
    L = lib()
    n = ctypes.c_size_t(0)
    cap = 1024
    while True:
        out = np.zeros((cap, 4), dtype=np.int32)
        scratch = None
        if which == 2:
            import torch

            scratch = torch.zeros(256 + cap * 16, dtype=torch.uint8, device="cuda") if dev_scratch is None else dev_scratch
        st = L.cowa_plan_debug(ctypes.byref(pat), h_kv, N, BM, BN, which, out.ctypes.data_as(ctypes.c_void_p), cap,
                               ctypes.byref(n), ctypes.c_void_p(scratch.data_ptr()) if scratch is not None else None)
        if st == 4 and n.value > cap:
            cap = int(n.value)
            continue
        _check("cowa_plan_debug", st)
        return out[: n.value].copy()
