// cowa_api.cu -- the extern "C" boundary of libcowa.so (declared in include/cowa.h).
//
// Validates every argument before any launch, builds the TMA tensor maps, carves the
// caller's workspace and launches the kernels on the caller's stream.  No device memory
// is allocated here and no exception crosses the boundary.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <vector>

#include "cowa_internal.h"

namespace cowa {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // resolved once through the runtime; thread-safe static initialisation
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride_ok(int64_t s) { return s > 0 && ((s * 2) % 16) == 0; }

cowa_status check_pattern(const cowa_pattern* pat, int Hkv, Pat* out) {
  if (!pat) return COWA_ERR_INVALID_ARG;
  const int H = pat->h_kv_global > 0 ? pat->h_kv_global : Hkv;
  if (pat->S < 0 || pat->T < pat->S || pat->L < 1 || pat->D < 1) return COWA_ERR_INVALID_ARG;
  if (H < 1 || H % pat->D != 0) return COWA_ERR_INVALID_ARG;
  if (pat->kv_head_base < 0 || pat->kv_head_base > H - Hkv) return COWA_ERR_INVALID_ARG;  // no overflow
  out->S = pat->S; out->L = pat->L; out->T = pat->T; out->D = pat->D;
  out->G0 = pat->kv_head_base; out->H = H;
  return COWA_OK;
}

float scale_of(const cowa_pattern* pat, int d) {
  return pat->softmax_scale > 0.f ? pat->softmax_scale : 1.0f / sqrtf((float)d);
}

cowa_status check_heads(int B, int N, int Hq, int Hkv, int d) {
  if (B < 1 || N < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return COWA_ERR_INVALID_ARG;
  if (Hq / Hkv > 8) return COWA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return COWA_ERR_UNSUPPORTED;
  return COWA_OK;
}

cowa_status check_tensor(const cowa_tensor& t) {
  if (!t.ptr) return COWA_ERR_INVALID_ARG;
  if (!aligned16(t.ptr) || !stride_ok(t.stride_t) || !stride_ok(t.stride_h) || !stride_ok(t.stride_b))
    return COWA_ERR_ALIGNMENT;
  return COWA_OK;
}

cowa_status check_ws(void* ws, size_t have, size_t need) {
  if (have < need || !ws) return COWA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return COWA_ERR_WORKSPACE;
  return COWA_OK;
}

#define COWA_TRY(x)                         \
  do {                                      \
    cowa_status _s = (x);                   \
    if (_s != COWA_OK) return _s;           \
  } while (0)

}  // namespace

bool make_tmap_bf16(CUtensorMap* map, const void* base, int d, int n_t, int n_h, int n_b, int64_t stride_t,
                    int64_t stride_h, int64_t stride_b, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)n_t, (cuuint64_t)n_h, (cuuint64_t)n_b};
  cuuint64_t strides[3] = {(cuuint64_t)stride_t * 2, (cuuint64_t)stride_h * 2, (cuuint64_t)stride_b * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_u8(CUtensorMap* map, const void* base, int d, int n_t, int n_h, int n_b, int64_t stride_t,
                  int64_t stride_h, int64_t stride_b, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)n_t, (cuuint64_t)n_h, (cuuint64_t)n_b};
  cuuint64_t strides[3] = {(cuuint64_t)stride_t, (cuuint64_t)stride_h, (cuuint64_t)stride_b};
  cuuint32_t box[4] = {128, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {
// a tensor of one-byte elements: pointer and byte strides multiples of 16
cowa_status check_tensor8(const cowa_tensor& t) {
  if (!t.ptr) return COWA_ERR_INVALID_ARG;
  auto ok = [](int64_t v) { return v > 0 && v % 16 == 0; };
  if (!aligned16(t.ptr) || !ok(t.stride_t) || !ok(t.stride_h) || !ok(t.stride_b)) return COWA_ERR_ALIGNMENT;
  return COWA_OK;
}
}  // namespace

}  // namespace cowa

using namespace cowa;

extern "C" {

int cowa_version(void) { return 1; }

cowa_status cowa_debug_wait_timeout(void* ws, size_t ws_bytes, int64_t limit_ns, void* stream) {
  COWA_TRY(check_ws(ws, ws_bytes, kWsHeader));
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return COWA_ERR_INVALID_ARG;
  return launch_wait_timeout_probe(reinterpret_cast<uint32_t*>(ws), (unsigned long long)limit_ns,
                                   reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? COWA_OK
             : COWA_ERR_CUDA;
}

const char* cowa_status_string(cowa_status s) {
  switch (s) {
    case COWA_OK: return "ok";
    case COWA_ERR_INVALID_ARG: return "invalid argument (shape, pattern or null pointer)";
    case COWA_ERR_UNSUPPORTED: return "unsupported configuration (head dim must be 64 or 128, H_q/H_kv <= 8)";
    case COWA_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case COWA_ERR_WORKSPACE: return "workspace too small, null or not 256-byte aligned";
    case COWA_ERR_CUDA: return "CUDA error";
    case COWA_ERR_TIMEOUT: return "a device-side bounded wait ran out";
    case COWA_ERR_CHECK: return "a device-side self-check of the debug build failed";
  }
  return "unknown status";
}

cowa_status cowa_workspace_status(void* ws, void* stream) {
  if (!ws) return COWA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess) return COWA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return COWA_ERR_CUDA;
  if (word != 0) {
    // clear the status word and the self-check record (words 1 and 2) for the next call
    if (cudaMemsetAsync(ws, 0, 3 * sizeof(word), s) != cudaSuccess) return COWA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return COWA_ERR_CUDA;
    return (word & 2u) ? COWA_ERR_CHECK : COWA_ERR_TIMEOUT;
  }
  return COWA_OK;
}

// ------------------------------------------------------------------------------ decode
// ------------------------------------------------------------------------------ compacted cache
namespace {
constexpr int kCompactSpan = 1 << 30;  // positions are unbounded: the split count follows the pattern
}

int cowa_compact_rows(const cowa_pattern* pat, int Hkv) {
  Pat p;
  if (Hkv < 1 || check_pattern(pat, Hkv, &p) != COWA_OK) return 0;
  return compact_geom(p).rows;
}

cowa_status cowa_compact_build(const cowa_pattern* pat, int B, int N, int Hkv, int d, cowa_tensor k, cowa_tensor v,
                               void* k_compact, void* v_compact, void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  if (compact_geom(p).rows <= 0) return COWA_ERR_UNSUPPORTED;  // layout larger than an int row count
  COWA_TRY(check_heads(B, N, Hkv, Hkv, d));
  COWA_TRY(check_tensor(k));
  COWA_TRY(check_tensor(v));
  if (!k_compact || !v_compact) return COWA_ERR_INVALID_ARG;
  if (!aligned16(k_compact) || !aligned16(v_compact)) return COWA_ERR_ALIGNMENT;
  return launch_compact_build(p, B, N, Hkv, d, k.ptr, k.stride_b, k.stride_t, k.stride_h, v.ptr, v.stride_b,
                              v.stride_t, v.stride_h, k_compact, v_compact,
                              reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? COWA_OK
             : COWA_ERR_CUDA;
}

cowa_status cowa_compact_append(const cowa_pattern* pat, int B, int Hkv, int d, const void* k_new, const void* v_new,
                                const int32_t* pos, void* k_compact, void* v_compact, void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  if (compact_geom(p).rows <= 0) return COWA_ERR_UNSUPPORTED;  // layout larger than an int row count
  COWA_TRY(check_heads(B, 1, Hkv, Hkv, d));
  if (!k_new || !v_new || !pos || !k_compact || !v_compact) return COWA_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_compact) || !aligned16(v_compact))
    return COWA_ERR_ALIGNMENT;
  return launch_compact_append(p, B, Hkv, d, k_new, v_new, pos, k_compact, v_compact,
                               reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? COWA_OK
             : COWA_ERR_CUDA;
}

size_t cowa_decode_compact_workspace_size(const cowa_pattern* pat, int B, int Hq, int Hkv, int d) {
  Pat p;
  if (check_pattern(pat, Hkv, &p) != COWA_OK || check_heads(B, 1, Hq, Hkv, d) != COWA_OK) return 0;
  const int chunk = decode_chunk_tokens(p, B, Hkv, kCompactSpan);
  const int ns = decode_num_splits(p, kCompactSpan, chunk, true);
  return kWsHeader + align_up((size_t)B * Hq * ns * (d + 2) * sizeof(float), 256);
}

cowa_status cowa_decode_compact(const cowa_pattern* pat, int B, int Hq, int Hkv, int d, const void* q_t,
                                const void* k_compact, const void* v_compact, const int32_t* pos, void* o,
                                float* lse_or_null, void* ws, size_t ws_bytes, void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  if (compact_geom(p).rows <= 0) return COWA_ERR_UNSUPPORTED;  // layout larger than an int row count
  COWA_TRY(check_heads(B, 1, Hq, Hkv, d));
  if (!q_t || !pos || !o || !k_compact || !v_compact) return COWA_ERR_INVALID_ARG;
  if (!aligned16(q_t) || !aligned16(o) || !aligned16(k_compact) || !aligned16(v_compact) ||
      (lse_or_null && (reinterpret_cast<uintptr_t>(lse_or_null) & 3u)))
    return COWA_ERR_ALIGNMENT;
  COWA_TRY(check_ws(ws, ws_bytes, cowa_decode_compact_workspace_size(pat, B, Hq, Hkv, d)));

  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.pat = p; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d; a.T_cap = kCompactSpan;
  a.q_t = q_t; a.pos = pos; a.o = o; a.lse = lse_or_null;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.partials = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kWsHeader);
  a.chunk = decode_chunk_tokens(p, B, Hkv, kCompactSpan);
  a.n_split = decode_num_splits(p, kCompactSpan, a.chunk, true);
  a.scale_log2 = scale_of(pat, d) * 1.4426950408889634f;
  a.compact = 1;
  a.cg = compact_geom(p);
  const int64_t rows = a.cg.rows;
  if (!make_tmap_bf16(&a.tm_k, k_compact, d, (int)rows, Hkv, B, d, rows * d, (int64_t)Hkv * rows * d,
                      64) ||
      !make_tmap_bf16(&a.tm_v, v_compact, d, (int)rows, Hkv, B, d, rows * d, (int64_t)Hkv * rows * d,
                      64))
    return COWA_ERR_CUDA;
  return launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COWA_OK : COWA_ERR_CUDA;
}

size_t cowa_decode_workspace_size(const cowa_pattern* pat, int B, int Hq, int Hkv, int d, int T_cap) {
  Pat p;
  if (check_pattern(pat, Hkv, &p) != COWA_OK || check_heads(B, 1, Hq, Hkv, d) != COWA_OK || T_cap < 1) return 0;
  const int chunk = decode_chunk_tokens(p, B, Hkv, T_cap);
  const int ns = decode_num_splits(p, T_cap, chunk);
  return kWsHeader + align_up((size_t)B * Hq * ns * (d + 2) * sizeof(float), 256);
}

cowa_status cowa_decode(const cowa_pattern* pat, int B, int Hq, int Hkv, int d, int T_cap, const void* q_t,
                        cowa_tensor k_cache, cowa_tensor v_cache, const int32_t* pos, void* o, float* lse_or_null,
                        void* ws, size_t ws_bytes, void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  COWA_TRY(check_heads(B, 1, Hq, Hkv, d));
  if (T_cap < 1 || !q_t || !pos || !o) return COWA_ERR_INVALID_ARG;
  COWA_TRY(check_tensor(k_cache));
  COWA_TRY(check_tensor(v_cache));
  if (!aligned16(q_t) || !aligned16(o) || (lse_or_null && (reinterpret_cast<uintptr_t>(lse_or_null) & 3u)))
    return COWA_ERR_ALIGNMENT;
  COWA_TRY(check_ws(ws, ws_bytes, cowa_decode_workspace_size(pat, B, Hq, Hkv, d, T_cap)));

  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.pat = p; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d; a.T_cap = T_cap;
  a.q_t = q_t; a.pos = pos; a.o = o; a.lse = lse_or_null;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.partials = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kWsHeader);
  a.chunk = decode_chunk_tokens(p, B, Hkv, T_cap);
  a.n_split = decode_num_splits(p, T_cap, a.chunk);
  a.scale_log2 = scale_of(pat, d) * 1.4426950408889634f;
  if (!make_tmap_bf16(&a.tm_k, k_cache.ptr, d, T_cap, Hkv, B, k_cache.stride_t, k_cache.stride_h,
                      k_cache.stride_b, 64) ||
      !make_tmap_bf16(&a.tm_v, v_cache.ptr, d, T_cap, Hkv, B, v_cache.stride_t, v_cache.stride_h,
                      v_cache.stride_b, 64))
    return COWA_ERR_CUDA;
  return launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COWA_OK : COWA_ERR_CUDA;
}

// ------------------------------------------------------------------------------ E4M3 cache
size_t cowa_decode_fp8_workspace_size(const cowa_pattern* pat, int B, int Hq, int Hkv, int d, int T_cap) {
  return d == 128 ? cowa_decode_workspace_size(pat, B, Hq, Hkv, d, T_cap) : 0;
}

cowa_status cowa_decode_fp8(const cowa_pattern* pat, int B, int Hq, int Hkv, int d, int T_cap, const void* q_t,
                            cowa_tensor k_cache, cowa_tensor v_cache, float k_scale, float v_scale,
                            const int32_t* pos, void* o, float* lse_or_null, void* ws, size_t ws_bytes,
                            void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  COWA_TRY(check_heads(B, 1, Hq, Hkv, d));
  if (d != 128) return COWA_ERR_UNSUPPORTED;
  if (T_cap < 1 || !q_t || !pos || !o || !(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(k_scale) ||
      !isfinite(v_scale))
    return COWA_ERR_INVALID_ARG;
  COWA_TRY(check_tensor8(k_cache));
  COWA_TRY(check_tensor8(v_cache));
  if (!aligned16(q_t) || !aligned16(o) || (lse_or_null && (reinterpret_cast<uintptr_t>(lse_or_null) & 3u)))
    return COWA_ERR_ALIGNMENT;
  COWA_TRY(check_ws(ws, ws_bytes, cowa_decode_fp8_workspace_size(pat, B, Hq, Hkv, d, T_cap)));

  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.pat = p; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d; a.T_cap = T_cap;
  a.q_t = q_t; a.pos = pos; a.o = o; a.lse = lse_or_null;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.partials = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kWsHeader);
  a.chunk = decode_chunk_tokens(p, B, Hkv, T_cap);
  a.n_split = decode_num_splits(p, T_cap, a.chunk);
  a.scale_log2 = scale_of(pat, d) * 1.4426950408889634f * k_scale;
  a.kv8 = 1;
  a.v_scale = v_scale;
  if (!make_tmap_u8(&a.tm_k, k_cache.ptr, d, T_cap, Hkv, B, k_cache.stride_t, k_cache.stride_h, k_cache.stride_b,
                    64) ||
      !make_tmap_u8(&a.tm_v, v_cache.ptr, d, T_cap, Hkv, B, v_cache.stride_t, v_cache.stride_h, v_cache.stride_b,
                    64))
    return COWA_ERR_CUDA;
  return launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COWA_OK : COWA_ERR_CUDA;
}

// compacted E4M3 cache: rows of d = 128 codes (128 bytes, the row size of a d = 64 bf16 cache, so
// the row-copy kernels of the bf16 cache serve it with strides counted in 2-byte units)
cowa_status cowa_compact_build_fp8(const cowa_pattern* pat, int B, int N, int Hkv, int d, cowa_tensor k,
                                   cowa_tensor v, void* k_compact, void* v_compact, void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  if (compact_geom(p).rows <= 0) return COWA_ERR_UNSUPPORTED;  // layout larger than an int row count
  COWA_TRY(check_heads(B, N, Hkv, Hkv, d));
  if (d != 128) return COWA_ERR_UNSUPPORTED;
  COWA_TRY(check_tensor8(k));
  COWA_TRY(check_tensor8(v));
  if (!k_compact || !v_compact) return COWA_ERR_INVALID_ARG;
  if (!aligned16(k_compact) || !aligned16(v_compact)) return COWA_ERR_ALIGNMENT;
  return launch_compact_build(p, B, N, Hkv, 64, k.ptr, k.stride_b / 2, k.stride_t / 2, k.stride_h / 2, v.ptr,
                              v.stride_b / 2, v.stride_t / 2, v.stride_h / 2, k_compact, v_compact,
                              reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? COWA_OK
             : COWA_ERR_CUDA;
}

cowa_status cowa_compact_append_fp8(const cowa_pattern* pat, int B, int Hkv, int d, const void* k_new,
                                    const void* v_new, const int32_t* pos, void* k_compact, void* v_compact,
                                    void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  if (compact_geom(p).rows <= 0) return COWA_ERR_UNSUPPORTED;  // layout larger than an int row count
  COWA_TRY(check_heads(B, 1, Hkv, Hkv, d));
  if (d != 128) return COWA_ERR_UNSUPPORTED;
  if (!k_new || !v_new || !pos || !k_compact || !v_compact) return COWA_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_compact) || !aligned16(v_compact))
    return COWA_ERR_ALIGNMENT;
  return launch_compact_append(p, B, Hkv, 64, k_new, v_new, pos, k_compact, v_compact,
                               reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? COWA_OK
             : COWA_ERR_CUDA;
}

size_t cowa_decode_fp8_compact_workspace_size(const cowa_pattern* pat, int B, int Hq, int Hkv, int d) {
  return d == 128 ? cowa_decode_compact_workspace_size(pat, B, Hq, Hkv, d) : 0;
}

cowa_status cowa_decode_fp8_compact(const cowa_pattern* pat, int B, int Hq, int Hkv, int d, const void* q_t,
                                    const void* k_compact, const void* v_compact, float k_scale, float v_scale,
                                    const int32_t* pos, void* o, float* lse_or_null, void* ws, size_t ws_bytes,
                                    void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  if (compact_geom(p).rows <= 0) return COWA_ERR_UNSUPPORTED;  // layout larger than an int row count
  COWA_TRY(check_heads(B, 1, Hq, Hkv, d));
  if (d != 128) return COWA_ERR_UNSUPPORTED;
  if (!q_t || !pos || !o || !k_compact || !v_compact || !(k_scale > 0.f) || !(v_scale > 0.f) ||
      !isfinite(k_scale) || !isfinite(v_scale))
    return COWA_ERR_INVALID_ARG;
  if (!aligned16(q_t) || !aligned16(o) || !aligned16(k_compact) || !aligned16(v_compact) ||
      (lse_or_null && (reinterpret_cast<uintptr_t>(lse_or_null) & 3u)))
    return COWA_ERR_ALIGNMENT;
  COWA_TRY(check_ws(ws, ws_bytes, cowa_decode_fp8_compact_workspace_size(pat, B, Hq, Hkv, d)));

  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.pat = p; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d; a.T_cap = kCompactSpan;
  a.q_t = q_t; a.pos = pos; a.o = o; a.lse = lse_or_null;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.partials = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kWsHeader);
  a.chunk = decode_chunk_tokens(p, B, Hkv, kCompactSpan);
  a.n_split = decode_num_splits(p, kCompactSpan, a.chunk, true);
  a.scale_log2 = scale_of(pat, d) * 1.4426950408889634f * k_scale;
  a.compact = 1;
  a.cg = compact_geom(p);
  a.kv8 = 1;
  a.v_scale = v_scale;
  const int64_t rows = a.cg.rows;
  if (!make_tmap_u8(&a.tm_k, k_compact, d, (int)rows, Hkv, B, d, rows * d, (int64_t)Hkv * rows * d, 64) ||
      !make_tmap_u8(&a.tm_v, v_compact, d, (int)rows, Hkv, B, d, rows * d, (int64_t)Hkv * rows * d, 64))
    return COWA_ERR_CUDA;
  return launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COWA_OK : COWA_ERR_CUDA;
}

cowa_status cowa_quantize_e4m3(const void* x, void* codes, int64_t n, float scale, void* stream) {
  if (!x || !codes || n < 0 || n % 8 != 0 || !(scale > 0.f) || !isfinite(scale)) return COWA_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(codes) & 7u)) return COWA_ERR_ALIGNMENT;
  const float inv = 1.0f / scale;
  return launch_quantize_e4m3(x, codes, n, inv, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? COWA_OK
             : COWA_ERR_CUDA;
}

// ------------------------------------------------------------------------------ forward
size_t cowa_fwd_workspace_size(const cowa_pattern* pat, int B, int N, int Hq, int Hkv, int d) {
  Pat p;
  if (check_pattern(pat, Hkv, &p) != COWA_OK || check_heads(B, N, Hq, Hkv, d) != COWA_OK) return 0;
  return kWsHeader;
}

cowa_status cowa_fwd(const cowa_pattern* pat, int B, int N, int Hq, int Hkv, int d, cowa_tensor q, cowa_tensor k,
                     cowa_tensor v, cowa_tensor o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  return cowa_fwd_chunk(pat, B, N, N, 0, Hq, Hkv, d, q, k, v, o, lse, ws, ws_bytes, stream);
}

cowa_status cowa_fwd_chunk(const cowa_pattern* pat, int B, int N_q, int N_k, int q_offset, int Hq, int Hkv, int d,
                           cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o, float* lse, void* ws,
                           size_t ws_bytes, void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  COWA_TRY(check_heads(B, N_q, Hq, Hkv, d));
  if (q_offset < 0 || N_k < 1 || (int64_t)q_offset + N_q > (int64_t)N_k) return COWA_ERR_INVALID_ARG;
  COWA_TRY(check_tensor(q));
  COWA_TRY(check_tensor(k));
  COWA_TRY(check_tensor(v));
  COWA_TRY(check_tensor(o));
  if (!lse) return COWA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return COWA_ERR_ALIGNMENT;
  COWA_TRY(check_ws(ws, ws_bytes, cowa_fwd_workspace_size(pat, B, N_q, Hq, Hkv, d)));

  FwdArgs a;
  memset(&a, 0, sizeof(a));
  a.pat = p; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.Nq = N_q; a.Nk = N_k; a.q_off = q_offset;
  a.o = o.ptr; a.o_sb = o.stride_b; a.o_st = o.stride_t; a.o_sh = o.stride_h;
  a.lse = lse;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.scale_log2 = scale_of(pat, d) * 1.4426950408889634f;
  if (!make_tmap_bf16(&a.tm_q, q.ptr, d, N_q, Hq, B, q.stride_t, q.stride_h, q.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_k, k.ptr, d, N_k, Hkv, B, k.stride_t, k.stride_h, k.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_v, v.ptr, d, N_k, Hkv, B, v.stride_t, v.stride_h, v.stride_b, 128))
    return COWA_ERR_CUDA;
  return launch_fwd(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COWA_OK : COWA_ERR_CUDA;
}

size_t cowa_fwd_varlen_workspace_size(const cowa_pattern* pat, int n_seq, int total, int Hq, int Hkv, int d) {
  Pat p;
  if (n_seq < 1 || check_pattern(pat, Hkv, &p) != COWA_OK || check_heads(1, total, Hq, Hkv, d) != COWA_OK) return 0;
  return kWsHeader + seq_table_bytes(n_seq);
}

cowa_status cowa_fwd_varlen(const cowa_pattern* pat, int n_seq, int total, int Hq, int Hkv, int d,
                            const int32_t* cu_seqlens, cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o,
                            float* lse, void* ws, size_t ws_bytes, void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  COWA_TRY(check_heads(1, total, Hq, Hkv, d));
  if (n_seq < 1 || !cu_seqlens || !lse) return COWA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return COWA_ERR_ALIGNMENT;
  COWA_TRY(check_tensor(q));
  COWA_TRY(check_tensor(k));
  COWA_TRY(check_tensor(v));
  COWA_TRY(check_tensor(o));
  COWA_TRY(check_ws(ws, ws_bytes, cowa_fwd_varlen_workspace_size(pat, n_seq, total, Hq, Hkv, d)));

  FwdArgs a;
  memset(&a, 0, sizeof(a));
  a.pat = p; a.B = 1; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.Nq = total; a.Nk = total; a.q_off = 0;
  a.varlen = 1; a.n_seq = n_seq; a.total = total; a.cu_seqlens = cu_seqlens;
  a.seq_tab = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(ws) + kWsHeader);
  a.o = o.ptr; a.o_sb = 0; a.o_st = o.stride_t; a.o_sh = o.stride_h;
  a.lse = lse;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.scale_log2 = scale_of(pat, d) * 1.4426950408889634f;
  if (!make_tmap_bf16(&a.tm_q, q.ptr, d, total, Hq, 1, q.stride_t, q.stride_h, q.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_k, k.ptr, d, total, Hkv, 1, k.stride_t, k.stride_h, k.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_v, v.ptr, d, total, Hkv, 1, v.stride_t, v.stride_h, v.stride_b, 128))
    return COWA_ERR_CUDA;
  return launch_fwd(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COWA_OK : COWA_ERR_CUDA;
}

// ------------------------------------------------------------------------------ backward
size_t cowa_bwd_workspace_size(const cowa_pattern* pat, int B, int N, int Hq, int Hkv, int d) {
  Pat p;
  if (check_pattern(pat, Hkv, &p) != COWA_OK || check_heads(B, N, Hq, Hkv, d) != COWA_OK) return 0;
  return kWsHeader + bwd_workspace_bytes(p, B, N, Hq, Hkv, d);
}

cowa_status cowa_bwd(const cowa_pattern* pat, int B, int N, int Hq, int Hkv, int d, cowa_tensor q, cowa_tensor k,
                     cowa_tensor v, cowa_tensor o, const float* lse, cowa_tensor dO, cowa_tensor dq, cowa_tensor dk,
                     cowa_tensor dv, void* ws, size_t ws_bytes, void* stream) {
  return cowa_bwd_stages(pat, B, N, Hq, Hkv, d, q, k, v, o, lse, dO, dq, dk, dv,
                         COWA_BWD_PREPROCESS | COWA_BWD_DKDV | COWA_BWD_DQ, ws, ws_bytes, stream);
}

cowa_status cowa_bwd_stages(const cowa_pattern* pat, int B, int N, int Hq, int Hkv, int d, cowa_tensor q,
                            cowa_tensor k, cowa_tensor v, cowa_tensor o, const float* lse, cowa_tensor dO,
                            cowa_tensor dq, cowa_tensor dk, cowa_tensor dv, int stages, void* ws, size_t ws_bytes,
                            void* stream) {
  if (stages <= 0 || stages > (COWA_BWD_PREPROCESS | COWA_BWD_DKDV | COWA_BWD_DQ)) return COWA_ERR_INVALID_ARG;
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  COWA_TRY(check_heads(B, N, Hq, Hkv, d));
  const cowa_tensor* all[] = {&q, &k, &v, &o, &dO, &dq, &dk, &dv};
  for (const cowa_tensor* t : all) COWA_TRY(check_tensor(*t));
  if (!lse) return COWA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return COWA_ERR_ALIGNMENT;
  COWA_TRY(check_ws(ws, ws_bytes, cowa_bwd_workspace_size(pat, B, N, Hq, Hkv, d)));

  BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.pat = p; a.B = B; a.N = N; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.o = o.ptr; a.o_sb = o.stride_b; a.o_st = o.stride_t; a.o_sh = o.stride_h;
  a.dO = dO.ptr; a.do_sb = dO.stride_b; a.do_st = dO.stride_t; a.do_sh = dO.stride_h;
  a.lse = lse;
  a.dq = dq.ptr; a.dq_sb = dq.stride_b; a.dq_st = dq.stride_t; a.dq_sh = dq.stride_h;
  a.dk = dk.ptr; a.dk_sb = dk.stride_b; a.dk_st = dk.stride_t; a.dk_sh = dk.stride_h;
  a.dv = dv.ptr; a.dv_sb = dv.stride_b; a.dv_st = dv.stride_t; a.dv_sh = dv.stride_h;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.lse_ld = N;
  a.N_pad = (N + 127) / 128 * 128;
  a.delta = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kWsHeader);
  a.lse2 = a.delta + (size_t)B * Hq * a.N_pad;
  {
    // long dK/dV key tiles split by query range: chunk table and fp32 partials after the statistics
    const KvSplit sp = kv_split_plan(p, B, N, Hq, Hkv);
    if (sp.chunk > 0) {
      if (sp.n_entries > 0x7fffffffLL) return COWA_ERR_UNSUPPORTED;
      char* base = reinterpret_cast<char*>(ws) + kWsHeader + align_up(2 * (size_t)B * Hq * a.N_pad * sizeof(float), 256);
      a.kv_chunk = sp.chunk;
      a.n_split = (int)sp.n_entries;
      a.kv_tab = reinterpret_cast<int4*>(base);
      a.kv_part = reinterpret_cast<float*>(base + align_up((size_t)sp.n_entries * sizeof(int4), 256));
    }
  }
  a.scale = scale_of(pat, d);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  if (!make_tmap_bf16(&a.tm_q, q.ptr, d, N, Hq, B, q.stride_t, q.stride_h, q.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_k, k.ptr, d, N, Hkv, B, k.stride_t, k.stride_h, k.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_v, v.ptr, d, N, Hkv, B, v.stride_t, v.stride_h, v.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_do, dO.ptr, d, N, Hq, B, dO.stride_t, dO.stride_h, dO.stride_b, 128))
    return COWA_ERR_CUDA;
  return launch_bwd(a, stages, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? COWA_OK : COWA_ERR_CUDA;
}

// ------------------------------------------------------------------------------ packed backward
namespace {
// 128 x the tile bound of a packed batch: every sequence's statistics start at its own tile
long long packed_rows_pad(int total, int n_seq) { return packed_tiles_bound(total, n_seq) * 128; }

// The key-tile split of a packed batch is planned as for one sequence of all `total` rows (the
// longest ranges a batch of that size can have); the device fills a table of `cap` slots.
int varlen_split_cap(const Pat& p, int total, int Hq, int Hkv, int* chunk) {
  const KvSplit sp = kv_split_plan(p, 1, total, Hq, Hkv);
  *chunk = sp.chunk;
  if (sp.chunk == 0) return 0;
  const long long cap = 2 * sp.n_entries + 64;
  return cap > 0x7fffffffLL ? -1 : (int)cap;
}

size_t varlen_split_bytes(int cap, int Hkv, long long rows, int d) {
  if (cap <= 0) return 0;
  return align_up((size_t)Hkv * (size_t)(rows / 128) * sizeof(int32_t), 256) + align_up((size_t)cap * sizeof(int4), 256) +
         (size_t)cap * 2 * 128 * d * sizeof(float);
}
}  // namespace

size_t cowa_bwd_varlen_workspace_size(const cowa_pattern* pat, int n_seq, int total, int Hq, int Hkv, int d) {
  Pat p;
  if (n_seq < 1 || check_pattern(pat, Hkv, &p) != COWA_OK || check_heads(1, total, Hq, Hkv, d) != COWA_OK) return 0;
  const long long rows = packed_rows_pad(total, n_seq);
  if (rows > 0x7fffffffLL) return 0;
  int chunk;
  const int cap = varlen_split_cap(p, total, Hq, Hkv, &chunk);
  if (cap < 0) return 0;
  return kWsHeader + seq_table_bytes(n_seq) + align_up(2 * (size_t)Hq * (size_t)rows * sizeof(float), 256) +
         varlen_split_bytes(cap, Hkv, rows, d);
}

cowa_status cowa_bwd_varlen(const cowa_pattern* pat, int n_seq, int total, int Hq, int Hkv, int d,
                            const int32_t* cu_seqlens, cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o,
                            const float* lse, cowa_tensor dO, cowa_tensor dq, cowa_tensor dk, cowa_tensor dv,
                            void* ws, size_t ws_bytes, void* stream) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  COWA_TRY(check_heads(1, total, Hq, Hkv, d));
  if (n_seq < 1 || !cu_seqlens || !lse) return COWA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return COWA_ERR_ALIGNMENT;
  const cowa_tensor* all[] = {&q, &k, &v, &o, &dO, &dq, &dk, &dv};
  for (const cowa_tensor* t : all) COWA_TRY(check_tensor(*t));
  const size_t need = cowa_bwd_varlen_workspace_size(pat, n_seq, total, Hq, Hkv, d);
  if (need == 0) return COWA_ERR_INVALID_ARG;
  COWA_TRY(check_ws(ws, ws_bytes, need));

  BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.pat = p; a.B = 1; a.N = total; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.varlen = 1; a.n_seq = n_seq; a.total = total;
  a.seq_tab = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(ws) + kWsHeader);
  a.o = o.ptr; a.o_sb = 0; a.o_st = o.stride_t; a.o_sh = o.stride_h;
  a.dO = dO.ptr; a.do_sb = 0; a.do_st = dO.stride_t; a.do_sh = dO.stride_h;
  a.lse = lse;
  a.lse_ld = total;
  a.dq = dq.ptr; a.dq_sb = 0; a.dq_st = dq.stride_t; a.dq_sh = dq.stride_h;
  a.dk = dk.ptr; a.dk_sb = 0; a.dk_st = dk.stride_t; a.dk_sh = dk.stride_h;
  a.dv = dv.ptr; a.dv_sb = 0; a.dv_st = dv.stride_t; a.dv_sh = dv.stride_h;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.N_pad = (int)packed_rows_pad(total, n_seq);
  a.delta = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kWsHeader + seq_table_bytes(n_seq));
  a.lse2 = a.delta + (size_t)Hq * a.N_pad;
  {
    // long key tiles split by query range, planned on the device: flags, table, fp32 partials
    int chunk;
    const int cap = varlen_split_cap(p, total, Hq, Hkv, &chunk);
    if (cap > 0) {
      char* base = reinterpret_cast<char*>(a.lse2 + (size_t)Hq * a.N_pad);
      base = reinterpret_cast<char*>(ws) + align_up((size_t)(base - reinterpret_cast<char*>(ws)), 256);
      a.kv_chunk = chunk;
      a.n_split = cap;
      a.kv_bound = a.N_pad / 128;
      a.kv_flag = reinterpret_cast<int32_t*>(base);
      base += align_up((size_t)Hkv * a.kv_bound * sizeof(int32_t), 256);
      a.kv_tab = reinterpret_cast<int4*>(base);
      a.kv_part = reinterpret_cast<float*>(base + align_up((size_t)cap * sizeof(int4), 256));
    }
  }
  a.scale = scale_of(pat, d);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  if (!make_tmap_bf16(&a.tm_q, q.ptr, d, total, Hq, 1, q.stride_t, q.stride_h, q.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_k, k.ptr, d, total, Hkv, 1, k.stride_t, k.stride_h, k.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_v, v.ptr, d, total, Hkv, 1, v.stride_t, v.stride_h, v.stride_b, 128) ||
      !make_tmap_bf16(&a.tm_do, dO.ptr, d, total, Hq, 1, dO.stride_t, dO.stride_h, dO.stride_b, 128))
    return COWA_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (launch_seq_table(cu_seqlens, n_seq, total, a.seq_tab, st) != cudaSuccess) return COWA_ERR_CUDA;
  return launch_bwd(a, COWA_BWD_PREPROCESS | COWA_BWD_DKDV | COWA_BWD_DQ, st) == cudaSuccess ? COWA_OK
                                                                                            : COWA_ERR_CUDA;
}

// ------------------------------------------------------------------------------ introspection
cowa_status cowa_visible_counts(const cowa_pattern* pat, int Hkv, int N, int64_t* out) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  if (N < 1 || !out) return COWA_ERR_INVALID_ARG;
  for (int g = 0; g < Hkv; ++g) {
    const Range iv = interval_of(p, g);
    for (int t = 0; t < N; ++t) {
      Range r[3];
      const int n = row_ranges(p, iv, t, r);
      int64_t c = 0;
      for (int i = 0; i < n; ++i) c += r[i].hi - r[i].lo;
      out[(size_t)g * N + t] = c;
    }
  }
  return COWA_OK;
}

cowa_status cowa_plan_debug(const cowa_pattern* pat, int Hkv, int N, int BM, int BN, int which, int32_t* out,
                            size_t cap, size_t* n_written, void* dev_scratch) {
  Pat p;
  COWA_TRY(check_pattern(pat, Hkv, &p));
  if (N < 1 || BM < 1 || BN < 1 || !out || !n_written || which < 0 || which > 2) return COWA_ERR_INVALID_ARG;
  size_t n = 0;
  auto emit = [&](int a0, int a1, int a2, int a3) {
    if (n < cap) {
      out[4 * n + 0] = a0; out[4 * n + 1] = a1; out[4 * n + 2] = a2; out[4 * n + 3] = a3;
    }
    ++n;
  };
  const int nq = (N + BM - 1) / BM, nk = (N + BN - 1) / BN;
  if (which == 0) {
    for (int g = 0; g < Hkv; ++g) {
      const Range iv = interval_of(p, g);
      for (int i = 0; i < nq; ++i) {
        const int t0 = i * BM, t1 = imin(N, t0 + BM);
        Range r[3];
        const int nr = fwd_tile_ranges(p, iv, t0, t1, BN, r);
        for (int x = 0; x < nr; ++x)
          for (int j = r[x].lo; j < r[x].hi; ++j)
            emit(g, i, j, tile_full(p, iv, t0, t1, j * BN, imin(N, j * BN + BN)) ? 1 : 0);
      }
    }
  } else if (which == 1) {
    for (int g = 0; g < Hkv; ++g) {
      const Range iv = interval_of(p, g);
      for (int j = 0; j < nk; ++j) {
        const Range rows = bwd_row_range(p, iv, j * BN, imin(N, j * BN + BN), N);
        if (rows.lo >= rows.hi) continue;
        for (int i = rows.lo / BM; i < (rows.hi + BM - 1) / BM; ++i) emit(g, j, i, 0);
      }
    }
  } else {
    if (!dev_scratch) return COWA_ERR_INVALID_ARG;
    unsigned long long* dcount = reinterpret_cast<unsigned long long*>(dev_scratch);
    int32_t* drec = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(dev_scratch) + 256);
    if (cudaMemset(dcount, 0, sizeof(unsigned long long)) != cudaSuccess) return COWA_ERR_CUDA;
    const size_t dcap = cap;  // the first 256 bytes of dev_scratch hold the counter
    if (launch_plan_debug(p, Hkv, N, BM, BN, drec, dcap, dcount, 0) != cudaSuccess) return COWA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return COWA_ERR_CUDA;
    unsigned long long cnt = 0;
    if (cudaMemcpy(&cnt, dcount, sizeof(cnt), cudaMemcpyDeviceToHost) != cudaSuccess) return COWA_ERR_CUDA;
    n = (size_t)cnt;
    const size_t ncopy = n < dcap ? n : dcap;
    if (ncopy && cudaMemcpy(out, drec, ncopy * 16, cudaMemcpyDeviceToHost) != cudaSuccess) return COWA_ERR_CUDA;
    *n_written = n;
    return n > dcap ? COWA_ERR_WORKSPACE : COWA_OK;
  }
  *n_written = n;
  return n > cap ? COWA_ERR_WORKSPACE : COWA_OK;
}

}  // extern "C"
