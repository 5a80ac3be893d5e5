// cowa_decode_noalloc.cu -- cowa_decode for callers that cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: inference runtimes and
// plugin hosts that reserve the whole device memory pool up front and forbid any further
// allocation on the serving path, or code that must not call cudaMalloc because it would
// synchronize the device in the middle of a latency-critical step.  For them the decode
// split partials and the status word live in a scratch array that is part of the library
// image itself: a file-scope __device__ variable, created once in every GPU's memory when
// the library's code is loaded there and kept until the process exits.  The caller still
// passes every input and output buffer.
//
// Nothing here allocates: the scratch address of each device is looked up once (on the
// first call made with that device current, and again only after that device's context has
// been replaced, e.g. by cudaDeviceReset) with cudaGetSymbolAddress, the status word is
// cleared with an asynchronous memset on the caller's stream, and the ordinary decode path
// runs with the scratch array as its workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "cowa_internal.h"

namespace cowa {
namespace {

// The scratch array.  Its name is only meaningful to device code and to the runtime's
// symbol lookup; host code must use the address returned by cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[COWA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchAddr {
  void* ptr = nullptr;             // device address of g_decode_scratch
  unsigned long long ctx_id = 0;   // the context it was looked up in
};
ScratchAddr g_scratch_addr[kMaxDevices];  // per device ordinal

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

void* driver_entry(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

// Unique id of the calling thread's current context (0 if there is none).  A device reset
// destroys the context the scratch address was looked up in; the library's device code is
// loaded again in the next context, possibly at another address, so the address is only
// reused while the context is the same one.
unsigned long long current_ctx_id() {
  static const CtxGetCurrentFn get_cur = reinterpret_cast<CtxGetCurrentFn>(driver_entry("cuCtxGetCurrent"));
  static const CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_entry("cuCtxGetId"));
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device: looked up once per device (and
// again only if that device's context has changed since).
cowa_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return COWA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr& e = g_scratch_addr[dev];
  unsigned long long id = current_ctx_id();
  if (e.ptr == nullptr || id == 0 || id != e.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return COWA_ERR_CUDA;
    if (id == 0) id = current_ctx_id();  // the lookup made the device's primary context current
    e.ptr = p;
    e.ctx_id = id;
  }
  *out = e.ptr;
  return COWA_OK;
}

}  // namespace
}  // namespace cowa

extern "C" cowa_status cowa_decode_noalloc(const cowa_pattern* pat, int B, int H_q, int H_kv, int d, int T_cap,
                                           const void* q_t, cowa_tensor k_cache, cowa_tensor v_cache,
                                           const int32_t* pos, void* o, float* lse_or_null, void* stream) {
  const size_t need = cowa_decode_workspace_size(pat, B, H_q, H_kv, d, T_cap);
  if (need == 0) {
    // invalid or unsupported arguments: let the ordinary entry point name the error (it
    // validates everything before it looks at a workspace and launches nothing)
    return cowa_decode(pat, B, H_q, H_kv, d, T_cap, q_t, k_cache, v_cache, pos, o, lse_or_null, nullptr, 0,
                       stream);
  }
  if (need > COWA_DECODE_NOALLOC_SCRATCH_BYTES) return COWA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const cowa_status st = cowa::scratch_on_current_device(&scratch);
  if (st != COWA_OK) return st;
  // the status word must start at zero; the split partials are fully rewritten by every call
  if (cudaMemsetAsync(scratch, 0, cowa::kWsHeader, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return COWA_ERR_CUDA;
  return cowa_decode(pat, B, H_q, H_kv, d, T_cap, q_t, k_cache, v_cache, pos, o, lse_or_null, scratch,
                     COWA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" cowa_status cowa_decode_noalloc_status(void* stream) {
  void* scratch = nullptr;
  const cowa_status st = cowa::scratch_on_current_device(&scratch);
  if (st != COWA_OK) return st;
  return cowa_workspace_status(scratch, stream);
}
