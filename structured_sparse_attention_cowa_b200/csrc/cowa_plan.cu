// cowa_plan.cu -- device-side evaluation of the forward tile plan, for introspection, and the
// bounded-wait probe.  The plan kernel runs exactly the planner code (cowa_pattern.h) that the
// attention kernels run on the fly, so a host test can compare the device plan with the host
// plan and the mask.  The probe kernel exercises the timeout path every kernel's waits share.
#include "cowa_internal.h"
#include "sm100_ptx.cuh"

namespace cowa {
namespace {

__global__ void plan_debug_kernel(Pat p, int Hkv, int N, int BM, int BN, int32_t* out, size_t cap,
                                  unsigned long long* count) {
  const int nq = (N + BM - 1) / BM;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= nq * Hkv) return;
  const int g = idx / nq, i = idx % nq;
  const Range iv = interval_of(p, g);
  const int t0 = i * BM, t1 = imin(N, t0 + BM);
  Range r[3];
  const int nr = fwd_tile_ranges(p, iv, t0, t1, BN, r);
  for (int x = 0; x < nr; ++x) {
    for (int j = r[x].lo; j < r[x].hi; ++j) {
      const unsigned long long slot = atomicAdd(count, 1ull);
      if (slot < cap) {
        int4 rec = make_int4(g, i, j, tile_full(p, iv, t0, t1, j * BN, imin(N, j * BN + BN)) ? 1 : 0);
        reinterpret_cast<int4*>(out)[slot] = rec;
      }
    }
  }
}

// One thread waits on an mbarrier that nothing will ever arrive on.  The wait gives up after
// limit_ns, records the timeout in the status word and the kernel returns normally.
__global__ void wait_timeout_probe_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  ptx::mbar_init(&bar, 1);
  ptx::fence_mbar_init();
  ptx::mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

}  // namespace

cudaError_t launch_wait_timeout_probe(uint32_t* status, unsigned long long limit_ns, cudaStream_t s) {
  wait_timeout_probe_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_plan_debug(const Pat& p, int Hkv, int N, int BM, int BN, int32_t* dev_out, size_t cap,
                              unsigned long long* dev_count, cudaStream_t s) {
  const int items = ((N + BM - 1) / BM) * Hkv;
  plan_debug_kernel<<<(items + 127) / 128, 128, 0, s>>>(p, Hkv, N, BM, BN, dev_out, cap, dev_count);
  return cudaGetLastError();
}

}  // namespace cowa
