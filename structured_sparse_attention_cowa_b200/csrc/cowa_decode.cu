// cowa_decode.cu -- split-KV CoWA decode: one new query token per sequence attends to the
// keys its KV head can see in the cache ("CoWindow Attention: Full Causal Coverage Is a
// Collective Property", Abstract: decoding with the same position-defined pattern as
// training; skillfed.io news summary, paragraph 4).
//
// HBM-bound: per (b, g) only the <= 3 visible token ranges at pos[b] (sink, interval_g,
// near-diagonal band) are read.  Each CTA owns one chunk of one range:
//   * a producer warp streams 64-token K and V sub-tiles into a shared-memory ring with
//     TMA (128-byte swizzle, coalesced 128-byte rows, no register staging);
//   * 8 compute warps: 8 lanes per token row, each lane one 16-byte unit per 64-wide
//     slice of d (128-bit shared loads, conflict-free under the swizzle), scores for all
//     query heads of the GQA group from fp32 registers, a 3-step shuffle reduction, an
//     online softmax in the log2 domain, and P*V accumulation in fp32;
//   * the lanes' partial (m, l, o) states are merged with shuffles, then across warps in
//     shared memory, and written as one fp32 partial per (b, h, split).
// A second kernel merges the splits of each (b, h) (max / rescaled sums, warp shuffles)
// and writes bf16 o and the fp32 lse.
#include <cuda_bf16.h>
#include <math.h>

#include "cowa_internal.h"
#include "sm100_ptx.cuh"

namespace cowa {
namespace {

constexpr int kDecWarps = 8;                        // compute warps per CTA
constexpr int kDecThreads = (kDecWarps + 1) * 32;   // + one TMA producer warp
constexpr int kSubTok = 64;                         // tokens per sub-tile (TMA box rows)
constexpr int kStages = 3;                          // sub-tile ring depth
constexpr int kBoxBytes = kSubTok * 128;            // one [64 rows x 64 bf16] box

template <int D>
struct DecGeom {
  static constexpr int kUnits = D / 64;                  // 16-byte units per lane per row
  static constexpr int kEPT = 8 * kUnits;                // elements per lane
  static constexpr int kTileBytes = kUnits * kBoxBytes;  // K (or V) sub-tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ float safe_ex2_diff(float a, float m) {
  // exp2(a - m) with a == -inf giving 0 even when m == -inf
  return a == -INFINITY ? 0.f : ptx::ex2(a - m);
}

template <int GRP, int D>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const __grid_constant__ DecodeArgs a) {
  using Geo = DecGeom<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ int abort_flag;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which chunk of which visible range this CTA owns (pure position arithmetic)
  int t = a.pos[b];
  t = t < 0 ? 0 : (t >= a.T_cap ? a.T_cap - 1 : t);
  const Range iv = interval_of(a.pat, g);
  Range rr[3];
  const int nr = row_ranges(a.pat, iv, t, rr);
  int c_lo = 0, c_hi = 0;
  {
    int idx = split;
    for (int r = 0; r < nr; ++r) {
      const int nch = (rr[r].hi - rr[r].lo + a.chunk - 1) / a.chunk;
      if (idx < nch) {
        c_lo = rr[r].lo + idx * a.chunk;
        c_hi = imin(rr[r].hi, c_lo + a.chunk);
        break;
      }
      idx -= nch;
    }
  }
  const int nsub = (c_hi - c_lo + kSubTok - 1) / kSubTok;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full_bar[s], 1);
      ptx::mbar_init(&empty_bar[s], kDecWarps);
    }
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecWarps) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::tma_prefetch_desc(&a.tm_k);
      ptx::tma_prefetch_desc(&a.tm_v);
      int issued = 0;
      for (int st = 0; st < nsub; ++st) {
        const int s = st % kStages;
        const uint32_t ph = (st / kStages) & 1;
        if (st >= kStages && !ptx::mbar_wait(&empty_bar[s], ph ^ 1, &abort_flag, a.status)) break;
        uint8_t* ks = smem + s * Geo::kStageBytes;
        uint8_t* vs = ks + Geo::kTileBytes;
        ptx::mbar_arrive_expect_tx(&full_bar[s], Geo::kStageBytes);
        const int t0 = c_lo + st * kSubTok;
#pragma unroll
        for (int u = 0; u < Geo::kUnits; ++u) {
          ptx::tma_load_4d(ks + u * kBoxBytes, &a.tm_k, &full_bar[s], u * 64, t0, g, b);
          ptx::tma_load_4d(vs + u * kBoxBytes, &a.tm_v, &full_bar[s], u * 64, t0, g, b);
        }
        issued = st + 1;
      }
      // never leave the CTA with copies in flight: wait for the last ones to land
      for (int st = (issued > kStages ? issued - kStages : 0); st < issued; ++st)
        ptx::mbar_wait(&full_bar[st % kStages], (st / kStages) & 1, nullptr, a.status);
    }
    return;
  }

  // ------------------------------------------------------------------ compute warps
  constexpr int EPT = Geo::kEPT;
  const int slot = lane >> 3;  // token slot of a 4-token step
  const int j = lane & 7;      // 16-byte unit within each 64-element slice of d
  float q[GRP][EPT];
  float acc[GRP][EPT];
  float m[GRP], l[GRP];
  {
    const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(a.q_t) + ((size_t)b * a.Hq + (size_t)g * GRP) * D;
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
#pragma unroll
      for (int u = 0; u < Geo::kUnits; ++u) {
        const uint4 w = *reinterpret_cast<const uint4*>(qb + hh * D + u * 64 + j * 8);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          q[hh][u * 8 + 2 * e] = bf16lo(ww[e]) * a.scale_log2;
          q[hh][u * 8 + 2 * e + 1] = bf16hi(ww[e]) * a.scale_log2;
        }
      }
#pragma unroll
      for (int e = 0; e < EPT; ++e) acc[hh][e] = 0.f;
      m[hh] = -INFINITY;
      l[hh] = 0.f;
    }
  }

  const uint32_t smem_base = ptx::smem_u32(smem);
  bool ok = true;
  for (int st = 0; st < nsub; ++st) {
    const int s = st % kStages;
    if (!ptx::mbar_wait_warp(&full_bar[s], (st / kStages) & 1, &abort_flag, a.status)) { ok = false; break; }
    const uint32_t ks = smem_base + s * Geo::kStageBytes;
    const uint32_t vs = ks + Geo::kTileBytes;
#pragma unroll
    for (int step = 0; step < kSubTok / (kDecWarps * 4); ++step) {
      const int r = warp * (kSubTok / kDecWarps) + step * 4 + slot;  // row in the sub-tile
      const int tok = c_lo + st * kSubTok + r;
      const bool valid = tok < c_hi;
      const uint32_t off = r * 128 + ((j ^ (r & 7)) << 4);  // 128-byte swizzle
      float sc[GRP];
#pragma unroll
      for (int hh = 0; hh < GRP; ++hh) sc[hh] = 0.f;
#pragma unroll
      for (int u = 0; u < Geo::kUnits; ++u) {
        const uint4 kw = lds128(ks + u * kBoxBytes + off);
        const uint32_t ww[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float k0 = bf16lo(ww[e]), k1 = bf16hi(ww[e]);
#pragma unroll
          for (int hh = 0; hh < GRP; ++hh) {
            sc[hh] = fmaf(q[hh][u * 8 + 2 * e], k0, sc[hh]);
            sc[hh] = fmaf(q[hh][u * 8 + 2 * e + 1], k1, sc[hh]);
          }
        }
      }
      float p[GRP];
#pragma unroll
      for (int hh = 0; hh < GRP; ++hh) {
        float x = sc[hh];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x = valid ? x : -INFINITY;
        if (x > m[hh]) {
          const float f = safe_ex2_diff(m[hh], x);
          l[hh] *= f;
#pragma unroll
          for (int e = 0; e < EPT; ++e) acc[hh][e] *= f;
          m[hh] = x;
        }
        p[hh] = valid ? ptx::ex2(x - m[hh]) : 0.f;
        l[hh] += p[hh];
      }
#pragma unroll
      for (int u = 0; u < Geo::kUnits; ++u) {
        const uint4 vw = lds128(vs + u * kBoxBytes + off);
        const uint32_t ww[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v0 = bf16lo(ww[e]), v1 = bf16hi(ww[e]);
#pragma unroll
          for (int hh = 0; hh < GRP; ++hh) {
            acc[hh][u * 8 + 2 * e] = fmaf(p[hh], v0, acc[hh][u * 8 + 2 * e]);
            acc[hh][u * 8 + 2 * e + 1] = fmaf(p[hh], v1, acc[hh][u * 8 + 2 * e + 1]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty_bar[s]);
  }

  // ---- merge the four token slots of the warp (lanes j, j+8, j+16, j+24)
#pragma unroll
  for (int offs = 8; offs <= 16; offs <<= 1) {
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[hh], offs);
      const float lo = __shfl_xor_sync(0xffffffffu, l[hh], offs);
      const float mn = fmaxf(m[hh], mo);
      const float fa = safe_ex2_diff(m[hh], mn), fb = safe_ex2_diff(mo, mn);
      l[hh] = l[hh] * fa + lo * fb;
#pragma unroll
      for (int e = 0; e < EPT; ++e) {
        const float ao = __shfl_xor_sync(0xffffffffu, acc[hh][e], offs);
        acc[hh][e] = acc[hh][e] * fa + ao * fb;
      }
      m[hh] = mn;
    }
  }

  // ---- merge the warps through shared memory (the ring is drained: reuse it)
  asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
  if (!ok || abort_flag) return;
  float* red = reinterpret_cast<float*>(smem);  // [warp][GRP][D + 2]
  if (lane < 8) {
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
      float* rw = red + (warp * GRP + hh) * (D + 2);
      if (lane == 0) { rw[0] = m[hh]; rw[1] = l[hh]; }
#pragma unroll
      for (int u = 0; u < Geo::kUnits; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) rw[2 + u * 64 + j * 8 + e] = acc[hh][u * 8 + e];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
  for (int x = threadIdx.x; x < GRP * D; x += kDecWarps * 32) {
    const int hh = x / D, dc = x % D;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) mx = fmaxf(mx, red[(w * GRP + hh) * (D + 2)]);
    float o = 0.f, ll = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float* rw = red + (w * GRP + hh) * (D + 2);
      const float f = safe_ex2_diff(rw[0], mx);
      o += f * rw[2 + dc];
      ll += f * rw[1];
    }
    const int h = g * GRP + hh;
    float* out = a.partials + (((size_t)b * a.Hq + h) * a.n_split + split) * (D + 2);
    out[2 + dc] = o;
    if (dc == 0) { out[0] = mx; out[1] = ll; }
  }
}

// One warp per (b, h): merge the n_split partial states, write bf16 o and fp32 lse.
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= a.B * a.Hq) return;
  const float* P = a.partials + (size_t)wid * a.n_split * (D + 2);
  float mx = -INFINITY;
  for (int i = lane; i < a.n_split; i += 32) mx = fmaxf(mx, P[(size_t)i * (D + 2)]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  constexpr int E = D / 32;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float l = 0.f;
  for (int i = 0; i < a.n_split; ++i) {
    const float* pi = P + (size_t)i * (D + 2);
    const float mi = pi[0];
    if (mi == -INFINITY) continue;
    const float f = ptx::ex2(mi - mx);
    l += f * pi[1];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] += f * pi[2 + lane + 32 * e];
  }
  const float inv = 1.f / l;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.o) + (size_t)wid * D;
#pragma unroll
  for (int e = 0; e < E; ++e) o[lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
  if (a.lse && lane == 0) a.lse[wid] = (mx + log2f(l)) * 0.69314718055994530942f;
}

template <int GRP, int D>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t s) {
  using Geo = DecGeom<D>;
  auto kern = decode_split_kernel<GRP, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_split, a.Hkv, a.B);
  kern<<<grid, kDecThreads, Geo::kSmemBytes, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int warps = a.B * a.Hq;
  decode_combine_kernel<D><<<(warps * 32 + 255) / 256, 256, 0, s>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t s) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_decode_t<1, D>(a, s);
    case 2: return launch_decode_t<2, D>(a, s);
    case 3: return launch_decode_t<3, D>(a, s);
    case 4: return launch_decode_t<4, D>(a, s);
    case 5: return launch_decode_t<5, D>(a, s);
    case 6: return launch_decode_t<6, D>(a, s);
    case 7: return launch_decode_t<7, D>(a, s);
    case 8: return launch_decode_t<8, D>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int decode_chunk_tokens(const Pat& p, int B, int Hkv, int T_cap) {
  (void)p; (void)B; (void)Hkv; (void)T_cap;
  return 1024;
}

int decode_num_splits(const Pat& p, int T_cap, int chunk) {
  // chunks of the three ranges, each cut from its own start: sink, widest interval, band
  const int64_t R = (int64_t)p.T - p.S;
  const int64_t wmax = R > 0 ? (R + p.H - 1) / p.H : 0;
  const int64_t sink = p.S < T_cap ? p.S : T_cap;
  const int64_t band = p.L < T_cap ? p.L : T_cap;
  const int64_t lr = wmax < T_cap ? wmax : T_cap;
  int64_t n = (sink + chunk - 1) / chunk + (lr + chunk - 1) / chunk + (band + chunk - 1) / chunk;
  return (int)(n < 1 ? 1 : n);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.d == 64) return launch_decode_d<64>(a, s);
  if (a.d == 128) return launch_decode_d<128>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace cowa
