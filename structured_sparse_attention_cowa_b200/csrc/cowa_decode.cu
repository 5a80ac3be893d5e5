// cowa_decode.cu -- split-KV CoWA decode: one new query token per sequence attends to the
// keys its KV head can see in the cache ("CoWindow Attention: Full Causal Coverage Is a
// Collective Property", Abstract: decoding with the same position-defined pattern as
// training; skillfed.io news summary, paragraph 4).
//
// HBM-bound: per (b, g) only the <= 3 visible token ranges at pos[b] (sink, interval_g,
// near-diagonal band) are read.  Each CTA owns one chunk of one range:
//   * a producer warp streams 64-token K and V sub-tiles into a shared-memory ring with TMA
//     (128-byte swizzle, whole 128-byte rows, nothing staged through registers);
//   * 4 compute warps each take 16 tokens of every sub-tile.  Per (b, g) decode is the
//     contraction [grp x d] . [d x n]: scores and P.V run on warp-level tensor-core MMAs
//     (m16n8k16, bf16 in, fp32 accumulate; the grp query heads are rows 0..grp-1 of the 16-row
//     A operand), with K fragments from ldmatrix and V fragments from ldmatrix.trans on the
//     swizzled tiles.  This keeps the instruction count per token small enough that the
//     kernel is limited by HBM, not by the CUDA cores;
//   * online softmax in the log2 domain with a lazy rescale of the accumulators;
//   * the warps' partial (m, l, o) states are merged in shared memory and written as one fp32
//     partial per (b, h, split).
// A second kernel merges the splits of each (b, h) (max / rescaled sums, warp shuffles)
// and writes bf16 o and the fp32 lse.
//
// The same kernel reads a compacted per-head cache (sink, band ring, own interval; see
// CompactGeom): the visible positions then form three disjoint sets, each read from its own
// region in 64-aligned blocks (64 consecutive rows), with positions outside the CTA's chunk
// masked.  Two small kernels keep that cache: one builds it from a prefill's K/V, one appends
// a decoded token to every region that holds its position.
#include <cuda_bf16.h>
#include <math.h>

#include "cowa_internal.h"
#include "sm100_ptx.cuh"

namespace cowa {
namespace {

constexpr int kDecWarps = 4;                        // compute warps per CTA
constexpr int kDecThreads = (kDecWarps + 1) * 32;   // + one TMA producer warp
constexpr int kSubTok = 64;                         // tokens per sub-tile (TMA box rows)
constexpr int kStages = 3;                          // sub-tile ring depth (bf16 cache)
constexpr int kMaxStages = 4;                       // ring depth of the E4M3 cache (half-size stages)
constexpr int kBoxBytes = kSubTok * 128;            // one [64 rows x 64 bf16] box
constexpr float kDecRescale = 8.0f;                 // lazy-rescale threshold, log2 units

// KV8: the cache holds E4M3 codes (one byte per element) instead of bf16.  Each compute thread
// loads the code bytes its MMA fragments need straight from the ring into registers and widens
// them there to f16 (E4M3 values are exact in f16); the MMAs then run in f16.  To make those
// bytes contiguous, the head dimension is visited in a permuted order (a sum over d, and a
// relabelling of the output columns, so the result is unchanged):
//   scores: k-chunk c, in-chunk index kappa of the m16n8k16 operands  <->  d = 32 t + 4 c + j,
//           t = (kappa mod 8) / 2, j = (kappa mod 2) + 2 [kappa >= 8]  (thread t reads bytes
//           [32 t, 32 t + 32) of a key row; the query fragments are gathered to match);
//   P.V:    n-tile jn, column nu  <->  d = 16 nu + jn  (thread g of an MMA group reads bytes
//           [16 g, 16 g + 16) of each of its 4 value rows), undone when the output is stored.
template <int D, bool KV8 = false>
struct DecGeom {
  static_assert(!KV8 || D == 128, "the E4M3 cache needs whole 128-byte rows (d = 128)");
  static constexpr int kUnits = KV8 ? 1 : D / 64;          // 128-byte TMA boxes per row
  static constexpr int kBoxElems = KV8 ? 128 : 64;         // elements per box row
  static constexpr int kTileBytes = kUnits * kBoxBytes;    // K (or V) sub-tile as stored
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = KV8 ? kMaxStages : ::cowa::kStages;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kSmemBytes = kRingBytes + 1024;
};

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  // the low byte becomes the low half
  uint32_t r;
  asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(r) : "r"(two_codes));
  return r;
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));  // first source -> upper half
  return r;
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void mma_16816_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// shared address of 16-byte unit u (d elements 8u..8u+7) of token row r of a swizzled tile
__device__ __forceinline__ uint32_t unit_addr(uint32_t tile, int r, int u) {
  return tile + (u >> 3) * kBoxBytes + r * 128 + (((u & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ float safe_ex2_diff(float a, float m) {
  // exp2(a - m) with a == -inf giving 0 even when m == -inf
  return a == -INFINITY ? 0.f : ptx::ex2(a - m);
}

template <int GRP, int D, bool KV8>
__device__ __forceinline__ void decode_split_body(const DecodeArgs& a) {
  static_assert(GRP >= 1 && GRP <= 8, "query heads per KV head must fit the MMA's first 8 rows");
  using Geo = DecGeom<D, KV8>;
  constexpr int KS = D / 16;  // k-steps of the score MMA
  constexpr int NT = D / 8;   // n-tiles of the P.V MMA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kStages = Geo::kStages;
  __shared__ __align__(8) uint64_t full_bar[kMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
  __shared__ int abort_flag;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which chunk of which visible range this CTA owns (pure position arithmetic)
  int t = a.pos[b];
  t = t < 0 ? 0 : (a.compact || t < a.T_cap ? t : a.T_cap - 1);
  const Range iv = interval_of(a.pat, g);
  Range rr[3];
  int region[3] = {0, 0, 0};
  int nr;
  if (!a.compact) {
    nr = row_ranges(a.pat, iv, t, rr);  // merged ranges of positions = cache rows
  } else {
    // three disjoint sets, each read from its own region: sink, the interval keys before the
    // band, the band without the sink
    const int sink_hi = imin(a.pat.S, t + 1);
    const int band_lo = imax(0, t - a.pat.L + 1);
    rr[0] = Range{0, sink_hi};
    rr[1] = Range{iv.lo, imin(imin(iv.hi, t + 1), band_lo)};
    rr[2] = Range{imax(band_lo, sink_hi), t + 1};
    region[0] = 0; region[1] = 1; region[2] = 2;
    nr = 3;
  }
  // chunks of each range: cut from its start on the full cache; on the compacted cache cut at
  // 64-aligned positions (chunk is a multiple of 64), so only a range's first chunk begins
  // inside a 64-row block
  int c_lo = 0, c_hi = 0, c_reg = 0;
  {
    int idx = split;
    for (int r = 0; r < nr; ++r) {
      if (rr[r].hi <= rr[r].lo) continue;
      const int base = a.compact ? (rr[r].lo & ~(kSubTok - 1)) : rr[r].lo;
      const int nch = (rr[r].hi - base + a.chunk - 1) / a.chunk;
      if (idx < nch) {
        c_lo = imax(rr[r].lo, base + idx * a.chunk);
        c_hi = imin(rr[r].hi, base + (idx + 1) * a.chunk);
        c_reg = region[r];
        break;
      }
      idx -= nch;
    }
  }
  // sub-tiles start at c_lo (full cache) or at the 64-aligned position below it (compacted
  // cache: an aligned block is 64 consecutive rows of one region); tokens outside
  // [c_lo, c_hi) are masked
  const int p_base = a.compact ? (c_lo & ~(kSubTok - 1)) : c_lo;
  const int nsub = c_hi > c_lo ? (c_hi - p_base + kSubTok - 1) / kSubTok : 0;
  const int lo64 = iv.lo & ~(kSubTok - 1);
  auto cache_row = [&](int pp) -> int {  // cache row of the sub-tile at position pp
    if (!a.compact) return pp;
    if (c_reg == 0) return pp;
    if (c_reg == 1) return a.cg.IB + (pp - lo64);
    return a.cg.S64 + (pp % a.cg.R);
  };

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
        const int row = cache_row(p_base + st * kSubTok);
        // (debug builds) the sub-tile starts inside the cache (a compacted block ends inside it too)
        if (!ptx::dbg_check(row >= 0 && (a.compact ? row + kSubTok <= a.cg.rows : row < a.T_cap) && b < a.B,
                            a.status, &abort_flag, 0x401, row))
          break;
        ptx::mbar_arrive_expect_tx(&full_bar[s], Geo::kStageBytes);
#pragma unroll
        for (int u = 0; u < Geo::kUnits; ++u) {
          ptx::tma_load_4d(ks + u * kBoxBytes, &a.tm_k, &full_bar[s], u * Geo::kBoxElems, row, g, b);
          ptx::tma_load_4d(vs + u * kBoxBytes, &a.tm_v, &full_bar[s], u * Geo::kBoxElems, row, g, b);
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
  const int gr = lane >> 2;  // fragment row = query head of the group (rows >= GRP are zero)
  const int tq = lane & 3;   // fragment column pair
  // A fragments of Q (rows 8..15 of the 16-row operand are zero: a1 = a3 = 0)
  uint32_t qa[KS][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const __nv_bfloat16*>(a.q_t) + ((size_t)b * a.Hq + (size_t)g * GRP + imin(gr, GRP - 1)) * D);
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      if constexpr (KV8) {
        // permuted k order (see DecGeom): chunk kk of thread tq is d = 32 tq + 4 kk .. + 3; f16
        // operands (bf16 values of the usual range are exact in f16)
        qa[kk][0] = gr < GRP ? bf16x2_to_f16x2(qrow[16 * tq + 2 * kk]) : 0u;
        qa[kk][1] = gr < GRP ? bf16x2_to_f16x2(qrow[16 * tq + 2 * kk + 1]) : 0u;
      } else {
        qa[kk][0] = gr < GRP ? qrow[8 * kk + tq] : 0u;
        qa[kk][1] = gr < GRP ? qrow[8 * kk + 4 + tq] : 0u;
      }
    }
  }
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_used = -INFINITY, lsum = 0.f;

  const uint32_t smem_base = ptx::smem_u32(smem);
  const int row0 = warp * 16;  // this warp's tokens within each sub-tile
  bool ok = true;
  for (int st = 0; st < nsub; ++st) {
    const int s = st % kStages;
    if (!ptx::mbar_wait_warp(&full_bar[s], (st / kStages) & 1, &abort_flag, a.status)) { ok = false; break; }
    const uint32_t kt = smem_base + s * Geo::kStageBytes;
    const uint32_t vt = kt + Geo::kTileBytes;
    // ---- scores S[head][token] for two 8-token n-tiles
    float sc[2][4];
    uint4 vr[4];  // E4M3 only: bytes [16 gr, 16 gr + 16) of value rows 2tq, 2tq+1, 2tq+8, 2tq+9
    if constexpr (KV8) {
      // key codes straight into registers: thread tq takes bytes [32 tq, 32 tq + 32) of key row
      // 8 nt + gr (two 16-byte units of the swizzled row), which are its B fragments of all 8
      // k-chunks in the permuted order; value codes likewise (see DecGeom)
      uint32_t kw[2][8];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int r = row0 + 8 * nt + gr;
        const uint32_t rb = kt + r * 128;
        const uint4 x0 = lds128(rb + (((2 * tq) ^ (r & 7)) << 4));
        const uint4 x1 = lds128(rb + (((2 * tq + 1) ^ (r & 7)) << 4));
        kw[nt][0] = x0.x; kw[nt][1] = x0.y; kw[nt][2] = x0.z; kw[nt][3] = x0.w;
        kw[nt][4] = x1.x; kw[nt][5] = x1.y; kw[nt][6] = x1.z; kw[nt][7] = x1.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = row0 + 2 * tq + (i & 1) + 8 * (i >> 1);
        vr[i] = lds128(vt + r * 128 + ((gr ^ (r & 7)) << 4));
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty_bar[s]);  // the stage's bytes are in registers
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          const uint32_t aa[4] = {qa[kk][0], 0u, qa[kk][1], 0u};
          mma_16816_f16(sc[nt], aa, e4m3x2_to_f16x2(kw[nt][kk] & 0xffffu), e4m3x2_to_f16x2(kw[nt][kk] >> 16));
        }
      }
    } else {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < KS / 2; ++k2) {
          uint32_t bb[4];
          const uint32_t a0[4] = {qa[2 * k2][0], 0u, qa[2 * k2][1], 0u};
          const uint32_t a1[4] = {qa[2 * k2 + 1][0], 0u, qa[2 * k2 + 1][1], 0u};
          ptx::ldsm_x4(unit_addr(kt, row0 + 8 * nt + (lane & 7), 4 * k2 + (lane >> 3)), bb);
          ptx::mma_16816(sc[nt], a0, bb[0], bb[1]);
          ptx::mma_16816(sc[nt], a1, bb[2], bb[3]);
        }
      }
    }
    // ---- online softmax (log2 domain) over this warp's 16 tokens
    const int tok0 = p_base + st * kSubTok + row0 + 2 * tq;
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = tok0 + 8 * (e >> 1) + (e & 1);
      x[e] = (tok >= c_lo && tok < c_hi) ? sc[e >> 1][e & 1] * a.scale_log2 : -INFINITY;
    }
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_used, mx);
    if (m_new != -INFINITY && (m_used == -INFINITY || m_new > m_used + kDecRescale)) {
      const float alpha = ptx::ex2(m_used - m_new);  // 0 when nothing was visible before
      lsum *= alpha;
#pragma unroll
      for (int n = 0; n < NT; ++n) { acc[n][0] *= alpha; acc[n][1] *= alpha; }
      m_used = m_new;
    }
    const float m_eff = m_used == -INFINITY ? 0.f : m_used;
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = ptx::ex2(x[e] - m_eff);
      lsum += p[e];
    }
    // P as the A operand: tokens 2tq, 2tq+1 (first n-tile) and 8+2tq, 9+2tq (second)
    uint32_t pa[4];
    if constexpr (KV8) {
      pa[0] = pack_f16(p[0], p[1]); pa[2] = pack_f16(p[2], p[3]);
    } else {
      pa[0] = ptx::pack_bf16(p[0], p[1]); pa[2] = ptx::pack_bf16(p[2], p[3]);
    }
    pa[1] = pa[3] = 0u;
    // ---- O[head][d] += P[head][token] V[token][d]
    if constexpr (KV8) {
      // n-tile jn, column gr is d = 16 gr + jn: byte jn of this thread's value bytes.  Bytes of
      // rows (2tq, 2tq+1) and (2tq+8, 2tq+9) are interleaved into E4M3 pairs, then widened.
      const uint32_t A[4] = {vr[0].x, vr[0].y, vr[0].z, vr[0].w}, B[4] = {vr[1].x, vr[1].y, vr[1].z, vr[1].w};
      const uint32_t C[4] = {vr[2].x, vr[2].y, vr[2].z, vr[2].w}, E[4] = {vr[3].x, vr[3].y, vr[3].z, vr[3].w};
#pragma unroll
      for (int jw = 0; jw < 4; ++jw) {
        const uint32_t ab[2] = {prmt(A[jw], B[jw], 0x5140u), prmt(A[jw], B[jw], 0x7362u)};
        const uint32_t ce[2] = {prmt(C[jw], E[jw], 0x5140u), prmt(C[jw], E[jw], 0x7362u)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int sh = (e & 1) * 16;
          mma_16816_f16(acc[4 * jw + e], pa, e4m3x2_to_f16x2((ab[e >> 1] >> sh) & 0xffffu),
                        e4m3x2_to_f16x2((ce[e >> 1] >> sh) & 0xffffu));
        }
      }
    } else {
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t bb[4];
        ptx::ldsm_x4_trans(unit_addr(vt, row0 + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * np + (lane >> 4)), bb);
        ptx::mma_16816(acc[2 * np], pa, bb[0], bb[1]);
        ptx::mma_16816(acc[2 * np + 1], pa, bb[2], bb[3]);
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty_bar[s]);
    }
  }
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);

  // ---- merge the warps through shared memory (the ring is drained: reuse it)
  asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
  if (!ok || abort_flag) return;
  float* red = reinterpret_cast<float*>(smem);  // [warp][8 rows][D + 2]
  {
    float* rw = red + (warp * 8 + gr) * (D + 2);
    if (tq == 0) { rw[0] = m_used; rw[1] = lsum; }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      if constexpr (KV8) {  // columns 2tq, 2tq+1 of n-tile n are d = 32 tq + n and 32 tq + 16 + n
        rw[2 + 32 * tq + n] = acc[n][0];
        rw[2 + 32 * tq + 16 + n] = acc[n][1];
      } else {
        rw[2 + 8 * n + 2 * tq] = acc[n][0];
        rw[2 + 8 * n + 2 * tq + 1] = acc[n][1];
      }
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
  for (int xi = threadIdx.x; xi < GRP * D; xi += kDecWarps * 32) {
    const int hh = xi / D, dc = xi % D;
    float mxw = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) mxw = fmaxf(mxw, red[(w * 8 + hh) * (D + 2)]);
    float o = 0.f, ll = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float* rw = red + (w * 8 + hh) * (D + 2);
      const float f = safe_ex2_diff(rw[0], mxw);
      o += f * rw[2 + dc];
      ll += f * rw[1];
    }
    const int h = g * GRP + hh;
    float* out = a.partials + (((size_t)b * a.Hq + h) * a.n_split + split) * (D + 2);
    out[2 + dc] = KV8 ? o * a.v_scale : o;
    if (dc == 0) { out[0] = mxw; out[1] = ll; }
  }
}

// bf16 cache
template <int GRP, int D>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const __grid_constant__ DecodeArgs a) {
  decode_split_body<GRP, D, false>(a);
}
// E4M3 cache: three CTAs per SM (a 4-stage ring each; measured 5% faster than two CTAs with a
// 6-stage ring at the 128K decode configuration)
template <int GRP>
__global__ void __launch_bounds__(kDecThreads, 3) decode_split_e4m3_kernel(const __grid_constant__ DecodeArgs a) {
  decode_split_body<GRP, 128, true>(a);
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

// ------------------------------------------------------------------ compacted cache upkeep
// Appends the token at pos[b] (k_new / v_new [B, H_kv, D] contiguous) to every region that holds
// it.  One block per (KV head, b); 16-byte copies.
template <int D>
__global__ void __launch_bounds__(D / 8) compact_append_kernel(Pat pat, CompactGeom cg, const uint4* k_new,
                                                                 const uint4* v_new, const int32_t* pos, uint4* kc,
                                                                 uint4* vc, int Hkv) {
  const int g = blockIdx.x, b = blockIdx.y, u = threadIdx.x;
  const int p = pos[b];
  if (p < 0) return;
  const Range iv = interval_of(pat, g);
  const size_t src = ((size_t)b * Hkv + g) * (D / 8) + u;
  const uint4 kk = k_new[src], vv = v_new[src];
  const size_t head = ((size_t)b * Hkv + g) * (size_t)cg.rows;
  auto put = [&](int row) {
    kc[(head + row) * (D / 8) + u] = kk;
    vc[(head + row) * (D / 8) + u] = vv;
  };
  put(cg.S64 + p % cg.R);
  if (p < pat.S) put(p);
  if (p >= iv.lo && p < iv.hi) put(cg.IB + p - (iv.lo & ~(kSubTok - 1)));
}

// Builds the compacted cache from the keys and values of positions 0..N-1 (strided
// [B, N, H_kv, D]): block (x, g, b) handles positions [64x, 64x + 64).
template <int D>
__global__ void __launch_bounds__(128) compact_build_kernel(Pat pat, CompactGeom cg, const __nv_bfloat16* k,
                                                             const __nv_bfloat16* v, int64_t sb, int64_t st,
                                                             int64_t sh, int64_t vsb, int64_t vst, int64_t vsh,
                                                             int N, uint4* kc, uint4* vc, int Hkv) {
  const int g = blockIdx.y, b = blockIdx.z;
  const Range iv = interval_of(pat, g);
  const int lo64 = iv.lo & ~(kSubTok - 1);
  const size_t head = ((size_t)b * Hkv + g) * (size_t)cg.rows;
  constexpr int U = D / 8;
  for (int x = threadIdx.x; x < kSubTok * U; x += blockDim.x) {
    const int p = blockIdx.x * kSubTok + x / U, u = x % U;
    if (p >= N) continue;
    const bool in_ring = p >= N - cg.R, in_sink = p < pat.S, in_iv = p >= iv.lo && p < iv.hi;
    if (!in_ring && !in_sink && !in_iv) continue;
    const uint4 kk = reinterpret_cast<const uint4*>(k + b * sb + (int64_t)p * st + g * sh)[u];
    const uint4 vv = reinterpret_cast<const uint4*>(v + b * vsb + (int64_t)p * vst + g * vsh)[u];
    auto put = [&](int row) {
      kc[(head + row) * U + u] = kk;
      vc[(head + row) * U + u] = vv;
    };
    if (in_ring) put(cg.S64 + p % cg.R);
    if (in_sink) put(p);
    if (in_iv) put(cg.IB + p - lo64);
  }
}

template <int GRP, int D, bool KV8>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t s) {
  using Geo = DecGeom<D, KV8>;
  void (*kern)(const DecodeArgs);
  if constexpr (KV8) kern = decode_split_e4m3_kernel<GRP>;
  else kern = decode_split_kernel<GRP, D>;
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

template <int D, bool KV8 = false>
cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t s) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_decode_t<1, D, KV8>(a, s);
    case 2: return launch_decode_t<2, D, KV8>(a, s);
    case 3: return launch_decode_t<3, D, KV8>(a, s);
    case 4: return launch_decode_t<4, D, KV8>(a, s);
    case 5: return launch_decode_t<5, D, KV8>(a, s);
    case 6: return launch_decode_t<6, D, KV8>(a, s);
    case 7: return launch_decode_t<7, D, KV8>(a, s);
    case 8: return launch_decode_t<8, D, KV8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int decode_chunk_tokens(const Pat& p, int B, int Hkv, int T_cap) {
  (void)p; (void)B; (void)Hkv; (void)T_cap;
  return 1024;
}

int decode_num_splits(const Pat& p, int T_cap, int chunk, bool compact) {
  // chunks of the three ranges, each cut from its own start (compacted cache: from the
  // 64-aligned position below it, up to 63 more positions per range): sink, widest interval, band
  const int64_t R = (int64_t)p.T - p.S;
  const int64_t wmax = R > 0 ? (R + p.H - 1) / p.H : 0;
  const int64_t sink = p.S < T_cap ? p.S : T_cap;
  const int64_t band = p.L < T_cap ? p.L : T_cap;
  const int64_t lr = wmax < T_cap ? wmax : T_cap;
  const int64_t a = compact ? kSubTok - 1 : 0;
  int64_t n = (sink + a + chunk - 1) / chunk + (lr + a + chunk - 1) / chunk + (band + a + chunk - 1) / chunk;
  return (int)(n < 1 ? 1 : n);
}

// Sizes in 64-bit; a layout whose rows would not fit an int (a band of ~2^31 positions) is
// reported as rows = 0, which the entry points reject.
CompactGeom compact_geom(const Pat& p) {
  CompactGeom c{};
  const int64_t t = kSubTok;
  const int64_t s64 = ((int64_t)p.S + t - 1) / t * t;
  const int64_t r = ((int64_t)p.L + t - 1) / t * t + t;
  int64_t w = 0;
  for (int slot = 0; slot < p.H; slot += p.H / p.D) {  // the distinct interval slots
    const int lo = bound(p, slot), hi = bound(p, slot + 1);
    if (hi > lo) w = w > (int64_t)hi - (lo & ~(kSubTok - 1)) ? w : (int64_t)hi - (lo & ~(kSubTok - 1));
  }
  w = (w + t - 1) / t * t;
  if (s64 + r + w > 0x7fffffffLL) return c;
  c.S64 = (int)s64;
  c.R = (int)r;
  c.IB = (int)(s64 + r);
  c.W = (int)w;
  c.rows = (int)(s64 + r + w);
  return c;
}

cudaError_t launch_compact_append(const Pat& p, int B, int Hkv, int d, const void* k_new, const void* v_new,
                                  const int32_t* pos, void* kc, void* vc, cudaStream_t s) {
  const CompactGeom cg = compact_geom(p);
  dim3 grid(Hkv, B);
  if (d == 128)
    compact_append_kernel<128><<<grid, 16, 0, s>>>(p, cg, static_cast<const uint4*>(k_new),
                                                   static_cast<const uint4*>(v_new), pos, static_cast<uint4*>(kc),
                                                   static_cast<uint4*>(vc), Hkv);
  else if (d == 64)
    compact_append_kernel<64><<<grid, 8, 0, s>>>(p, cg, static_cast<const uint4*>(k_new),
                                                 static_cast<const uint4*>(v_new), pos, static_cast<uint4*>(kc),
                                                 static_cast<uint4*>(vc), Hkv);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_compact_build(const Pat& p, int B, int N, int Hkv, int d, const void* k, int64_t ksb, int64_t kst,
                                 int64_t ksh, const void* v, int64_t vsb, int64_t vst, int64_t vsh, void* kc, void* vc,
                                 cudaStream_t s) {
  const CompactGeom cg = compact_geom(p);
  dim3 grid((N + kSubTok - 1) / kSubTok, Hkv, B);
  auto kb = static_cast<const __nv_bfloat16*>(k);
  auto vb = static_cast<const __nv_bfloat16*>(v);
  if (d == 128)
    compact_build_kernel<128><<<grid, 128, 0, s>>>(p, cg, kb, vb, ksb, kst, ksh, vsb, vst, vsh, N,
                                                   static_cast<uint4*>(kc), static_cast<uint4*>(vc), Hkv);
  else if (d == 64)
    compact_build_kernel<64><<<grid, 128, 0, s>>>(p, cg, kb, vb, ksb, kst, ksh, vsb, vst, vsh, N,
                                                  static_cast<uint4*>(kc), static_cast<uint4*>(vc), Hkv);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.kv8) return a.d == 128 ? launch_decode_d<128, true>(a, s) : cudaErrorInvalidValue;
  if (a.d == 64) return launch_decode_d<64>(a, s);
  if (a.d == 128) return launch_decode_d<128>(a, s);
  return cudaErrorInvalidValue;
}

// E4M3 codes of x * inv_scale (bf16 in, round to nearest even, saturating at +-448); n elements,
// n even.  One thread per 8 elements.
__global__ void quantize_e4m3_kernel(const uint4* __restrict__ x, uint2* __restrict__ q, int64_t n8, float inv_scale) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const uint4 v = x[i];
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t lo16, hi16;
    {
      const float f0 = __uint_as_float(w[2 * j] << 16) * inv_scale;
      const float f1 = __uint_as_float(w[2 * j] & 0xffff0000u) * inv_scale;
      uint16_t c;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(f1), "f"(f0));  // first source -> upper byte
      lo16 = c;
    }
    {
      const float f0 = __uint_as_float(w[2 * j + 1] << 16) * inv_scale;
      const float f1 = __uint_as_float(w[2 * j + 1] & 0xffff0000u) * inv_scale;
      uint16_t c;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(f1), "f"(f0));
      hi16 = c;
    }
    out[j] = lo16 | (hi16 << 16);
  }
  q[i] = make_uint2(out[0], out[1]);
}

cudaError_t launch_quantize_e4m3(const void* x, void* q, int64_t n, float inv_scale, cudaStream_t s) {
  const int64_t n8 = n / 8;
  if (n8 > 0)
    quantize_e4m3_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(static_cast<const uint4*>(x),
                                                                     static_cast<uint2*>(q), n8, inv_scale);
  return cudaGetLastError();
}

}  // namespace cowa
