// cowa_bwd.cu -- CoWA backward on sm_100a: gradients of exact softmax attention over the
// position-defined visible set ("CoWindow Attention: Full Causal Coverage Is a Collective
// Property", Abstract: forward and backward latency of the operator during training).
//
// With P = exp(scale * q.k - lse) on visible pairs (0 elsewhere), dP = dO v^T,
// Delta = rowsum(dO * O) and dS = P * (dP - Delta):
//   dV_g = sum_h P^T dO_h,   dK_g = scale * sum_h dS^T Q_h,   dQ_h = scale * dS K_g.
// Three kernels, no atomics (results are deterministic):
//   1. preprocess: -Delta and -lse*log2(e) per row into the workspace, padded to whole tiles
//      (padded rows get -lse = -inf so they contribute P = 0);
//   2. dK/dV: one CTA per (b, KV head g, 128-key tile j); K_j, V_j stay in shared memory and
//      the CTA walks the single contiguous range of query tiles that see tile j (sink and
//      interval keys are seen by every later query, band keys by the next L queries) for
//      every query head of the group, in sub-steps of 64 query rows.  S^T = K Q^T and
//      dP^T = V dO^T of a sub-step land in one of two TMEM buffers, so the MMAs of sub-step
//      m+1 run while the elementwise softmax works on sub-step m; the softmax writes P^T and
//      dS^T back into the buffer as bf16, where they are the A operand of dV += P^T dO and
//      dK += dS^T Q (tcgen05 MMA with A in TMEM).  The packed P^T / dS^T sit at columns that
//      overlap only the S^T / dP^T columns the writing warp has already read, so no warp
//      waits for another;
//   3. dQ: one CTA per (b, query head h, 128-row tile i) over the forward tile plan.  The
//      softmax warps load S and dP of a KV tile into registers and release them at once, so
//      the MMA warp computes S and dP of the next tile while dS of this one is being formed;
//      dS goes to a double-buffered bf16 region of TMEM and dQ += dS K reads it as A.
// Warp roles in both attention kernels: 4 NP elementwise softmax warps (NP per TMEM lane
// quadrant, each owning 1/NP of the columns; dQ: NP = 4 at d = 128, dK/dV: NP = 2), then the
// TMA producer and the MMA issuer.
#include <cuda_bf16.h>
#include <math.h>

#include <type_traits>

#include "cowa_internal.h"
#include "kernel_common.cuh"
#include "sm100_ptx.cuh"

namespace cowa {
namespace {

constexpr int kStatBytes = 1024;  // lse2[128] + delta[128] of one query tile

template <int D>
struct BwdGeom {
  static constexpr int kTileBytes = kTile * D * 2;  // one 128-row bf16 tile of width D
  // dK/dV kernel: K, V resident + 2 slots of {Q, dO, stats}
  static constexpr int kSlotKV = 2 * kTileBytes + kStatBytes;
  static constexpr int kSmemKV = 2 * kTileBytes + 2 * kSlotKV + 1024;
  // dQ kernel: Q, dO resident + a 3-slot K ring (a K tile lives until its dQ MMA) and a
  // 2-slot V ring (a V tile is free once its dP MMA is done)
  static constexpr int kKSlots = 3, kVSlots = 2;
  static constexpr int kSmemQ = (2 + kKSlots + kVSlots) * kTileBytes + 1024;
  static constexpr int kColAcc = 256;  // first accumulator column
};

// ------------------------------------------------------------------------------ preprocess
// One block of 256 threads per (128-row tile, head, batch).  D/8 lanes per row, 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __grid_constant__ BwdArgs a) {
  constexpr int LPR = D / 8;            // lanes per row
  constexpr int RPI = 256 / LPR;        // rows per iteration of the block
  const int tg = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  // tile tg of the statistics: tile i of batch b, or of the sequence it falls in (packed batch)
  int i = tg, row0 = 0, N = a.N;
  if (a.varlen) {
    if (tg >= a.seq_tab[a.n_seq]) return;  // past the last sequence: no statistics read there
    const int sq = seq_of_tile(a.seq_tab, a.n_seq, tg);
    i = tg - a.seq_tab[sq];
    row0 = a.seq_tab[a.n_seq + 1 + sq];
    N = a.seq_tab[2 * a.n_seq + 1 + sq];
  }
  const int sub = threadIdx.x % LPR, rr = threadIdx.x / LPR;
  const size_t base = ((size_t)b * a.Hq + h) * a.N_pad + (size_t)tg * kTile;
  const size_t lse_base = ((size_t)b * a.Hq + h) * a.lse_ld + row0;
  for (int r = rr; r < kTile; r += RPI) {
    const int t = i * kTile + r;  // row within the sequence
    float acc = 0.f;
    if (t < N) {
      const int64_t row = (int64_t)row0 + t;
      const uint4 ov = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.o) + b * a.o_sb +
                                                      row * a.o_st + h * a.o_sh + sub * 8);
      const uint4 dv = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.dO) + b * a.do_sb +
                                                      row * a.do_st + h * a.do_sh + sub * 8);
      const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(dw[e] << 16), acc);
        acc = fmaf(__uint_as_float(ow[e] & 0xffff0000u), __uint_as_float(dw[e] & 0xffff0000u), acc);
      }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0) {  // negated, so that the softmaxes add them with packed fp32x2 instructions
      a.delta[base + r] = -acc;
      a.lse2[base + r] = t < N ? -(a.lse[lse_base + t] * 1.4426950408889634f) : -INFINITY;
    }
  }
}

// ------------------------------------------------------------------------------ dK / dV
// TMEM columns: two sub-step buffers at 0 and 128, each S^T [+0, +64) and dP^T [+64, +128)
// for 64 query rows; dV [256, 256+D), dK [256+D, 256+2D).  NP softmax warps per lane quadrant
// each own CW = 64/NP query columns; a warp writes its packed bf16 P^T (dS^T) into the upper
// half of the S^T (dP^T) columns it has just read, so no warp overwrites columns another warp
// has yet to read.  K step kk (16 query rows) of the dV / dK MMAs reads A at pt_col(kk) and
// 64 + pt_col(kk).
constexpr int kSub = 64;  // query rows per sub-step
template <int NP>
__device__ __forceinline__ constexpr uint32_t pt_col(int kk) {
  constexpr int CW = kSub / NP, KPW = CW / 16;  // query columns and K steps per warp
  return (uint32_t)((kk / KPW) * CW + CW / 2 + 8 * (kk % KPW));
}
template <int D, int NP>
__global__ void __launch_bounds__((4 * NP + 2) * 32, 1) bwd_dkdv_kernel(const __grid_constant__ BwdArgs a) {
  using Geo = BwdGeom<D>;
  constexpr int kSoftWarps = 4 * NP, kKProducer = 4 * NP, kKMma = 4 * NP + 1;
  constexpr int CW = kSub / NP;  // query columns per softmax warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  __shared__ __align__(8) uint64_t kv_full, slot_full[2], slot_empty[2], sdp_full[2], p_ready[2], acc_full,
      mma_final;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = a.Hq / a.Hkv;
  // the chunks of split key tiles first (each about the mean work of an SM), then every key tile,
  // lowest first: their query ranges (sink, early intervals) are the longest
  int j, g, b, kc = -1;  // kc >= 0: chunk kc of a split key tile
  if ((int)blockIdx.x < a.n_split) {
    const int4 e = a.kv_tab[blockIdx.x];
    if (e.w < 0) return;  // an unused slot of a packed batch's table (whole CTA, before any barrier)
    j = e.x; g = e.y; b = e.z; kc = e.w;
  } else {
    const int x = (int)blockIdx.x - a.n_split;
    j = x / (a.Hkv * a.B);
    const int rem = x % (a.Hkv * a.B);
    g = rem % a.Hkv; b = rem / a.Hkv;
  }
  // the rows of this CTA's sequence: [row0, row0 + N) of the token axis; statistics tiles from tile0
  int row0 = 0, N = a.N, tile0 = 0;
  const int tg = j;  // the key tile on the packed token axis (a packed batch)
  if (a.varlen) {
    if (j >= a.seq_tab[a.n_seq]) return;  // whole CTA, before any barrier or TMEM use
    const int sq = seq_of_tile(a.seq_tab, a.n_seq, j);
    tile0 = a.seq_tab[sq];
    j -= tile0;
    row0 = a.seq_tab[a.n_seq + 1 + sq];
    N = a.seq_tab[2 * a.n_seq + 1 + sq];
  }
  const int s0 = j * kTile, s1 = imin(N, s0 + kTile);
  const Range iv = interval_of(a.pat, g);
  const Range rows = bwd_row_range(a.pat, iv, s0, s1, N);
  int i_lo = rows.lo / kTile, i_hi = (rows.hi + kTile - 1) / kTile;
  const bool split = a.kv_chunk > 0 && (a.varlen ? a.kv_flag[(size_t)g * a.kv_bound + tg] != 0
                                                 : i_hi - i_lo > a.kv_chunk);
  if (split) {
    if (kc < 0) return;  // a split tile: its chunk CTAs do the work (before any barrier or TMEM use)
    i_lo += kc * a.kv_chunk;
    i_hi = imin(i_hi, i_lo + a.kv_chunk);
  }
  const int nsteps = (i_hi - i_lo) * grp;

  uint8_t* sK = smem;
  uint8_t* sV = smem + Geo::kTileBytes;
  uint8_t* sSlot = smem + 2 * Geo::kTileBytes;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&kv_full, 1);
    for (int s = 0; s < 2; ++s) { ptx::mbar_init(&slot_full[s], 1); ptx::mbar_init(&slot_empty[s], 1); }
    for (int bb = 0; bb < 2; ++bb) {
      ptx::mbar_init(&sdp_full[bb], 1);
      ptx::mbar_init(&p_ready[bb], kSoftWarps);
    }
    ptx::mbar_init(&acc_full, 1);
    ptx::mbar_init(&mma_final, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kKMma) {
    ptx::tmem_alloc(&tmem_base_sh, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int nsub = 2 * nsteps;  // 64-row sub-steps

  if (warp == kKProducer) {
    if (lane == 0) {
      ptx::tma_prefetch_desc(&a.tm_q);
      ptx::tma_prefetch_desc(&a.tm_do);
      // (debug builds) the key tile lies inside the sequence, the head and batch inside the call
      const bool kv_ok = ptx::dbg_check(s0 >= 0 && s0 < N && g < a.Hkv && b < a.B, a.status, &abort_flag, 0x201, s0);
      if (kv_ok) {
        ptx::mbar_arrive_expect_tx(&kv_full, 2 * Geo::kTileBytes);
        for (int u = 0; u < D / 64; ++u) {
          ptx::tma_load_4d(sK + u * 16384, &a.tm_k, &kv_full, u * 64, row0 + s0, g, b);
          ptx::tma_load_4d(sV + u * 16384, &a.tm_v, &kv_full, u * 64, row0 + s0, g, b);
        }
      }
      int issued = 0;
      for (int n = 0; kv_ok && n < nsteps; ++n) {
        const int slot = n & 1;
        if (n >= 2 && !ptx::mbar_wait(&slot_empty[slot], ((n >> 1) - 1) & 1, &abort_flag, a.status)) break;
        const int i = i_lo + n / grp, h = g * grp + n % grp;
        // (debug builds) the planned query tile lies inside the sequence and its statistics
        if (!ptx::dbg_check(i >= 0 && i * kTile < N && h < a.Hq && (tile0 + i + 1) * kTile <= a.N_pad, a.status,
                            &abort_flag, 0x202, i))
          break;
        uint8_t* dst = sSlot + slot * Geo::kSlotKV;
        ptx::mbar_arrive_expect_tx(&slot_full[slot], Geo::kSlotKV);
        for (int u = 0; u < D / 64; ++u) {
          ptx::tma_load_4d(dst + u * 16384, &a.tm_q, &slot_full[slot], u * 64, row0 + i * kTile, h, b);
          ptx::tma_load_4d(dst + Geo::kTileBytes + u * 16384, &a.tm_do, &slot_full[slot], u * 64, row0 + i * kTile,
                           h, b);
        }
        const size_t so = ((size_t)b * a.Hq + h) * a.N_pad + (size_t)(tile0 + i) * kTile;
        ptx::bulk_load(dst + 2 * Geo::kTileBytes, a.lse2 + so, 512, &slot_full[slot]);
        ptx::bulk_load(dst + 2 * Geo::kTileBytes + 512, a.delta + so, 512, &slot_full[slot]);
        issued = n + 1;
      }
      if (kv_ok) ptx::mbar_wait(&kv_full, 0, nullptr, a.status);
      for (int n = (issued > 2 ? issued - 2 : 0); n < issued; ++n)
        ptx::mbar_wait(&slot_full[n & 1], (n >> 1) & 1, nullptr, a.status);
    }
  } else if (warp == kKMma) {
    // whole warp on the issue path, one elected lane issues (uniform descriptors)
    constexpr uint32_t idesc_s = ptx::idesc_bf16(128, kSub, false, false);
    constexpr uint32_t idesc_o = ptx::idesc_bf16(128, D, false, true);
    const uint64_t k_desc = ptx::smem_desc_sw128(ptx::smem_u32(sK), 16, 1024);
    const uint64_t v_desc = ptx::smem_desc_sw128(ptx::smem_u32(sV), 16, 1024);
    const uint64_t slot_desc_k = ptx::smem_desc_sw128(ptx::smem_u32(sSlot), 16, 1024);     // K-major reads
    const uint64_t slot_desc_mn = ptx::smem_desc_sw128(ptx::smem_u32(sSlot), 16384, 1024);  // MN-major reads
    // S^T, dP^T of sub-step m (query rows 64*(m&1).. of step m>>1) into buffer m & 1.  The
    // buffer's previous P^T / dS^T were read by dV / dK of sub-step m-2, issued earlier.
    auto issue_sdp = [&](int m) -> bool {
      const int n = m >> 1, hq = m & 1;
      if (hq == 0 && !ptx::mbar_wait_warp(&slot_full[n & 1], (n >> 1) & 1, &abort_flag, a.status)) return false;
      ptx::tc_fence_after();
      const uint32_t q_off = (n & 1) * Geo::kSlotKV + hq * (kSub * 128), do_off = q_off + Geo::kTileBytes;
      const uint32_t buf = tmem + 128 * (m & 1);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        ptx::mma_bf16_ss_warp(buf, ptx::desc_advance(k_desc, off), ptx::desc_advance(slot_desc_k, q_off + off),
                              idesc_s, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        ptx::mma_bf16_ss_warp(buf + 64, ptx::desc_advance(v_desc, off), ptx::desc_advance(slot_desc_k, do_off + off),
                              idesc_s, kk > 0);
      }
      ptx::mma_commit_warp(&sdp_full[m & 1]);
      return true;
    };
    bool ok = ptx::mbar_wait_warp(&kv_full, 0, &abort_flag, a.status);
    ptx::tc_fence_after();
    if (ok && nsub > 0) ok = issue_sdp(0);
    for (int m = 0; ok && m < nsub; ++m) {
      if (m + 1 < nsub && !(ok = issue_sdp(m + 1))) break;
      if (!(ok = ptx::mbar_wait_warp(&p_ready[m & 1], (m >> 1) & 1, &abort_flag, a.status))) break;
      ptx::tc_fence_after();
      const int n = m >> 1, hq = m & 1;
      const uint32_t q_off = (n & 1) * Geo::kSlotKV + hq * (kSub * 128), do_off = q_off + Geo::kTileBytes;
      const uint32_t buf = tmem + 128 * (m & 1);
      // dV += P^T dO  and  dK += dS^T Q : A (P^T, dS^T) in TMEM, B (dO, Q) MN-major in smem
#pragma unroll
      for (int kk = 0; kk < kSub / 16; ++kk)
        ptx::mma_bf16_ts_warp(tmem + Geo::kColAcc, buf + pt_col<NP>(kk),
                              ptx::desc_advance(slot_desc_mn, do_off + kk * 2048), idesc_o, (m > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < kSub / 16; ++kk)
        ptx::mma_bf16_ts_warp(tmem + Geo::kColAcc + D, buf + 64 + pt_col<NP>(kk),
                              ptx::desc_advance(slot_desc_mn, q_off + kk * 2048), idesc_o, (m > 0 || kk > 0) ? 1u : 0u);
      if (hq == 1) ptx::mma_commit_warp(&slot_empty[n & 1]);
    }
    if (ok) ptx::mma_commit_warp(&acc_full);
    ptx::mma_commit_warp(&mma_final);
    ptx::mbar_wait(&mma_final, 0, nullptr, a.status);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise softmax (4 NP warps)
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;  // key row of the tile = TMEM lane
    const int s = s0 + r;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const bool special = s < a.pat.S || (s >= iv.lo && s < iv.hi);
    // rows [s, t_hi) see key s (min(N, s + L), without overflow for a window up to INT_MAX)
    const int t_hi = special ? N : (a.pat.L >= N - s ? N : s + a.pat.L);
    const float sl2 = a.scale_log2;
    bool ok = true;
    // query tile of the current step and its two sub-steps' mask flags, advanced incrementally
    // (every grp steps) instead of dividing and re-testing the tile on every sub-step
    int i_cur = i_lo, h_cnt = 0;
    // (two scalars, not an array indexed by the sub-step: that would live in local memory)
    bool nm0, nm1;
    auto masks_of = [&](int i) {
      const int u0 = i * kTile;
      nm0 = !tile_full(a.pat, iv, u0, imin(N, u0 + kSub), s0, s1);
      nm1 = !tile_full(a.pat, iv, u0 + kSub, imin(N, u0 + 2 * kSub), s0, s1);
    };
    masks_of(i_cur);
    for (int m = 0; m < nsub; ++m) {
      const int n = m >> 1, hq = m & 1;
      if (hq == 0 && m > 0 && ++h_cnt == grp) {
        h_cnt = 0;
        masks_of(++i_cur);
      }
      const int t0 = i_cur * kTile + hq * kSub;  // first query row of the sub-step
      const bool need_mask = hq ? nm1 : nm0;
      if (!(ok = ptx::mbar_wait_warp(&sdp_full[m & 1], (m >> 1) & 1, &abort_flag, a.status))) break;
      ptx::tc_fence_after();
      const uint32_t buf = lane_base + 128 * (m & 1);
      // this warp's CW query columns of the sub-step
      uint32_t sv[CW], pv[CW];
      if constexpr (CW == 32) {
        ptx::tmem_ld32(buf + CW * part, sv);
        ptx::tmem_ld32(buf + 64 + CW * part, pv);
      } else {
        ptx::tmem_ld16(buf + CW * part, sv);
        ptx::tmem_ld16(buf + 64 + CW * part, pv);
      }
      ptx::tmem_wait_ld();
      const float* stat = reinterpret_cast<const float*>(sSlot + (n & 1) * Geo::kSlotKV + 2 * Geo::kTileBytes) +
                          hq * kSub + CW * part;
      // the element loop is instantiated with and without the mask, chosen once per sub-step
      auto body = [&](auto masked) {
        constexpr bool kMask = decltype(masked)::value;
        // the statistics are stored negated: x = s * scale * log2(e) + (-lse2), dS = P (dP + (-Delta))
        // (scalar fp32 here: packed fp32x2 measured 1.5% slower in this kernel, 7% faster in dQ)
        const float4* lse4 = reinterpret_cast<const float4*>(stat);
        const float4* del4 = reinterpret_cast<const float4*>(stat + 128);
        uint32_t pw[CW / 2], dw[CW / 2];
#pragma unroll
        for (int c4 = 0; c4 < CW / 4; ++c4) {
          const float4 ls = lse4[c4], dl = del4[c4];
          const float lsv[4] = {ls.x, ls.y, ls.z, ls.w}, dlv[4] = {dl.x, dl.y, dl.z, dl.w};
          float pf[4], df[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int cl = c4 * 4 + e;
            float p = ptx::ex2(fmaf(__uint_as_float(sv[cl]), sl2, lsv[e]));
            if (kMask) {
              const int t = t0 + CW * part + cl;
              if (!(t >= s && t < t_hi)) p = 0.f;
            }
            pf[e] = p;
            df[e] = p * (__uint_as_float(pv[cl]) + dlv[e]);
          }
          pw[2 * c4] = ptx::pack_bf16(pf[0], pf[1]);
          pw[2 * c4 + 1] = ptx::pack_bf16(pf[2], pf[3]);
          dw[2 * c4] = ptx::pack_bf16(df[0], df[1]);
          dw[2 * c4 + 1] = ptx::pack_bf16(df[2], df[3]);
        }
        // packed columns of this warp's query columns: the upper half of the columns it just read
        if constexpr (CW == 32) {
          ptx::tmem_st16(buf + CW * part + CW / 2, pw);
          ptx::tmem_st16(buf + 64 + CW * part + CW / 2, dw);
        } else {
          ptx::tmem_st8(buf + CW * part + CW / 2, pw);
          ptx::tmem_st8(buf + 64 + CW * part + CW / 2, dw);
        }
      };
      if (need_mask) body(std::true_type{});
      else body(std::false_type{});
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&p_ready[m & 1]);
    }
    if (ok && nsteps > 0 && ptx::mbar_wait_warp(&acc_full, 0, &abort_flag, a.status)) {
      ptx::tc_fence_after();
      constexpr int HC = D / NP;  // accumulator columns of this warp
      static_assert(HC % 32 == 0, "dV / dK columns per softmax warp must be whole 32-column loads");
      uint32_t dvv[HC], dkv[HC];
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) {
        ptx::tmem_ld32(lane_base + Geo::kColAcc + part * HC + c * 32, dvv + c * 32);
        ptx::tmem_ld32(lane_base + Geo::kColAcc + D + part * HC + c * 32, dkv + c * 32);
      }
      ptx::tmem_wait_ld();
      if (kc >= 0) {
        // a chunk of a split tile: fp32 partials [dV | dK][128 key rows][D], dK not yet scaled
        float* pv = a.kv_part + (size_t)blockIdx.x * 2 * kTile * D + (size_t)r * D + part * HC;
        float* pk = pv + (size_t)kTile * D;
#pragma unroll
        for (int c4 = 0; c4 < HC / 4; ++c4) {
          reinterpret_cast<float4*>(pv)[c4] =
              make_float4(__uint_as_float(dvv[4 * c4]), __uint_as_float(dvv[4 * c4 + 1]),
                          __uint_as_float(dvv[4 * c4 + 2]), __uint_as_float(dvv[4 * c4 + 3]));
          reinterpret_cast<float4*>(pk)[c4] =
              make_float4(__uint_as_float(dkv[4 * c4]), __uint_as_float(dkv[4 * c4 + 1]),
                          __uint_as_float(dkv[4 * c4 + 2]), __uint_as_float(dkv[4 * c4 + 3]));
        }
      } else if (s < N) {
        __nv_bfloat16* dvr = reinterpret_cast<__nv_bfloat16*>(a.dv) + b * a.dv_sb + ((int64_t)row0 + s) * a.dv_st +
                             g * a.dv_sh + part * HC;
        __nv_bfloat16* dkr = reinterpret_cast<__nv_bfloat16*>(a.dk) + b * a.dk_sb + ((int64_t)row0 + s) * a.dk_st +
                             g * a.dk_sh + part * HC;
#pragma unroll
        for (int c8 = 0; c8 < HC / 8; ++c8) {
          uint32_t w[4], x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            w[e] = ptx::pack_bf16(__uint_as_float(dvv[c8 * 8 + 2 * e]), __uint_as_float(dvv[c8 * 8 + 2 * e + 1]));
            x[e] = ptx::pack_bf16(__uint_as_float(dkv[c8 * 8 + 2 * e]) * a.scale,
                                  __uint_as_float(dkv[c8 * 8 + 2 * e + 1]) * a.scale);
          }
          reinterpret_cast<uint4*>(dvr)[c8] = make_uint4(w[0], w[1], w[2], w[3]);
          reinterpret_cast<uint4*>(dkr)[c8] = make_uint4(x[0], x[1], x[2], x[3]);
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kKMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ dQ
// TMEM columns: S [0,128), dP [128,256), dQ [256, 256+D), dS double buffer 2 x 64 after dQ.
// NP softmax warps per TMEM lane quadrant (each owns 128/NP key columns of S and dP and D/NP
// columns of the dQ accumulator), then the TMA producer and the MMA issuer.
template <int D, int NP>
__global__ void __launch_bounds__((4 * NP + 2) * 32, 1) bwd_dq_kernel(const __grid_constant__ BwdArgs a) {
  using Geo = BwdGeom<D>;
  constexpr int kSoftWarps = 4 * NP, kQProducer = 4 * NP, kQMma = 4 * NP + 1;
  constexpr int CW = kTile / NP;  // key columns per softmax warp
  constexpr uint32_t kColDS = Geo::kColAcc + D;  // first dS buffer
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  // ds_ready is per dS buffer: a barrier can then never run two phases ahead of its waiter
  // consumed_s / consumed_dp: the softmax holds S / dP of the tile in registers, so the next
  // tile's S / dP MMAs may overwrite their columns (S can start before dP has been read)
  __shared__ __align__(8) uint64_t q_full, k_full[3], k_empty[3], v_full[2], v_empty[2], sdp_full, consumed_s,
      consumed_dp, ds_ready[2], acc_full, mma_final;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = a.Hq / a.Hkv;
  const int per_i = a.B * a.Hq;
  // heaviest (last) query tiles first; the rows of this CTA's sequence are [row0, row0 + N) of
  // the token axis, its statistics tiles start at tile0
  int i, row0 = 0, N = a.N, tile0 = 0;
  if (!a.varlen) {
    i = (a.N + kTile - 1) / kTile - 1 - (int)(blockIdx.x / per_i);
  } else {
    const int tg = a.seq_tab[a.n_seq] - 1 - (int)(blockIdx.x / per_i);
    if (tg < 0) return;  // whole CTA, before any barrier or TMEM use
    const int sq = seq_of_tile(a.seq_tab, a.n_seq, tg);
    tile0 = a.seq_tab[sq];
    i = tg - tile0;
    row0 = a.seq_tab[a.n_seq + 1 + sq];
    N = a.seq_tab[2 * a.n_seq + 1 + sq];
  }
  const int rem = blockIdx.x % per_i;
  const int h = rem % a.Hq, b = rem / a.Hq;
  const int g = h / grp;
  const int t0 = i * kTile, t1 = imin(N, t0 + kTile);
  const Range iv = interval_of(a.pat, g);
  const Tiles T = plan_tiles(a.pat, iv, t0, t1);
  const int ntiles = T.count;
  constexpr int KS = Geo::kKSlots, VS = Geo::kVSlots;

  uint8_t* sQ = smem;
  uint8_t* sDO = smem + Geo::kTileBytes;
  uint8_t* sK = smem + 2 * Geo::kTileBytes;
  uint8_t* sV = sK + KS * Geo::kTileBytes;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&q_full, 1);
    for (int s = 0; s < KS; ++s) { ptx::mbar_init(&k_full[s], 1); ptx::mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < VS; ++s) { ptx::mbar_init(&v_full[s], 1); ptx::mbar_init(&v_empty[s], 1); }
    ptx::mbar_init(&sdp_full, 1);
    ptx::mbar_init(&consumed_s, kSoftWarps);
    ptx::mbar_init(&consumed_dp, kSoftWarps);
    ptx::mbar_init(&ds_ready[0], kSoftWarps);
    ptx::mbar_init(&ds_ready[1], kSoftWarps);
    ptx::mbar_init(&acc_full, 1);
    ptx::mbar_init(&mma_final, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kQMma) {
    ptx::tmem_alloc(&tmem_base_sh, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kQProducer) {
    if (lane == 0) {
      ptx::tma_prefetch_desc(&a.tm_k);
      ptx::tma_prefetch_desc(&a.tm_v);
      // (debug builds) the query tile lies inside the sequence, the head and batch inside the call
      const bool q_ok = ptx::dbg_check(t0 >= 0 && t0 < N && h < a.Hq && b < a.B, a.status, &abort_flag, 0x301, t0);
      if (q_ok) {
        ptx::mbar_arrive_expect_tx(&q_full, 2 * Geo::kTileBytes);
        for (int u = 0; u < D / 64; ++u) {
          ptx::tma_load_4d(sQ + u * 16384, &a.tm_q, &q_full, u * 64, row0 + t0, h, b);
          ptx::tma_load_4d(sDO + u * 16384, &a.tm_do, &q_full, u * 64, row0 + t0, h, b);
        }
      }
      TileCursor cur;
      cur.init(T);
      int issued = 0;
      for (int n = 0; q_ok && n < ntiles; ++n, cur.next(T)) {
        const int ks = n % KS, vs = n % VS;
        if (n >= KS && !ptx::mbar_wait(&k_empty[ks], ((n / KS) - 1) & 1, &abort_flag, a.status)) break;
        // (debug builds) every planned KV tile lies inside the sequence
        if (!ptx::dbg_check(cur.j >= 0 && cur.j * kTile < N, a.status, &abort_flag, 0x302, cur.j)) break;
        ptx::mbar_arrive_expect_tx(&k_full[ks], Geo::kTileBytes);
        for (int u = 0; u < D / 64; ++u)
          ptx::tma_load_4d(sK + ks * Geo::kTileBytes + u * 16384, &a.tm_k, &k_full[ks], u * 64, row0 + cur.j * kTile,
                           g, b);
        if (n >= VS && !ptx::mbar_wait(&v_empty[vs], ((n / VS) - 1) & 1, &abort_flag, a.status)) {
          issued = -(n + 1);  // K of tile n is in flight, V is not
          break;
        }
        ptx::mbar_arrive_expect_tx(&v_full[vs], Geo::kTileBytes);
        for (int u = 0; u < D / 64; ++u)
          ptx::tma_load_4d(sV + vs * Geo::kTileBytes + u * 16384, &a.tm_v, &v_full[vs], u * 64, row0 + cur.j * kTile,
                           g, b);
        issued = n + 1;
      }
      // drain: every copy issued must have landed before the CTA exits
      if (q_ok) ptx::mbar_wait(&q_full, 0, nullptr, a.status);
      const int nk = issued < 0 ? -issued : issued, nv = issued < 0 ? -issued - 1 : issued;
      for (int n = (nk > KS ? nk - KS : 0); n < nk; ++n) ptx::mbar_wait(&k_full[n % KS], (n / KS) & 1, nullptr, a.status);
      for (int n = (nv > VS ? nv - VS : 0); n < nv; ++n) ptx::mbar_wait(&v_full[n % VS], (n / VS) & 1, nullptr, a.status);
    }
  } else if (warp == kQMma) {
    // whole warp on the issue path, one elected lane issues (uniform descriptors)
    constexpr uint32_t idesc_s = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_o = ptx::idesc_bf16(128, D, false, true);
    const uint64_t q_desc = ptx::smem_desc_sw128(ptx::smem_u32(sQ), 16, 1024);
    const uint64_t do_desc = ptx::smem_desc_sw128(ptx::smem_u32(sDO), 16, 1024);
    const uint64_t k_desc = ptx::smem_desc_sw128(ptx::smem_u32(sK), 16, 1024);
    const uint64_t k_desc_mn = ptx::smem_desc_sw128(ptx::smem_u32(sK), 16384, 1024);
    const uint64_t v_desc = ptx::smem_desc_sw128(ptx::smem_u32(sV), 16, 1024);
    // S = Q K^T and dP = dO V^T of KV tile n into the S / dP columns; V_n is free afterwards.
    // For n > 0 each half waits until the softmax has read that half of tile n-1.
    auto issue_sdp = [&](int n) -> bool {
      if (n > 0 && !ptx::mbar_wait_warp(&consumed_s, (n - 1) & 1, &abort_flag, a.status)) return false;
      if (!ptx::mbar_wait_warp(&k_full[n % KS], (n / KS) & 1, &abort_flag, a.status)) return false;
      ptx::tc_fence_after();
      const uint64_t kd = ptx::desc_advance(k_desc, (n % KS) * Geo::kTileBytes);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        ptx::mma_bf16_ss_warp(tmem + 0, ptx::desc_advance(q_desc, off), ptx::desc_advance(kd, off), idesc_s, kk > 0);
      }
      if (n > 0 && !ptx::mbar_wait_warp(&consumed_dp, (n - 1) & 1, &abort_flag, a.status)) return false;
      if (!ptx::mbar_wait_warp(&v_full[n % VS], (n / VS) & 1, &abort_flag, a.status)) return false;
      ptx::tc_fence_after();
      const uint64_t vd = ptx::desc_advance(v_desc, (n % VS) * Geo::kTileBytes);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        ptx::mma_bf16_ss_warp(tmem + 128, ptx::desc_advance(do_desc, off), ptx::desc_advance(vd, off), idesc_s, kk > 0);
      }
      ptx::mma_commit_warp(&sdp_full);
      ptx::mma_commit_warp(&v_empty[n % VS]);
      return true;
    };
    bool ok = ptx::mbar_wait_warp(&q_full, 0, &abort_flag, a.status);
    ptx::tc_fence_after();
    if (ok && ntiles > 0) ok = issue_sdp(0);
    for (int n = 0; ok && n < ntiles; ++n) {
      // the softmax holds S(n), dP(n) in registers: compute the next tile's S and dP now
      if (n + 1 < ntiles && !(ok = issue_sdp(n + 1))) break;
      if (!(ok = ptx::mbar_wait_warp(&ds_ready[n & 1], (n >> 1) & 1, &abort_flag, a.status))) break;
      ptx::tc_fence_after();
      // dQ += dS K : A = dS (TMEM buffer n & 1), B = K MN-major in smem
      const uint64_t kd = ptx::desc_advance(k_desc_mn, (n % KS) * Geo::kTileBytes);
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        ptx::mma_bf16_ts_warp(tmem + Geo::kColAcc, tmem + kColDS + (n & 1) * 64 + kk * 8,
                              ptx::desc_advance(kd, kk * 2048), idesc_o, (n > 0 || kk > 0) ? 1u : 0u);
      ptx::mma_commit_warp(&k_empty[n % KS]);
    }
    if (ok) ptx::mma_commit_warp(&acc_full);
    ptx::mma_commit_warp(&mma_final);
    ptx::mbar_wait(&mma_final, 0, nullptr, a.status);
    __syncwarp();
  } else {
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;  // query row = TMEM lane
    const int t = t0 + r;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const size_t so = ((size_t)b * a.Hq + h) * a.N_pad + (size_t)(tile0 + i) * kTile + r;
    const float nlse2 = a.lse2[so], ndelta = a.delta[so];  // stored negated
    const uint64_t nlse2x2 = ptx::f2_pack(nlse2, nlse2), ndeltax2 = ptx::f2_pack(ndelta, ndelta);
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = ptx::f2_pack(sl2, sl2);
    // visible key ranges of row t (absolute positions)
    const int sink_end = imin(a.pat.S, t + 1);
    const int band_lo = imax(0, t - a.pat.L + 1);
    const int lr_lo = iv.lo, lr_hi = imin(iv.hi, t + 1);
    bool ok = true;
    TileCursor cur;
    cur.init(T);
    for (int n = 0; n < ntiles; ++n, cur.next(T)) {
      const int s0 = cur.j * kTile;
      const bool need_mask = (s0 + kTile > N) || !tile_full(a.pat, iv, t0, t1, s0, imin(N, s0 + kTile));
      if (!(ok = ptx::mbar_wait_warp(&sdp_full, n & 1, &abort_flag, a.status))) break;
      ptx::tc_fence_after();
      uint32_t sv[CW], pv[CW];
#pragma unroll
      for (int c = 0; c < CW / 32; ++c) ptx::tmem_ld32(lane_base + part * CW + 32 * c, sv + 32 * c);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < CW / 32; ++c)  // in flight while S is released
        ptx::tmem_ld32(lane_base + 128 + part * CW + 32 * c, pv + 32 * c);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&consumed_s);  // S columns may be overwritten now
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&consumed_dp);  // dP columns too
      // dS buffer n & 1 was last read by dQ(n-2), which the commit of S(n) covers.  The element
      // loop is instantiated with and without the mask, chosen once per tile; two columns per
      // packed fp32x2 instruction
      auto chunks = [&](auto masked) {
        constexpr bool kMask = decltype(masked)::value;
#pragma unroll
        for (int c = 0; c < CW / 32; ++c) {
          uint32_t dw[16];
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) {
            const int cl = 32 * c + 2 * c2;
            float x0, x1;
            ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(sv[cl]), __uint_as_float(sv[cl + 1])), sl2x2,
                                       nlse2x2),
                           x0, x1);
            float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
            if (kMask) {
              const int s = s0 + part * CW + cl;
              const bool vis0 = s <= t && (s < sink_end || s >= band_lo || (s >= lr_lo && s < lr_hi));
              const bool vis1 = s + 1 <= t && (s + 1 < sink_end || s + 1 >= band_lo || (s + 1 >= lr_lo && s + 1 < lr_hi));
              if (!vis0) p0 = 0.f;
              if (!vis1) p1 = 0.f;
            }
            const uint64_t dd = ptx::f2_mul(
                ptx::f2_pack(p0, p1),
                ptx::f2_add(ptx::f2_pack(__uint_as_float(pv[cl]), __uint_as_float(pv[cl + 1])), ndeltax2));
            float d0, d1;
            ptx::f2_unpack(dd, d0, d1);
            dw[c2] = ptx::pack_bf16(d0, d1);
          }
          ptx::tmem_st16(lane_base + kColDS + (n & 1) * 64 + part * (CW / 2) + 16 * c, dw);
        }
      };
      if (need_mask) chunks(std::true_type{});
      else chunks(std::false_type{});
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&ds_ready[n & 1]);
    }
    if (ok && ntiles > 0 && ptx::mbar_wait_warp(&acc_full, 0, &abort_flag, a.status)) {
      ptx::tc_fence_after();
      constexpr int HC = D / NP;  // accumulator columns of this warp
      static_assert(HC % 32 == 0, "dQ columns per softmax warp must be whole 32-column loads");
      uint32_t dqv[HC];
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) ptx::tmem_ld32(lane_base + Geo::kColAcc + part * HC + c * 32, dqv + c * 32);
      ptx::tmem_wait_ld();
      if (t < N) {
        __nv_bfloat16* dqr = reinterpret_cast<__nv_bfloat16*>(a.dq) + b * a.dq_sb + ((int64_t)row0 + t) * a.dq_st +
                             h * a.dq_sh + part * HC;
#pragma unroll
        for (int c8 = 0; c8 < HC / 8; ++c8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = ptx::pack_bf16(__uint_as_float(dqv[c8 * 8 + 2 * e]) * a.scale,
                                  __uint_as_float(dqv[c8 * 8 + 2 * e + 1]) * a.scale);
          reinterpret_cast<uint4*>(dqr)[c8] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kQMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// softmax warps per lane quadrant of the dQ kernel: 4 at d = 128 (32 key columns each); at d = 64
// the accumulator's 64 columns allow 2
#ifndef COWA_DQ_PARTS
#define COWA_DQ_PARTS 4
#endif
template <int D>
constexpr int kDqParts = D == 128 ? COWA_DQ_PARTS : 2;
// softmax warps per lane quadrant of the dK/dV kernel (64 / NP query columns each); 4 measured
// 5% slower than 2 on B200 for this kernel
#ifndef COWA_DKDV_PARTS
#define COWA_DKDV_PARTS 2
#endif
template <int D>
constexpr int kDkdvParts = D == 128 ? COWA_DKDV_PARTS : 2;

// ------------------------------------------------------------------------------ split key tiles
// Query tiles of key tile j for local KV head g (the dK/dV kernel's range).
__host__ __device__ __forceinline__ int kv_range_tiles(const Pat& p, Range iv, int j, int N) {
  const int s0 = j * kTile, s1 = imin(N, s0 + kTile);
  const Range r = bwd_row_range(p, iv, s0, s1, N);
  return (r.hi + kTile - 1) / kTile - r.lo / kTile;
}

// The chunk table of a split call (one block): every key tile (g-major, then j) whose range
// exceeds `chunk` query tiles contributes ceil(range / chunk) consecutive entries {j, g, b, k},
// batch element by batch element (entries of b at b * per_b).
__global__ void __launch_bounds__(256) kv_split_table_kernel(Pat p, int N, int B, int Hkv, int chunk, int4* tab) {
  __shared__ int offs[256];
  __shared__ int per_b;
  const int nq = (N + kTile - 1) / kTile, pairs = Hkv * nq, t = threadIdx.x;
  const int per = (pairs + 255) / 256;
  const int lo = imin(pairs, t * per), hi = imin(pairs, lo + per);
  int cnt = 0;
  for (int q = lo; q < hi; ++q) {
    const int g = q / nq, j = q % nq;
    const int n = kv_range_tiles(p, interval_of(p, g), j, N);
    if (n > chunk) cnt += (n + chunk - 1) / chunk;
  }
  offs[t] = cnt;
  __syncthreads();
  if (t == 0) {  // exclusive scan of 256 counts, in order
    int acc = 0;
    for (int i = 0; i < 256; ++i) { const int v = offs[i]; offs[i] = acc; acc += v; }
    per_b = acc;
  }
  __syncthreads();
  int e = offs[t];
  for (int q = lo; q < hi; ++q) {
    const int g = q / nq, j = q % nq;
    const int n = kv_range_tiles(p, interval_of(p, g), j, N);
    if (n <= chunk) continue;
    for (int k = 0; k < (n + chunk - 1) / chunk; ++k, ++e)
      for (int bb = 0; bb < B; ++bb) tab[(size_t)bb * per_b + e] = make_int4(j, g, bb, k);
  }
}

// The chunk table of a packed batch (one block, after the sequence table): the same rule over
// the packed key tiles of every sequence, within `cap` slots.  Tiles are taken in order while
// their chunks fit; kv_flag marks the split ones, the rest stay whole; unused slots hold chunk -1.
__global__ void __launch_bounds__(256) kv_split_table_varlen_kernel(Pat p, const int32_t* seq_tab, int n_seq, int Hkv,
                                                                    int chunk, int cap, int bound, int4* tab,
                                                                    int32_t* flag) {
  __shared__ int offs[256];
  const int tiles = seq_tab[n_seq], pairs = Hkv * tiles, t = threadIdx.x;
  for (int i = t; i < cap; i += 256) tab[i] = make_int4(0, 0, 0, -1);
  const int per = (pairs + 255) / 256;
  const int lo = imin(pairs, t * per), hi = imin(pairs, lo + per);
  auto range_of = [&](int q, int& g, int& tg) {
    g = q / tiles;
    tg = q % tiles;
    const int sq = seq_of_tile(seq_tab, n_seq, tg);
    return kv_range_tiles(p, interval_of(p, g), tg - seq_tab[sq], seq_tab[2 * n_seq + 1 + sq]);
  };
  int cnt = 0;
  for (int q = lo; q < hi; ++q) {
    int g, tg;
    const int n = range_of(q, g, tg);
    if (n > chunk) cnt += (n + chunk - 1) / chunk;
  }
  offs[t] = cnt;
  __syncthreads();
  if (t == 0) {
    int acc = 0;
    for (int i = 0; i < 256; ++i) { const int v = offs[i]; offs[i] = acc; acc += v; }
  }
  __syncthreads();  // also orders the sentinel fill before the entries below
  int e = offs[t];
  for (int q = lo; q < hi; ++q) {
    int g, tg;
    const int n = range_of(q, g, tg);
    const int m = n > chunk ? (n + chunk - 1) / chunk : 0;
    const bool fits = m > 0 && e + m <= cap;
    flag[(size_t)g * bound + tg] = fits ? 1 : 0;
    if (fits)
      for (int k = 0; k < m; ++k) tab[e + k] = make_int4(tg, g, 0, k);
    e += m;
  }
}

// dk, dv of the split key tiles: the chunks' fp32 partials summed in chunk order (one block per
// tile, run by the block of its first chunk), dk scaled, rounded to bf16.
template <int D>
__global__ void __launch_bounds__(256) kv_split_reduce_kernel(const __grid_constant__ BwdArgs a) {
  const int e0 = blockIdx.x;
  const int4 t = a.kv_tab[e0];
  if (t.w != 0) return;  // not a tile's first chunk (or an unused slot)
  int j = t.x, row0 = 0, N = a.N;
  const int g = t.y, b = t.z;
  if (a.varlen) {  // the key tile's sequence on the packed token axis
    const int sq = seq_of_tile(a.seq_tab, a.n_seq, j);
    j -= a.seq_tab[sq];
    row0 = a.seq_tab[a.n_seq + 1 + sq];
    N = a.seq_tab[2 * a.n_seq + 1 + sq];
  }
  int n = 1;  // the tile's chunks are consecutive entries
  while (e0 + n < a.n_split && a.kv_tab[e0 + n].w == n) ++n;
  const int s0 = j * kTile;
  for (int idx = threadIdx.x; idx < kTile * D / 4; idx += blockDim.x) {
    const int r = idx / (D / 4), c4 = idx % (D / 4);
    float4 sv = make_float4(0.f, 0.f, 0.f, 0.f), sk = sv;
    for (int c = 0; c < n; ++c) {
      const float* pp = a.kv_part + (size_t)(e0 + c) * 2 * kTile * D + (size_t)r * D;
      const float4 v = reinterpret_cast<const float4*>(pp)[c4];
      const float4 k = reinterpret_cast<const float4*>(pp + (size_t)kTile * D)[c4];
      sv.x += v.x; sv.y += v.y; sv.z += v.z; sv.w += v.w;
      sk.x += k.x; sk.y += k.y; sk.z += k.z; sk.w += k.w;
    }
    if (s0 + r < N) {
      __nv_bfloat16* dvr = reinterpret_cast<__nv_bfloat16*>(a.dv) + b * a.dv_sb +
                           ((int64_t)row0 + s0 + r) * a.dv_st + g * a.dv_sh + c4 * 4;
      __nv_bfloat16* dkr = reinterpret_cast<__nv_bfloat16*>(a.dk) + b * a.dk_sb +
                           ((int64_t)row0 + s0 + r) * a.dk_st + g * a.dk_sh + c4 * 4;
      *reinterpret_cast<uint2*>(dvr) = make_uint2(ptx::pack_bf16(sv.x, sv.y), ptx::pack_bf16(sv.z, sv.w));
      *reinterpret_cast<uint2*>(dkr) = make_uint2(ptx::pack_bf16(sk.x * a.scale, sk.y * a.scale),
                                                  ptx::pack_bf16(sk.z * a.scale, sk.w * a.scale));
    }
  }
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs& a, int stages, cudaStream_t s) {
  using Geo = BwdGeom<D>;
  const int nq = a.N_pad / kTile;
  cudaError_t e;
  if (stages & COWA_BWD_PREPROCESS) {
    bwd_preprocess_kernel<D><<<dim3(nq, a.Hq, a.B), 256, 0, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (stages & COWA_BWD_DKDV) {
    constexpr int NPK = kDkdvParts<D>;
    auto kdkdv = bwd_dkdv_kernel<D, NPK>;
    if ((e = cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::kSmemKV)) != cudaSuccess)
      return e;
    const long long n_kv = (long long)nq * a.Hkv * a.B + a.n_split;
    if (n_kv > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (a.n_split > 0) {
      if (a.varlen)
        kv_split_table_varlen_kernel<<<1, 256, 0, s>>>(a.pat, a.seq_tab, a.n_seq, a.Hkv, a.kv_chunk, a.n_split,
                                                       a.kv_bound, a.kv_tab, a.kv_flag);
      else
        kv_split_table_kernel<<<1, 256, 0, s>>>(a.pat, a.N, a.B, a.Hkv, a.kv_chunk, a.kv_tab);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    kdkdv<<<(unsigned)n_kv, (4 * NPK + 2) * 32, Geo::kSmemKV, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.n_split > 0) {
      kv_split_reduce_kernel<D><<<a.n_split, 256, 0, s>>>(a);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  if (stages & COWA_BWD_DQ) {
    constexpr int NP = kDqParts<D>;
    auto kdq = bwd_dq_kernel<D, NP>;
    if ((e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::kSmemQ)) != cudaSuccess)
      return e;
    const long long n_q = (long long)nq * a.Hq * a.B;
    if (n_q > 0x7fffffffLL) return cudaErrorInvalidValue;
    kdq<<<(unsigned)n_q, (4 * NP + 2) * 32, Geo::kSmemQ, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

// Split plan of a call (see BwdArgs).  A key tile whose query range is longer than the work an
// SM averages over the launch would finish last whatever the order (a sink key tile walks every
// query tile of every head of its group): with few KV heads per call (KV-head tensor
// parallelism, layers with one or two KV heads) that one CTA sets the kernel's time.  Such
// ranges are cut into chunks of about that mean work; calls whose longest range is within it
// (the 8-head layers, where the other heads' tiles fill the SMs) are not split.
KvSplit kv_split_plan(const Pat& p, int B, int N, int Hq, int Hkv) {
  constexpr long long kSms = 148;  // B200
  KvSplit sp{0, 0};
  const int nq = (N + kTile - 1) / kTile;
  long long total = 0;
  int longest = 0;
  for (int g = 0; g < Hkv; ++g) {
    const Range iv = interval_of(p, g);
    for (int j = 0; j < nq; ++j) {
      const int n = kv_range_tiles(p, iv, j, N);
      total += n;
      longest = imax(longest, n);
    }
  }
  // query tiles per SM over the launch (each costs the same grp heads x 2 sub-steps everywhere)
  const long long per_sm = total * B / kSms;
  const int chunk = (int)(per_sm > 8 ? per_sm : 8);
  if (longest <= chunk) return sp;
  sp.chunk = chunk;
  for (int g = 0; g < Hkv; ++g) {
    const Range iv = interval_of(p, g);
    for (int j = 0; j < nq; ++j) {
      const int n = kv_range_tiles(p, iv, j, N);
      if (n > chunk) sp.n_entries += (n + chunk - 1) / chunk;
    }
  }
  sp.n_entries *= B;
  (void)Hq;  // every key tile walks its query tiles for all Hq / Hkv heads alike
  return sp;
}

size_t bwd_workspace_bytes(const Pat& p, int B, int N, int Hq, int Hkv, int d) {
  const size_t n_pad = (size_t)(N + kTile - 1) / kTile * kTile;
  size_t bytes = align_up(2 * (size_t)B * Hq * n_pad * sizeof(float), 256);
  const KvSplit sp = kv_split_plan(p, B, N, Hq, Hkv);
  if (sp.chunk > 0)
    bytes += align_up((size_t)sp.n_entries * sizeof(int4), 256) + (size_t)sp.n_entries * 2 * kTile * d * sizeof(float);
  return bytes;
}

cudaError_t launch_bwd(const BwdArgs& a, int stages, cudaStream_t s) {
  if (a.d == 64) return launch_bwd_d<64>(a, stages, s);
  if (a.d == 128) return launch_bwd_d<128>(a, stages, s);
  return cudaErrorInvalidValue;
}

}  // namespace cowa
