// cowa_fwd.cu -- CoWA forward on sm_100a: exact softmax attention over the position-defined
// visible set of each KV head ("CoWindow Attention: Full Causal Coverage Is a Collective
// Property", Abstract; skillfed.io news summary, paragraphs 2 and 7).
//
// One CTA = (batch b, KV head g, 128-row query tile i, a pair of query heads of g's GQA
// group).  The two heads share every K/V tile the CTA loads and the same tile plan, because
// the mask depends on g only.  Warp roles (12 warps = 3 warpgroups):
//   warps 0-3  softmax for head slot 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax for head slot 1
//   warp  8    TMA producer: Q once, then K_j, V_j of every visited KV tile into a 5-slot ring
//   warp  9    tcgen05 MMA issuer (the whole warp walks the loop, one elected lane issues):
//              S = Q K^T into TMEM, O += P V into TMEM
//   warps 10-11 idle (they complete the third warpgroup)
// The same kernel serves a block of queries at an offset against keys already written
// (chunked prefill: query rows q_off.., keys 0..Nk-1) and packed variable-length batches (each
// CTA finds its sequence in per-sequence tile offsets and works on that sequence's rows).
// Registers: the kernel is compiled for 168 per thread (384 * 168 = 64512 at launch); the two
// softmax warpgroups then raise theirs to 216 and the third lowers to 72
// (2*128*216 + 128*72 = 64512), so a whole 128-column score row stays in registers.  The
// launcher checks the compiled count before the first launch, because a split larger than
// the launch allocation would wait forever.
// The visited KV tiles come from the planner (sink tiles, interval_g tiles, near-diagonal
// band, merged); only tiles that are not entirely visible apply the element mask.
//
// Softmax: online, in the log2 domain, with a lazy rescale of O (only when the running max
// grows by more than 2^8; the final division uses the same stale max, so the result is
// exact).  P is rounded to bf16 and written back into TMEM over the S columns it came from,
// where the P V MMA reads it as its A operand (no shared-memory round trip).  fp32
// accumulation throughout.  Exponentials run on the special-function unit (an FMA-pipe
// polynomial share measured slower on B200 here).  Each tile's exponentials use the running
// max from before the tile while the tile's own max is gathered in the same pass; the tile is
// redone only when that max grows the running one past the rescale threshold, so the common
// path never waits for a row reduction and gives the same bits as max-first.
//
// MMA order per KV tile n: S0(n), PV1(n-1), S1(n), PV0(n).  Softmax 0 works on S0(n) while
// the tensor core runs PV1(n-1) and S1(n), softmax 1 on S1(n) during PV0(n) and S0(n+1).
// tcgen05 MMAs of one thread execute in issue order, so S_k(n+1) overwriting P_k(n) is safe
// once PV_k(n) is issued, and the commit that announces S_k(n) also covers PV_k(n-1).
//
// TMEM (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 [256, 256+D), O1 [256+D, 256+2D).
#include <cuda_bf16.h>
#include <math.h>

#include "cowa_internal.h"
#include "kernel_common.cuh"
#include "sm100_ptx.cuh"

namespace cowa {
namespace {

constexpr int kBM = kTile, kBN = kTile;
constexpr int kFwdThreads = 384;
constexpr int kRegsLaunch = 168, kRegsSoftmax = 216, kRegsOther = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther == kFwdThreads * kRegsLaunch,
              "register split must add up to the launch allocation");
constexpr int kRingMax = 8;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct FwdGeom {
  static constexpr int kQBytes = kBM * D * 2;   // one head's Q tile
  static constexpr int kKVBytes = kBN * D * 2;  // one K or V tile
  // K/V ring depth: a K or V tile takes ~5000 cycles to arrive from L2 under full load, so
  // each slot must be refilled about two tile periods ahead (5 x 32 KB for d = 128)
  static constexpr int kRing = D == 128 ? 5 : kRingMax;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = 2 * kQBytes;
  static constexpr int kSmem = kOffRing + kRing * kKVBytes + 1024;  // + alignment slack
  static_assert(kRing <= kRingMax && kSmem <= 227 * 1024, "shared memory budget");
  static constexpr int kColO = 256;
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1) cowa_fwd_kernel(const __grid_constant__ FwdArgs a) {
  using Geo = FwdGeom<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t kv_full[kRingMax], kv_empty[kRingMax];
  __shared__ __align__(8) uint64_t s_full[2], p_ready[2], o_done[2];
  __shared__ __align__(8) uint64_t mma_final;
  // single-head tile (odd GQA group): softmax 1's running max and sum per row for the merge
  __shared__ __align__(8) uint64_t merge_ready;
  __shared__ float merge_m[kBM], merge_l[kBM];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: heaviest (last) query tiles first; all heads/pairs of one tile adjacent
  const int grp = a.Hq / a.Hkv;
  const int npair = (grp + 1) >> 1;
  const int per_i = a.B * a.Hkv * npair;
  int i, row0 = 0, Nq = a.Nq, Nk = a.Nk, q_off = a.q_off;  // row0: first row of the sequence
  if (!a.varlen) {
    i = (a.Nq + kBM - 1) / kBM - 1 - (int)(blockIdx.x / per_i);
  } else {
    // the grid is an upper bound on the q-tiles of the packed batch: find this CTA's sequence
    const int tiles = a.seq_tab[a.n_seq];
    const int tg = tiles - 1 - (int)(blockIdx.x / per_i);
    if (tg < 0) return;  // whole CTA, before any barrier or TMEM use
    const int sq = seq_of_tile(a.seq_tab, a.n_seq, tg);
    i = tg - a.seq_tab[sq];
    row0 = a.seq_tab[a.n_seq + 1 + sq];
    Nq = Nk = a.seq_tab[2 * a.n_seq + 1 + sq];
    q_off = 0;
  }
  int rem = blockIdx.x % per_i;
  const int pair = rem % npair; rem /= npair;
  const int g = rem % a.Hkv;
  const int b = rem / a.Hkv;
  const int h0 = g * grp + 2 * pair;
  const bool has1 = (2 * pair + 1) < grp;
  // query rows of the tile: local q rows [i*BM, ...), absolute positions [t0, t1)
  const int t0 = q_off + i * kBM, t1 = imin(q_off + Nq, t0 + kBM);
  const Range iv = interval_of(a.pat, g);
  const Tiles T = plan_tiles(a.pat, iv, t0, t1);

  uint8_t* sQ = smem + Geo::kOffQ;
  uint8_t* sRing = smem + Geo::kOffRing;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&q_full, 1);
    for (int s = 0; s < Geo::kRing; ++s) { ptx::mbar_init(&kv_full[s], 1); ptx::mbar_init(&kv_empty[s], 1); }
    for (int k = 0; k < 2; ++k) {
      ptx::mbar_init(&s_full[k], 1);
      ptx::mbar_init(&p_ready[k], 4);
      ptx::mbar_init(&o_done[k], 1);
    }
    ptx::mbar_init(&mma_final, 1);
    ptx::mbar_init(&merge_ready, 4);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(&tmem_base_sh, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int ntiles = T.count;
  if (warp >= 8) {
    // warpgroup-wide register reallocation: this warpgroup gives registers to the softmax ones
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
  }
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::tma_prefetch_desc(&a.tm_q);
      ptx::tma_prefetch_desc(&a.tm_k);
      ptx::tma_prefetch_desc(&a.tm_v);
      // (debug builds) the work item addresses rows and heads of the call
      const bool q_ok = ptx::dbg_check(i >= 0 && i * kBM < Nq && h0 + (has1 ? 1 : 0) < a.Hq && b < a.B, a.status,
                                       &abort_flag, 0x101, i);
      if (q_ok) {
        ptx::mbar_arrive_expect_tx(&q_full, (has1 ? 2 : 1) * Geo::kQBytes);
        for (int u = 0; u < D / 64; ++u) {
          ptx::tma_load_4d(sQ + u * 16384, &a.tm_q, &q_full, u * 64, row0 + i * kBM, h0, b);
          if (has1) ptx::tma_load_4d(sQ + Geo::kQBytes + u * 16384, &a.tm_q, &q_full, u * 64, row0 + i * kBM, h0 + 1, b);
        }
      }
      TileCursor cur;
      cur.init(T);
      int issued = 0;
      for (int idx = 0; q_ok && idx < 2 * ntiles; ++idx) {
        const int s = idx % Geo::kRing;
        if (idx >= Geo::kRing && !ptx::mbar_wait(&kv_empty[s], ((idx / Geo::kRing) - 1) & 1, &abort_flag, a.status)) break;
        // (debug builds) every planned KV tile lies inside the keys of the call
        if (!ptx::dbg_check(cur.j >= 0 && cur.j * kBN < Nk, a.status, &abort_flag, 0x102, cur.j)) break;
        const bool is_v = idx & 1;
        uint8_t* dst = sRing + s * Geo::kKVBytes;
        ptx::mbar_arrive_expect_tx(&kv_full[s], Geo::kKVBytes);
        for (int u = 0; u < D / 64; ++u)
          ptx::tma_load_4d(dst + u * 16384, is_v ? &a.tm_v : &a.tm_k, &kv_full[s], u * 64, row0 + cur.j * kBN, g, b);
        if (is_v) cur.next(T);
        issued = idx + 1;
      }
      // drain: no copy may still be landing in shared memory when the CTA exits
      if (q_ok) ptx::mbar_wait(&q_full, 0, nullptr, a.status);
      for (int idx = (issued > Geo::kRing ? issued - Geo::kRing : 0); idx < issued; ++idx)
        ptx::mbar_wait(&kv_full[idx % Geo::kRing], (idx / Geo::kRing) & 1, nullptr, a.status);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp walks the issue loop (uniform operands); one elected lane issues each
    // MMA and commit.  Descriptors are built once and advanced by constant offsets.
    constexpr uint32_t idesc_s = ptx::idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_o = ptx::idesc_bf16(128, D, false, true);
    const uint64_t q_desc = ptx::smem_desc_sw128(ptx::smem_u32(sQ), 16, 1024);
    const uint64_t k_desc = ptx::smem_desc_sw128(ptx::smem_u32(sRing), 16, 1024);
    const uint64_t v_desc = ptx::smem_desc_sw128(ptx::smem_u32(sRing), 16384, 1024);
    const int nslot = has1 ? 2 : 1;

    auto issue_s = [&](int k, int kslot, int qk) {  // S_k = Q_qk K^T
      const uint64_t qd = ptx::desc_advance(q_desc, qk * Geo::kQBytes);
      const uint64_t kd = ptx::desc_advance(k_desc, kslot * Geo::kKVBytes);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        ptx::mma_bf16_ss_warp(tmem + k * 128, ptx::desc_advance(qd, off), ptx::desc_advance(kd, off), idesc_s,
                              kk > 0 ? 1u : 0u);
      }
    };
    // O_k (+)= P_k V: P_k (bf16, in TMEM over the S_k columns) is the A operand
    auto issue_pv = [&](int k, int vslot, bool accumulate) {
      const uint64_t vd = ptx::desc_advance(v_desc, vslot * Geo::kKVBytes);
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        ptx::mma_bf16_ts_warp(tmem + Geo::kColO + k * D, tmem + k * 128 + kk * 8, ptx::desc_advance(vd, kk * 2048),
                              idesc_o, (accumulate || kk > 0) ? 1u : 0u);
    };

    bool ok = ptx::mbar_wait_warp(&q_full, 0, &abort_flag, a.status);
    ptx::tc_fence_after();
    if (nslot == 1) {
      // One query head (odd group): the two softmax warpgroups take alternate KV tiles of it,
      // slot 0 the even ones and slot 1 the odd ones, each with its own running max, sum and
      // O accumulator (merged at the end), so the tensor core still alternates between two
      // softmaxes.  Iteration j: S0(2j), PV1(2j-1), S1(2j+1), PV0(2j).
      const int n0cnt = (ntiles + 1) / 2, n1cnt = ntiles / 2;
      for (int j = 0; ok && j < n0cnt; ++j) {
        const int ne = 2 * j, no = 2 * j + 1;
        const int kidx0 = 2 * ne, vidx0 = kidx0 + 1, kidx1 = 2 * no;
        if (!(ok = ptx::mbar_wait_warp(&kv_full[kidx0 % Geo::kRing], (kidx0 / Geo::kRing) & 1, &abort_flag,
                                       a.status)))
          break;
        ptx::tc_fence_after();
        issue_s(0, kidx0 % Geo::kRing, 0);
        ptx::mma_commit_warp(&s_full[0]);
        ptx::mma_commit_warp(&kv_empty[kidx0 % Geo::kRing]);
        if (j > 0) {  // PV1 of the previous odd tile 2j-1 (odd-tile index j-1)
          const int pv = 2 * (2 * j - 1) + 1;
          if (!(ok = ptx::mbar_wait_warp(&kv_full[pv % Geo::kRing], (pv / Geo::kRing) & 1, &abort_flag, a.status)))
            break;
          if (!(ok = ptx::mbar_wait_warp(&p_ready[1], (j - 1) & 1, &abort_flag, a.status))) break;
          ptx::tc_fence_after();
          issue_pv(1, pv % Geo::kRing, j - 1 > 0);
          ptx::mma_commit_warp(&kv_empty[pv % Geo::kRing]);
        }
        if (no < ntiles) {
          if (!(ok = ptx::mbar_wait_warp(&kv_full[kidx1 % Geo::kRing], (kidx1 / Geo::kRing) & 1, &abort_flag,
                                         a.status)))
            break;
          ptx::tc_fence_after();
          issue_s(1, kidx1 % Geo::kRing, 0);
          ptx::mma_commit_warp(&s_full[1]);
          ptx::mma_commit_warp(&kv_empty[kidx1 % Geo::kRing]);
        }
        if (!(ok = ptx::mbar_wait_warp(&kv_full[vidx0 % Geo::kRing], (vidx0 / Geo::kRing) & 1, &abort_flag,
                                       a.status)))
          break;
        if (!(ok = ptx::mbar_wait_warp(&p_ready[0], j & 1, &abort_flag, a.status))) break;
        ptx::tc_fence_after();
        issue_pv(0, vidx0 % Geo::kRing, j > 0);
        ptx::mma_commit_warp(&kv_empty[vidx0 % Geo::kRing]);
      }
      if (ok && ntiles > 0) {
        ptx::mma_commit_warp(&o_done[0]);
        if (ntiles % 2 == 0) {  // the last odd tile's PV1 is still to issue
          const int no = ntiles - 1, pv = 2 * no + 1;
          ok = ptx::mbar_wait_warp(&kv_full[pv % Geo::kRing], (pv / Geo::kRing) & 1, &abort_flag, a.status) &&
               ptx::mbar_wait_warp(&p_ready[1], (n1cnt - 1) & 1, &abort_flag, a.status);
          if (ok) {
            ptx::tc_fence_after();
            issue_pv(1, pv % Geo::kRing, n1cnt - 1 > 0);
            ptx::mma_commit_warp(&kv_empty[pv % Geo::kRing]);
          }
        }
        if (ok && n1cnt > 0) ptx::mma_commit_warp(&o_done[1]);
      }
    }
    for (int n = 0; ok && nslot == 2 && n < ntiles; ++n) {
      const int kidx = 2 * n, vidx = 2 * n + 1;
      const int kslot = kidx % Geo::kRing, vslot = vidx % Geo::kRing;
      if (!(ok = ptx::mbar_wait_warp(&kv_full[kslot], (kidx / Geo::kRing) & 1, &abort_flag, a.status))) break;
      ptx::tc_fence_after();
      // S0(n): P0(n-1) was consumed by PV0(n-1), issued earlier
      issue_s(0, kslot, 0);
      ptx::mma_commit_warp(&s_full[0]);
      if (nslot == 2) {
        // PV1(n-1): overlaps with softmax 0 working on S0(n)
        if (n > 0) {
          const int pv = 2 * (n - 1) + 1;
          if (!(ok = ptx::mbar_wait_warp(&p_ready[1], (n - 1) & 1, &abort_flag, a.status))) break;
          ptx::tc_fence_after();
          issue_pv(1, pv % Geo::kRing, n - 1 > 0);
          ptx::mma_commit_warp(&kv_empty[pv % Geo::kRing]);
        }
        issue_s(1, kslot, 1);
        ptx::mma_commit_warp(&s_full[1]);
      }
      ptx::mma_commit_warp(&kv_empty[kslot]);
      // PV0(n)
      if (!(ok = ptx::mbar_wait_warp(&kv_full[vslot], (vidx / Geo::kRing) & 1, &abort_flag, a.status))) break;
      if (!(ok = ptx::mbar_wait_warp(&p_ready[0], n & 1, &abort_flag, a.status))) break;
      ptx::tc_fence_after();
      issue_pv(0, vslot, n > 0);
    }
    if (ok && nslot == 2 && ntiles > 0) {
      ptx::mma_commit_warp(&o_done[0]);
      {
        const int n = ntiles - 1, pv = 2 * n + 1;
        if (ptx::mbar_wait_warp(&p_ready[1], n & 1, &abort_flag, a.status)) {
          ptx::tc_fence_after();
          issue_pv(1, pv % Geo::kRing, n > 0);
          ptx::mma_commit_warp(&kv_empty[pv % Geo::kRing]);
          ptx::mma_commit_warp(&o_done[1]);
        }
      }
    }
    // all issued MMAs complete before TMEM can be released
    ptx::mma_commit_warp(&mma_final);
    ptx::mbar_wait(&mma_final, 0, nullptr, a.status);
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int k = warp >> 2;  // head slot
    const bool split = !has1;  // one head: the two slots take alternate KV tiles of it
    {
      const int r = (warp & 3) * 32 + lane;  // query row in the tile = TMEM lane
      const int t = t0 + r;
      const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
      const uint32_t s_tm = lane_base + k * 128;
      const uint32_t o_tm = lane_base + Geo::kColO + k * D;
      float m_used = -INFINITY;
      const float sl2 = a.scale_log2;
      const uint64_t sl2x2 = ptx::f2_pack(sl2, sl2);
      uint64_t lsum = ptx::f2_pack(0.f, 0.f);
      bool ok = true;
      TileCursor cur;
      cur.init(T);
      int cnt = 0;  // tiles of this slot so far
      for (int n = 0; n < ntiles; ++n, cur.next(T)) {
        if (split && (n & 1) != k) continue;
        const int s0 = cur.j * kBN;
        const bool need_mask = (s0 + kBN > Nk) || !tile_full(a.pat, iv, t0, t1, s0, imin(Nk, s0 + kBN));
        if (!(ok = ptx::mbar_wait_warp(&s_full[k], cnt & 1, &abort_flag, a.status))) break;
        ptx::tc_fence_after();
        // visible key columns of row t within [s0, s0+128), relative to s0 (partial tiles only)
        const int sink_end = imin(a.pat.S, t + 1) - s0;
        const int band_lo = imax(0, t - a.pat.L + 1) - s0;
        const int diag_end = t + 1 - s0;
        const int lr_lo = iv.lo - s0, lr_hi = imin(iv.hi, t + 1) - s0;
        uint32_t xr[128];
#pragma unroll
        for (int q = 0; q < 4; ++q) ptx::tmem_ld32(s_tm + q * 32, xr + q * 32);
        ptx::tmem_wait_ld();
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const bool vis = (c < sink_end) || (c >= band_lo && c < diag_end) || (c >= lr_lo && c < lr_hi);
            if (!vis) xr[c] = 0xff800000u;  // -inf: gives exactly 0
          }
        }
        // P = 2^(s*scale*log2e - m) with m the running max from before this tile, rounded to
        // bf16 and written back into TMEM over the S columns (the A operand of P V); the tile's
        // row max is gathered in the same pass.  Only when that max grows the running one by
        // more than 2^8 (lazy rescale; rare after the first tiles) is the tile redone with the
        // new max, so the common path never waits for the row reduction.
        uint64_t ts[4];  // this tile's row sum, 4 independent packed accumulators
        float pm[8];     // partial row maxima
        auto pass = [&](float m) {
          const uint64_t negm = ptx::f2_pack(-m, -m);
#pragma unroll
          for (int e = 0; e < 4; ++e) ts[e] = ptx::f2_pack(0.f, 0.f);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pw[32];
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
              const int c = 64 * h + 2 * c2;
              float e0, e1;
              ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(xr[c]), __uint_as_float(xr[c + 1])), sl2x2, negm),
                             e0, e1);
              const float p0 = ptx::ex2(e0), p1 = ptx::ex2(e1);
              ts[c2 & 3] = ptx::f2_add(ts[c2 & 3], ptx::f2_pack(p0, p1));
              pw[c2] = ptx::pack_bf16(p0, p1);
            }
            ptx::tmem_st32(s_tm + 32 * h, pw);
          }
        };
        pass(m_used == -INFINITY ? 0.f : m_used);
        // row max (independent of the exponentials above, so it overlaps them)
#pragma unroll
        for (int e = 0; e < 8; ++e) pm[e] = fmaxf(__uint_as_float(xr[e]), __uint_as_float(xr[e + 8]));
#pragma unroll
        for (int c = 16; c < 128; c += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e) pm[e] = ptx::fmax3(pm[e], __uint_as_float(xr[c + e]), __uint_as_float(xr[c + 8 + e]));
        const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        const float m_new = fmaxf(m_used, mx * sl2);
        const bool grow = (m_new != -INFINITY) && (m_used == -INFINITY || m_new > m_used + kRescaleThreshold);
        if (__any_sync(0xffffffffu, grow)) {
          float alpha = 1.f;
          if (grow) {
            alpha = ptx::ex2(m_used - m_new);  // 0 when nothing was visible before
            m_used = m_new;
            lsum = ptx::f2_mul(lsum, ptx::f2_pack(alpha, alpha));
          }
          if (cnt > 0) {
            // O row *= alpha, a warp-collective TMEM round trip (alpha = 1 on the other lanes);
            // PV_k(n-1) has completed (the commit of S_k(n) covers it), so O_k is stable here
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t ov[32];
              ptx::tmem_ld32(o_tm + c * 32, ov);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
              ptx::tmem_st32(o_tm + c * 32, ov);
            }
          }
          // redo the tile from the scores still in registers (lanes whose max did not grow
          // recompute the same values); the stores replace the speculative P
          ptx::tmem_wait_st();
          pass(m_used == -INFINITY ? 0.f : m_used);
        }
        lsum = ptx::f2_add(lsum, ptx::f2_add(ptx::f2_add(ts[0], ts[1]), ptx::f2_add(ts[2], ts[3])));
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&p_ready[k]);
        ++cnt;
      }
      float la, lb;
      ptx::f2_unpack(lsum, la, lb);
      const float l = la + lb;
      // ---- epilogue
      const int rl = t - q_off;  // query row within the call's (or the sequence's) rows
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + (size_t)b * a.o_sb + (size_t)(row0 + rl) * a.o_st +
                            (size_t)h0 * a.o_sh;
      // lse: [B, H_q, N_q], or [H_q, total] for a packed batch
      const size_t lse_h0 = a.varlen ? (size_t)h0 * a.total + row0 + rl : ((size_t)b * a.Hq + h0) * a.Nq + rl;
      const size_t lse_step = a.varlen ? (size_t)a.total : (size_t)a.Nq;  // to the next head
      if (!split) {
        if (ok && ntiles > 0 && ptx::mbar_wait_warp(&o_done[k], 0, &abort_flag, a.status)) {
          ptx::tc_fence_after();
          const float inv = 1.f / l;
          if (t < t1) a.lse[lse_h0 + k * lse_step] = (m_used + log2f(l)) * 0.69314718055994530942f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            ptx::tmem_ld32(o_tm + c * 32, ov);  // warp-collective: every lane loads, valid rows store
            ptx::tmem_wait_ld();
            if (t < t1) {
#pragma unroll
              for (int c8 = 0; c8 < 4; ++c8) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  w[e] = ptx::pack_bf16(__uint_as_float(ov[c8 * 8 + 2 * e]) * inv,
                                        __uint_as_float(ov[c8 * 8 + 2 * e + 1]) * inv);
                reinterpret_cast<uint4*>(orow + (size_t)k * a.o_sh)[c * 4 + c8] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
      } else if (k == 1) {
        // hand this slot's running max and sum to slot 0, which merges the two halves
        const bool have = ok && cnt > 0 && ptx::mbar_wait_warp(&o_done[1], 0, &abort_flag, a.status);
        ptx::tc_fence_after();
        merge_m[r] = have ? m_used : -INFINITY;
        merge_l[r] = have ? l : 0.f;
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&merge_ready);
      } else if (ok && ntiles > 0 && ptx::mbar_wait_warp(&o_done[0], 0, &abort_flag, a.status) &&
                 ptx::mbar_wait_warp(&merge_ready, 0, &abort_flag, a.status)) {
        // O = (O0 2^(m0-m) + O1 2^(m1-m)) / (l0 2^(m0-m) + l1 2^(m1-m)), m = max(m0, m1)
        ptx::tc_fence_after();
        const float m1 = merge_m[r], l1 = merge_l[r];
        const float m = fmaxf(m_used, m1);
        const float f0 = m_used == -INFINITY ? 0.f : ptx::ex2(m_used - m);
        const float f1 = m1 == -INFINITY ? 0.f : ptx::ex2(m1 - m);
        const float lt = l * f0 + l1 * f1;
        const float inv = 1.f / lt, g0 = f0 * inv, g1 = f1 * inv;
        const bool two = ntiles > 1;  // slot 1 has tiles (uniform over the CTA)
        if (t < t1) a.lse[lse_h0] = (m + log2f(lt)) * 0.69314718055994530942f;
        const uint32_t o1_tm = lane_base + Geo::kColO + D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32], ow[32];
          ptx::tmem_ld32(o_tm + c * 32, ov);  // warp-collective: every lane loads, valid rows store
          if (two) ptx::tmem_ld32(o1_tm + c * 32, ow);
          ptx::tmem_wait_ld();
          if (t < t1) {
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int i0 = c8 * 8 + 2 * e;
                float x0 = __uint_as_float(ov[i0]) * g0, x1 = __uint_as_float(ov[i0 + 1]) * g0;
                if (two) {
                  x0 += __uint_as_float(ow[i0]) * g1;
                  x1 += __uint_as_float(ow[i0 + 1]) * g1;
                }
                w[e] = ptx::pack_bf16(x0, x1);
              }
              reinterpret_cast<uint4*>(orow)[c * 4 + c8] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// The sequence table of a packed batch (kernel_common.cuh) from cu_seqlens; one thread: the
// scan is over the sequences of one batch
__global__ void seq_table_kernel(const int32_t* cu, int n_seq, int total, int32_t* tab) {
  if (threadIdx.x != 0) return;
  int off = 0, prev_end = 0;
  for (int s = 0; s < n_seq; ++s) {
    const int st = imin(imax(cu[s], prev_end), total);
    const int en = imin(imax(cu[s + 1], st), total);
    tab[s] = off;
    tab[n_seq + 1 + s] = st;
    tab[2 * n_seq + 1 + s] = en - st;
    off += (en - st + kBM - 1) / kBM;
    prev_end = en;
  }
  tab[n_seq] = off;
}

template <int D>
cudaError_t launch_fwd_d(const FwdArgs& a, cudaStream_t s) {
  using Geo = FwdGeom<D>;
  auto kern = cowa_fwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::kSmem);
  if (e != cudaSuccess) return e;
  const int grp = a.Hq / a.Hkv;
  // packed batch: an upper bound on the q-tiles (sum of ceil(len/BM) <= total/BM + n_seq); the
  // sequence table is computed on the device first
  const long long nq = a.varlen ? packed_tiles_bound(a.total, a.n_seq) : (a.Nq + kBM - 1) / kBM;
  const long long nblk = nq * a.B * a.Hkv * ((grp + 1) / 2);
  if (nblk > 0x7fffffffLL) return cudaErrorInvalidValue;
  // the in-kernel register split assumes the compiled count equals the launch allocation
  static int regs_ok = -1;
  if (regs_ok < 0) {
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
    regs_ok = fa.numRegs == kRegsLaunch ? 1 : 0;
  }
  if (!regs_ok) return cudaErrorInvalidConfiguration;
  if (a.varlen) {
    if ((e = launch_seq_table(a.cu_seqlens, a.n_seq, a.total, a.seq_tab, s)) != cudaSuccess) return e;
  }
  kern<<<(unsigned)nblk, kFwdThreads, Geo::kSmem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_seq_table(const int32_t* cu_seqlens, int n_seq, int total, int32_t* tab, cudaStream_t s) {
  seq_table_kernel<<<1, 32, 0, s>>>(cu_seqlens, n_seq, total, tab);
  return cudaGetLastError();
}

cudaError_t launch_fwd(const FwdArgs& a, cudaStream_t s) {
  if (a.d == 64) return launch_fwd_d<64>(a, s);
  if (a.d == 128) return launch_fwd_d<128>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace cowa
