// cowa_internal.h -- declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/cowa.h"
#include "cowa_pattern.h"

namespace cowa {

// Every workspace starts with a 256-byte header whose first word is the device
// status (0 = ok, bit 0 = a bounded wait ran out).  Kernel data follows.
constexpr size_t kWsHeader = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Encode a 4-D bf16 tensor map over (d, t, h, b) with a box of (64, box_rows, 1, 1)
// and 128-byte swizzle.  Returns false if the driver rejects it.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int d, int n_t, int n_h, int n_b, int64_t stride_t,
                    int64_t stride_h, int64_t stride_b, int box_rows);

// ---- decode ----
// Compacted per-head decode cache: only what decode can see, rows of d bf16 per (b, KV head):
//   sink      rows [0, S64)           position p < S at row p
//   band ring rows [S64, S64 + R)     position p at row S64 + (p mod R); R = round64(L) + 64
//   interval  rows [IB, IB + W)       position p of the head's interval [lo, hi) at row
//                                     IB + p - round_down64(lo); IB = S64 + R
// Every 64-aligned block of positions maps to 64 consecutive rows of one region.
struct CompactGeom {
  int S64, R, IB, W, rows;
};
CompactGeom compact_geom(const Pat& p);

struct DecodeArgs {
  Pat pat;
  int B, Hq, Hkv, d, T_cap;
  const void* q_t;
  const int32_t* pos;
  void* o;
  float* lse;        // may be null
  float* partials;   // [B, Hq, n_split, d + 2]
  uint32_t* status;
  int chunk;         // tokens per split
  int n_split;
  float scale_log2;  // softmax scale * log2(e)
  // compacted cache (tm_k / tm_v over [B, H_kv, rows, d]): 0 = full cache indexed by position
  int compact;
  CompactGeom cg;
  // E4M3 cache (tm_k / tm_v over uint8 codes): scale_log2 then includes k_scale, and the
  // partial outputs are multiplied by v_scale
  int kv8;
  float v_scale;
  CUtensorMap tm_k, tm_v;
};
int decode_chunk_tokens(const Pat& p, int B, int Hkv, int T_cap);
int decode_num_splits(const Pat& p, int T_cap, int chunk, bool compact = false);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_quantize_e4m3(const void* x, void* q, int64_t n, float inv_scale, cudaStream_t s);
cudaError_t launch_compact_append(const Pat& p, int B, int Hkv, int d, const void* k_new, const void* v_new,
                                  const int32_t* pos, void* kc, void* vc, cudaStream_t s);
cudaError_t launch_compact_build(const Pat& p, int B, int N, int Hkv, int d, const void* k, int64_t ksb, int64_t kst,
                                 int64_t ksh, const void* v, int64_t vsb, int64_t vst, int64_t vsh, void* kc, void* vc,
                                 cudaStream_t s);

// ---- forward ----
struct FwdArgs {
  Pat pat;
  int B, Hq, Hkv, d;
  int Nq, Nk, q_off;  // query rows q_off .. q_off+Nq-1 (absolute positions) against keys 0 .. Nk-1
  // packed variable-length batch (varlen != 0): sequence s holds rows cu_seqlens[s] ..
  // cu_seqlens[s+1]-1 of q, k, v, o (B = 1) at positions 0..; seq_tab is the sequence table
  // of kernel_common.cuh (tile offsets, first rows, lengths), written first on the device
  int varlen, n_seq, total;
  const int32_t* cu_seqlens;
  int32_t* seq_tab;
  void* o;
  int64_t o_sb, o_st, o_sh;
  float* lse;
  uint32_t* status;
  float scale_log2;
  CUtensorMap tm_q, tm_k, tm_v;
};
cudaError_t launch_fwd(const FwdArgs& a, cudaStream_t s);

// ---- packed variable-length batches ----
// Bytes of the sequence table (3 n_seq + 1 int32, 256-aligned) and the kernel that writes it
// from cu_seqlens (device int32 [n_seq + 1]).
inline size_t seq_table_bytes(int n_seq) { return align_up((size_t)(3 * n_seq + 1) * sizeof(int32_t), 256); }
cudaError_t launch_seq_table(const int32_t* cu_seqlens, int n_seq, int total, int32_t* tab, cudaStream_t s);
// upper bound on the 128-row tiles of a packed batch: sum of ceil(len / 128) <= total / 128 + n_seq
inline long long packed_tiles_bound(int total, int n_seq) { return (long long)total / 128 + n_seq; }

// ---- backward ----
struct BwdArgs {
  Pat pat;
  int B, N, Hq, Hkv, d;
  // packed variable-length batch (varlen != 0, B = 1): the sequences of seq_tab (see
  // kernel_common.cuh) on a token axis of `total` rows; N is then unused
  int varlen, n_seq, total;
  int32_t* seq_tab;
  int lse_ld;        // row stride of lse: N ([B, Hq, N]) or total (packed: [Hq, total])
  const void* o; int64_t o_sb, o_st, o_sh;
  const void* dO; int64_t do_sb, do_st, do_sh;
  const float* lse;
  void* dq; int64_t dq_sb, dq_st, dq_sh;
  void* dk; int64_t dk_sb, dk_st, dk_sh;
  void* dv; int64_t dv_sb, dv_st, dv_sh;
  float* delta;      // [B, Hq, N_pad] fp32 workspace: rowsum(dO * O), 0 on padded rows
  float* lse2;       // [B, Hq, N_pad] fp32 workspace: lse * log2(e), +inf on padded rows
  int N_pad;         // N rounded up to a whole number of 128-row tiles (packed: 128 x the
                     // tile bound, each sequence's rows starting at its own tile)
  uint32_t* status;
  float scale;       // softmax scale
  float scale_log2;  // softmax scale * log2(e)
  // Query-range split of long dK/dV key tiles (kv_chunk > 0; see kv_split_plan): the grid
  // starts with n_split CTAs, one per chunk kv_tab[e] = {key tile, KV head, batch, chunk} of
  // kv_chunk query tiles; each writes fp32 partial dV, dK ([2][128][d]) to kv_part + e*2*128*d,
  // and a reduction kernel sums a tile's chunks in chunk order.  The unsplit CTA of such a tile
  // leaves at once.  Packed batches do not split (kv_chunk = 0).
  // A packed batch plans its split on the device (the host cannot see the lengths): n_split is
  // then a capacity, unused table slots hold chunk -1, and kv_flag[g * kv_bound + packed tile]
  // says which key tiles were split (a tile that does not fit the capacity stays whole).
  int kv_chunk, n_split;
  int4* kv_tab;
  float* kv_part;
  int32_t* kv_flag;
  int kv_bound;
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
};
struct KvSplit {
  int chunk;             // query tiles per chunk; 0: no key tile is split
  long long n_entries;   // chunks over all split key tiles and batch elements
};
KvSplit kv_split_plan(const Pat& p, int B, int N, int Hq, int Hkv);
// workspace after the header: Delta, lse2, then (split calls) the chunk table and partials
size_t bwd_workspace_bytes(const Pat& p, int B, int N, int Hq, int Hkv, int d);
cudaError_t launch_bwd(const BwdArgs& a, int stages, cudaStream_t s);

// ---- bounded-wait probe ----
cudaError_t launch_wait_timeout_probe(uint32_t* status, unsigned long long limit_ns, cudaStream_t s);

// ---- planner debug kernel ----
cudaError_t launch_plan_debug(const Pat& p, int Hkv, int N, int BM, int BN, int32_t* dev_out, size_t cap,
                              unsigned long long* dev_count, cudaStream_t s);

}  // namespace cowa
