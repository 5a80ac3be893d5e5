/*
 * cowa.h -- C ABI of libcowa.so: CoWindow Attention (CoWA) on NVIDIA B200 (sm_100a).
 *
 * What the operation is.  CoWA ("CoWindow Attention: Full Causal Coverage Is a
 * Collective Property", Abstract; skillfed.io news summary of 2026-09-30,
 * paragraphs 2, 4, 6 and 7) is exact softmax attention under a mask that is a
 * function of positions and of the global KV-head index only.  For KV head g
 * (global index G = kv_head_base + g, H = h_kv_global KV heads in the layer)
 * a query at position t sees key s iff s <= t and one of:
 *   - s is in the shared prefix sink      [0, S)
 *   - s is in the shared near-diagonal    (t-L, t]        (L >= 1 keys incl. t)
 *   - s is in G's long-range interval     [b_p, b_{p+1}),  b_i = S + floor(i*(T-S)/H),
 *                                                          p = (G mod D) * (H/D)
 * With D = H the H intervals partition [S, T) and the union over KV heads is
 * the whole causal prefix; D < H repeats D distinct intervals over the heads
 * (the duplicated-window ablation, news summary paragraph 3).  L >= T gives
 * dense causal attention (the FullAttn comparison of the Abstract).  The
 * interval formula and the D < H slot rule are this library's reading: the
 * pages state the principle, not a formula.
 *
 * Query head h uses KV head g = h / (H_q / H_kv) (grouped-query attention).
 * Each head applies its softmax over its own visible keys (news summary,
 * paragraph 7).  Scores are softmax_scale * q.k; lse is the natural log of
 * the softmax denominator.
 *
 * Conventions for every entry point:
 *   - Tensors are bf16 in device memory, described by cowa_tensor: a pointer
 *     plus element strides for batch, position and head; the head dimension d
 *     is contiguous.  Pointers and every stride * 2 bytes must be multiples
 *     of 16 bytes (COWA_ERR_ALIGNMENT otherwise).  d must be 64 or 128 and
 *     H_q / H_kv at most 8 (COWA_ERR_UNSUPPORTED otherwise).
 *   - The caller owns every buffer, including the workspace; the library never
 *     allocates device memory on a call.  Query the workspace size with the
 *     matching *_workspace_size function; a smaller ws_bytes returns
 *     COWA_ERR_WORKSPACE.  The workspace must be 256-byte aligned.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Argument errors are returned before any
 *     launch; a failed launch returns COWA_ERR_CUDA.  No exception crosses the
 *     ABI.  Outputs are deterministic (no atomics in any result).
 *   - Device-side waits are bounded: a wait that runs out sets a status word
 *     in the workspace and the kernel returns; cowa_workspace_status() reads
 *     it (COWA_ERR_TIMEOUT).
 *   - The library keeps no mutable global state on the call path; calls on
 *     different streams with different workspaces may run concurrently.
 *   - cowa_fwd, cowa_bwd and cowa_decode never synchronise the host and allocate
 *     nothing, so a step made of them can be captured in a CUDA graph on a
 *     capturing stream and replayed (same bits as the calls made directly).
 *     cowa_workspace_status synchronises and is not capturable.
 */
#ifndef COWA_H
#define COWA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  COWA_OK = 0,
  COWA_ERR_INVALID_ARG = 1, /* bad shape, pattern or null pointer */
  COWA_ERR_UNSUPPORTED = 2, /* head dim not in {64, 128}, or more than 8 query heads per KV
                               head (H_q / H_kv > 8); the E4M3-cache calls need d = 128; a
                               compacted cache whose rows per head would exceed INT_MAX */
  COWA_ERR_ALIGNMENT = 3,   /* pointer or stride not 16-byte aligned */
  COWA_ERR_WORKSPACE = 4,   /* workspace too small or misaligned */
  COWA_ERR_CUDA = 5,        /* CUDA runtime/driver error at launch */
  COWA_ERR_TIMEOUT = 6,     /* a device-side bounded wait ran out */
  COWA_ERR_CHECK = 7        /* a device-side self-check of a COWA_DEBUG build failed (a planned
                               tile or cache row outside the call's tensors); the access was
                               skipped.  Release builds never report it. */
} cowa_status;

/* Window parameters of one attention layer.
 *   S  prefix-sink size, 0 <= S <= T
 *   L  near-diagonal width in keys (includes the query's own key), L >= 1
 *   T  declared span: the long-range region is [S, T); T >= S
 *   D  number of distinct long-range intervals, 1 <= D, D divides h_kv_global
 *   kv_head_base  global index of this call's KV head 0 (0 on one GPU; under KV-head
 *                 tensor parallelism a call covers consecutive global heads G0 .. and
 *                 passes G0: r * H / P on rank r for a contiguous split)
 *   h_kv_global   H, KV heads in the whole layer (0 means "= H_kv of the call")
 *   softmax_scale multiplier of q.k (<= 0 means 1/sqrt(d)) */
typedef struct {
  int32_t S, L, T, D;
  int32_t kv_head_base;
  int32_t h_kv_global;
  float softmax_scale;
} cowa_pattern;

/* A bf16 device tensor with the head dimension contiguous.  Element (b, t, h, :)
 * starts at ptr + b*stride_b + t*stride_t + h*stride_h (strides in elements).
 * [B, N, H, d] contiguous has stride_t = H*d, stride_h = d, stride_b = N*H*d. */
typedef struct {
  void* ptr;
  int64_t stride_b, stride_t, stride_h;
} cowa_tensor;

/* ---- forward (training / prefill self-attention at positions 0..N-1) ------------------
 * Inputs  q [B, N, H_q, d], k and v [B, N, H_kv, d]   (bf16, cowa_tensor strides)
 * Outputs o [B, N, H_q, d] bf16; lse fp32, contiguous [B, H_q, N] (natural log), saved
 *         for cowa_bwd.
 * H_q must be a multiple of H_kv.  N >= 1. */
size_t cowa_fwd_workspace_size(const cowa_pattern* pat, int B, int N, int H_q, int H_kv, int d);
cowa_status cowa_fwd(const cowa_pattern* pat, int B, int N, int H_q, int H_kv, int d,
                     cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o, float* lse,
                     void* ws, size_t ws_bytes, void* stream);

/* ---- chunked prefill: a block of queries against keys already written -------------------
 * The same operation for the query rows at positions q_offset .. q_offset+N_q-1 against the
 * keys at positions 0 .. N_k-1.  The pattern is position arithmetic applied the same way in
 * training and inference (skillfed.io news summary of CoWindow Attention, paragraph 2), so a later
 * block of queries over a cache sees exactly the keys it would see in one full pass.  cowa_fwd is this call with q_offset = 0, N_q = N_k = N.
 * Inputs  q [B, N_q, H_q, d]; k and v hold keys 0 .. N_k-1 (any cowa_tensor strides: a cache in
 *         [B, H_kv, T_cap, d] layout is stride_t = d, stride_h = T_cap*d, stride_b = H_kv*T_cap*d)
 * Outputs o [B, N_q, H_q, d] bf16; lse fp32 contiguous [B, H_q, N_q].
 * Requires q_offset >= 0 and q_offset + N_q <= N_k (the block's own keys are present), else
 * COWA_ERR_INVALID_ARG before any launch.  Workspace: cowa_fwd_workspace_size with N = N_q.
 * Ownership, ordering and errors as for cowa_fwd. */
cowa_status cowa_fwd_chunk(const cowa_pattern* pat, int B, int N_q, int N_k, int q_offset, int H_q, int H_kv,
                           int d, cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o, float* lse,
                           void* ws, size_t ws_bytes, void* stream);

/* ---- packed variable-length batch (forward) -------------------------------------------------
 * n_seq sequences packed along the token axis: sequence s is rows cu_seqlens[s] ..
 * cu_seqlens[s+1]-1 of q [total, H_q, d], k and v [total, H_kv, d] (cowa_tensor strides; stride_b
 * unused but validated), at positions 0 .. len_s-1 each; o [total, H_q, d]; lse fp32
 * contiguous [H_q, total].  Each sequence gets exactly cowa_fwd over its own rows.
 * cu_seqlens: device int32 [n_seq + 1], non-decreasing from 0 to total (the device clamps the
 * offsets so that sequences stay in order, disjoint and inside [0, total), so a malformed array
 * cannot make the kernel touch rows outside the tensors).  Workspace:
 * cowa_fwd_varlen_workspace_size (status word + a sequence table of tile offsets, first rows
 * and lengths, computed on the device in the same stream).  Errors as for cowa_fwd. */
size_t cowa_fwd_varlen_workspace_size(const cowa_pattern* pat, int n_seq, int total, int H_q, int H_kv, int d);
cowa_status cowa_fwd_varlen(const cowa_pattern* pat, int n_seq, int total, int H_q, int H_kv, int d,
                            const int32_t* cu_seqlens, cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o,
                            float* lse, void* ws, size_t ws_bytes, void* stream);

/* ---- backward ---------------------------------------------------------------------------
 * Gradients of sum(dO * O) for the forward above, from the saved o and lse.
 * Inputs  q, k, v, o, lse as produced/consumed by cowa_fwd; dO [B, N, H_q, d] bf16.
 * Outputs dq [B, N, H_q, d], dk and dv [B, N, H_kv, d], bf16 (fp32 accumulation).
 * The workspace holds fp32 row statistics (Delta = rowsum(dO * O) and lse * log2(e) per
 * query row) and, when a call has few KV heads, the query-range split of its long dK/dV key
 * tiles: a table of chunks and their fp32 partial dk, dv (128 KB per chunk at d = 128), summed in
 * chunk order so that results stay deterministic.  The size depends on the pattern and shape. */
size_t cowa_bwd_workspace_size(const cowa_pattern* pat, int B, int N, int H_q, int H_kv, int d);
cowa_status cowa_bwd(const cowa_pattern* pat, int B, int N, int H_q, int H_kv, int d,
                     cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o, const float* lse,
                     cowa_tensor dO, cowa_tensor dq, cowa_tensor dk, cowa_tensor dv,
                     void* ws, size_t ws_bytes, void* stream);

/* Backward in stages.  `stages` is a bit mask of COWA_BWD_PREPROCESS (Delta and lse*log2(e)
 * into the workspace), COWA_BWD_DKDV (dk, dv) and COWA_BWD_DQ (dq); cowa_bwd is all three.
 * The dK/dV and dQ stages read what the preprocess stage wrote into the same workspace, so it
 * must have completed first (stream order); they are independent of each other and may run on
 * two streams that both wait for the preprocess.  Arguments are those of cowa_bwd; a stage
 * outside the mask does not touch its outputs. */
#define COWA_BWD_PREPROCESS 1
#define COWA_BWD_DKDV 2
#define COWA_BWD_DQ 4
cowa_status cowa_bwd_stages(const cowa_pattern* pat, int B, int N, int H_q, int H_kv, int d,
                            cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o, const float* lse,
                            cowa_tensor dO, cowa_tensor dq, cowa_tensor dk, cowa_tensor dv,
                            int stages, void* ws, size_t ws_bytes, void* stream);

/* ---- backward of a packed variable-length batch ---------------------------------------------
 * The gradients of cowa_fwd_varlen: n_seq sequences packed along the token axis, sequence s at
 * rows cu_seqlens[s] .. cu_seqlens[s+1]-1 of q, o, dO, dq [total, H_q, d] and k, v, dk, dv
 * [total, H_kv, d] (cowa_tensor strides; stride_b unused but validated), each at positions
 * 0 .. len_s-1; lse fp32 contiguous [H_q, total] as cowa_fwd_varlen writes it.  Each sequence gets
 * exactly cowa_bwd over its own rows (the pattern is applied the same way in training and
 * inference, skillfed.io news summary of CoWindow Attention, paragraph 2).  The launches do not
 * grow with n_seq: one small kernel turns cu_seqlens into a sequence table in the workspace, then
 * each of the three backward kernels runs once over all sequences (a grid over the bound
 * total/128 + n_seq of 128-row tiles; every CTA finds its sequence in the table).
 * cu_seqlens: DEVICE int32 [n_seq + 1], non-decreasing from 0 to total.  The device clamps the
 * offsets so that sequences stay in order, disjoint and inside [0, total) (a malformed table
 * cannot reach memory outside the tensors; its sequences are then the clamped ones).
 * Workspace: cowa_bwd_varlen_workspace_size(pat, n_seq, total, ...), including room for the
 * key-tile split of the longest batch of `total` rows (the split is planned on the device from
 * the actual lengths).  Other errors as for cowa_bwd. */
size_t cowa_bwd_varlen_workspace_size(const cowa_pattern* pat, int n_seq, int total, int H_q, int H_kv, int d);
cowa_status cowa_bwd_varlen(const cowa_pattern* pat, int n_seq, int total, int H_q, int H_kv, int d,
                            const int32_t* cu_seqlens, cowa_tensor q, cowa_tensor k, cowa_tensor v, cowa_tensor o,
                            const float* lse, cowa_tensor dO, cowa_tensor dq, cowa_tensor dk, cowa_tensor dv,
                            void* ws, size_t ws_bytes, void* stream);

/* ---- decode (one new token per sequence, KV cache) -----------------------------------------
 * q_t    [B, H_q, d] bf16, contiguous.
 * k_cache, v_cache: cowa_tensor over [B, T_cap, H_kv, d]-indexed (b, t, h) with any strides
 *        (e.g. [B, H_kv, T_cap, d] has stride_h = T_cap*d, stride_t = d).
 * pos    device int32 [B]: the new token's position; its own K/V are already written at
 *        pos[b]; 0 <= pos[b] < T_cap (entries outside are clamped into range).
 * o      [B, H_q, d] bf16 contiguous; lse_or_null fp32 [B, H_q] or NULL.
 * Reads only the cache rows the pattern makes visible at pos[b]. */
size_t cowa_decode_workspace_size(const cowa_pattern* pat, int B, int H_q, int H_kv, int d, int T_cap);
cowa_status cowa_decode(const cowa_pattern* pat, int B, int H_q, int H_kv, int d, int T_cap,
                        const void* q_t, cowa_tensor k_cache, cowa_tensor v_cache,
                        const int32_t* pos, void* o, float* lse_or_null,
                        void* ws, size_t ws_bytes, void* stream);

/* ---- compacted decode cache -----------------------------------------------------------------
 * The abstract of "CoWindow Attention: Full Causal Coverage Is a Collective Property" reports a
 * 7.6x lower per-rank peak operator memory during decoding at 128K: a KV head never reads
 * positions outside its sink, band and own interval, so only those need to be kept.  This layout
 * keeps exactly that, per (b, KV head), as rows of d bf16 in one contiguous
 * [B, H_kv, rows, d] array (rows = cowa_compact_rows):
 *   sink       rows [0, S64)            position p < S at row p                  (S64 = S rounded up to 64)
 *   band ring  rows [S64, S64 + R)      position p at row S64 + (p mod R)        (R = L rounded up to 64, + 64)
 *   interval   rows [S64 + R, rows)     position p of the head's interval [lo, hi) at row
 *                                       S64 + R + p - (lo rounded down to 64)
 * At 128K (S=128, L=4096, T=131072, 8 KV heads) that is 20,736 rows per head instead of 131,072.
 * The ring holds the last R positions, so positions must be appended in order (build from a
 * prefill, then one append per decoded token).  The caller owns both arrays. */
/* Rows per (b, KV head) of the compacted cache; 0 for an invalid pattern or one whose compacted
 * layout would need more than INT_MAX rows (a band L near INT_MAX: use the full cache). */
int cowa_compact_rows(const cowa_pattern* pat, int H_kv);
/* Fills the compacted cache from the keys and values of positions 0..N-1 (k, v as in cowa_fwd:
 * [B, N, H_kv, d] with any cowa_tensor strides).  Rows no position maps to are left untouched. */
cowa_status cowa_compact_build(const cowa_pattern* pat, int B, int N, int H_kv, int d, cowa_tensor k, cowa_tensor v,
                               void* k_compact, void* v_compact, void* stream);
/* Appends the token at pos[b] (device int32 [B]; negative entries are skipped): k_new, v_new are
 * [B, H_kv, d] bf16 contiguous; the token goes to every region that holds its position. */
cowa_status cowa_compact_append(const cowa_pattern* pat, int B, int H_kv, int d, const void* k_new,
                                const void* v_new, const int32_t* pos, void* k_compact, void* v_compact,
                                void* stream);
/* Decode over the compacted cache: the same result as cowa_decode over the full cache holding the
 * same positions (pos[b] >= 0 is the new token, already appended; negative entries are clamped
 * to 0).  Errors as for cowa_decode. */
size_t cowa_decode_compact_workspace_size(const cowa_pattern* pat, int B, int H_q, int H_kv, int d);
cowa_status cowa_decode_compact(const cowa_pattern* pat, int B, int H_q, int H_kv, int d, const void* q_t,
                                const void* k_compact, const void* v_compact, const int32_t* pos, void* o,
                                float* lse_or_null, void* ws, size_t ws_bytes, void* stream);

/* ---- decode over an E4M3 (8-bit float) cache ------------------------------------------
 * cowa_decode with the cache stored as E4M3 codes (OCP 8-bit floating point, the E4M3FN variant:
 * bias 7, no infinities, largest magnitude 448): the attention uses k_scale * e4m3(code) for
 * keys and v_scale * e4m3(code) for values.  Halves the bytes a decode step reads.  Source: the
 * decode-memory argument of "Sliding Window Attention Beats Linear Attention ...", section
 * "Engineering Advantages" (decode throughput is set by the cache bytes read); the pages fix no
 * cache precision, so the format, one scale per cache tensor and round-to-nearest-even saturating
 * quantisation are this library's reading.
 * k_cache, v_cache: uint8 codes, cowa_tensor with strides in bytes (multiples of 16); d must be
 * 128 (COWA_ERR_UNSUPPORTED otherwise).  k_scale, v_scale finite and > 0.  q_t bf16 as for
 * cowa_decode (used in f16 by the kernel: bf16 values of magnitude 2^-14 .. 65504 are exact in
 * f16).  Workspace: cowa_decode_fp8_workspace_size.  Errors as for cowa_decode. */
size_t cowa_decode_fp8_workspace_size(const cowa_pattern* pat, int B, int H_q, int H_kv, int d, int T_cap);
cowa_status cowa_decode_fp8(const cowa_pattern* pat, int B, int H_q, int H_kv, int d, int T_cap, const void* q_t,
                            cowa_tensor k_cache, cowa_tensor v_cache, float k_scale, float v_scale,
                            const int32_t* pos, void* o, float* lse_or_null, void* ws, size_t ws_bytes,
                            void* stream);

/* The compacted per-head cache (see cowa_compact_build) holding E4M3 codes: build from a full
 * E4M3 cache (uint8 cowa_tensor, byte strides), append one token's codes (k_new, v_new uint8
 * [B, H_kv, 128] contiguous), decode with the scales of cowa_decode_fp8.  d = 128 only. */
cowa_status cowa_compact_build_fp8(const cowa_pattern* pat, int B, int N, int H_kv, int d, cowa_tensor k,
                                   cowa_tensor v, void* k_compact, void* v_compact, void* stream);
cowa_status cowa_compact_append_fp8(const cowa_pattern* pat, int B, int H_kv, int d, const void* k_new,
                                    const void* v_new, const int32_t* pos, void* k_compact, void* v_compact,
                                    void* stream);
size_t cowa_decode_fp8_compact_workspace_size(const cowa_pattern* pat, int B, int H_q, int H_kv, int d);
cowa_status cowa_decode_fp8_compact(const cowa_pattern* pat, int B, int H_q, int H_kv, int d, const void* q_t,
                                    const void* k_compact, const void* v_compact, float k_scale, float v_scale,
                                    const int32_t* pos, void* o, float* lse_or_null, void* ws, size_t ws_bytes,
                                    void* stream);

/* E4M3 codes of x / scale for n bf16 elements (device pointers; n a multiple of 8; x 16-byte and
 * codes 8-byte aligned): a float32 multiply by the float32 reciprocal of scale, then round to
 * nearest even, saturating at +-448.  Stream-ordered; COWA_ERR_INVALID_ARG / COWA_ERR_ALIGNMENT
 * before any launch. */
cowa_status cowa_quantize_e4m3(const void* x, void* codes, int64_t n, float scale, void* stream);

/* ---- decode without a caller workspace -----------------------------------------------------
 * This entry point has no counterpart on the CoWA pages; it is a convenience of this library for
 * callers that cannot allocate device memory (runtimes that reserve the whole memory pool up
 * front and forbid allocations on the serving path, or code that must not call cudaMalloc
 * because it would synchronize the device).
 *
 * Same inputs, outputs and result as cowa_decode, but no workspace argument: the split partials
 * and the status word live in a scratch array of COWA_DECODE_NOALLOC_SCRATCH_BYTES (8 MiB) that is
 * a static device variable of the library.  Every GPU that loads the library holds one copy of it
 * until the process exits.  The call allocates nothing (no cudaMalloc, no allocating library
 * routine).
 *   - The first call made with a given device current looks up the scratch address on that
 *     device (cudaGetSymbolAddress); make that first call before any stream capture.  The
 *     lookup is repeated only if the device's context has been replaced since (after a
 *     cudaDeviceReset the library's device variables live at new addresses).
 *   - Every call shares the one scratch array of its device and leaves its contents behind.
 *     The status word is cleared at the start of each call.  Calls that overlap on the GPU
 *     (e.g. on two streams without ordering between them) race on the scratch and give
 *     undefined results: order them on one stream or synchronize between them.
 *   - A configuration whose workspace (cowa_decode_workspace_size) exceeds the scratch size
 *     returns COWA_ERR_WORKSPACE without launching.  Other argument errors are those of
 *     cowa_decode.  A device-side timeout leaves its status in the library's scratch; read it
 *     with cowa_decode_noalloc_status. */
#define COWA_DECODE_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
cowa_status cowa_decode_noalloc(const cowa_pattern* pat, int B, int H_q, int H_kv, int d, int T_cap,
                                const void* q_t, cowa_tensor k_cache, cowa_tensor v_cache,
                                const int32_t* pos, void* o, float* lse_or_null, void* stream);
/* Synchronizes `stream`, then reads and clears the status word in the current device's
 * cowa_decode_noalloc scratch: COWA_OK, or COWA_ERR_TIMEOUT if a bounded device wait of an
 * earlier cowa_decode_noalloc call on this device ran out (COWA_ERR_CUDA if the stream failed).
 * Copies 4 bytes to the host and allocates nothing. */
cowa_status cowa_decode_noalloc_status(void* stream);

/* ---- status --------------------------------------------------------------------------------
 * Synchronizes `stream`, reads and clears the device status word in `ws` (the workspace of an
 * earlier call), and returns COWA_OK, COWA_ERR_TIMEOUT, or (debug builds) COWA_ERR_CHECK
 * (COWA_ERR_CUDA if the stream failed).  A debug build records the first failed self-check in
 * the two 32-bit words after the status word (a check code: 0x1nn forward, 0x2nn dK/dV, 0x3nn
 * dQ, 0x4nn decode; and the offending tile index or cache row); they are cleared with it. */
cowa_status cowa_workspace_status(void* ws, void* stream);
const char* cowa_status_string(cowa_status s);

/* ---- planner introspection (host; tests and tools) -----------------------------------------
 * The same integer code the kernels run.
 * cowa_visible_counts: out[g*N + t] = number of keys visible to position t for local KV head g
 *   (host memory, H_kv*N int64).
 * cowa_plan_debug: writes records of the tile plan for tile sizes BM x BN into host `out`:
 *   which = 0  forward plan, records (g, i, j, full) for every visited (q-tile i, kv-tile j)
 *   which = 1  backward plan, records (g, j, i, 0) for every q-tile i that sees kv-tile j
 *   which = 2  forward plan evaluated by a device kernel (same records in arbitrary order;
 *              `out` is still host memory, `dev_scratch` must be device memory of at least
 *              256 + cap*16 bytes; the call synchronizes the device)
 *   Records are 4 int32 each, in (g, outer, inner) order.  *n_written receives the number of
 *   records; if it exceeds cap, only cap are written and COWA_ERR_WORKSPACE is returned. */
cowa_status cowa_visible_counts(const cowa_pattern* pat, int H_kv, int N, int64_t* out);
cowa_status cowa_plan_debug(const cowa_pattern* pat, int H_kv, int N, int BM, int BN, int which,
                            int32_t* out, size_t cap, size_t* n_written, void* dev_scratch);

/* Test hook for the failure path every kernel's device-side waits share: launches one CTA that
 * waits on a barrier nothing arrives on.  After limit_ns (1 us .. 10 s) the wait gives up, the
 * timeout is recorded in the status word of `ws` (>= 256 bytes) and the kernel returns; a
 * following cowa_workspace_status(ws, stream) reports COWA_ERR_TIMEOUT and the context stays
 * usable.  No fault, trap or hang is involved. */
cowa_status cowa_debug_wait_timeout(void* ws, size_t ws_bytes, int64_t limit_ns, void* stream);

int cowa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* COWA_H */
