/*
 * kvz.h — C ABI of libkvz, a B200 (sm_100a) implementation of the KVzip
 * query-agnostic KV-cache compression hot path:
 *
 *   score   -> S_{l,h}[j], the maximum cross-attention a context key receives
 *              while the model reconstructs the context
 *   select  -> the kept key indices (top ratio, per head or across all heads)
 *   compact -> the kept K/V rows gathered, in key order, into a packed cache
 *
 * Definitions follow "KVzip: Query-Agnostic KV Cache Compression with Context
 * Reconstruction" (analysis report, §2.1 problem statement, §3.2 "KV importance
 * scoring" and its equation for S_{l,h}, §4.1 "eviction structure").  The
 * keep-count rounding m = floor(rho * n) follows the SelKV page (§3.1).
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates device memory; scratch space is passed in ("workspace")
 *     with its size given by the matching *_workspace_size() function.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and returns after enqueueing its kernels.
 *   - The return value reports errors the host can detect before launching:
 *     null pointers, unsupported head dimension, bad sizes, misalignment,
 *     aliasing, short workspace, and launch failures (KVZ_ERR_CUDA).
 *   - `d_status` (nullable) is a device int32 the kernels write when they
 *     detect an error on the device (first error wins; the library never
 *     clears it).  Read it after synchronising the stream.  Codes are the
 *     kvz_status values.
 *   - Tensors are row-major and densely packed.  bf16 tensors are IEEE
 *     bfloat16 bit patterns.  Every base pointer must be 16-byte aligned.
 *   - Head index b enumerates the B = L*H KV heads of a call layer-major
 *     (b = l*H + h), so a whole model's cache is one call.
 *   - Results are deterministic: identical inputs give bit-identical S, idx,
 *     counts, offsets and compacted rows, independent of scheduling (for
 *     the same call arguments on the same GPU model: pass 1's grid follows
 *     the call's sizes and the SM count, and fixes which work units of its
 *     partial last wave are split over key ranges).
 */
#ifndef KVZ_H_
#define KVZ_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvz_status {
  KVZ_OK = 0,
  KVZ_ERR_INVALID_ARG = 1,   /* null pointer, size out of range, bad mode/ratio/scale */
  KVZ_ERR_UNSUPPORTED = 2,   /* head dimension d not in {64, 128} */
  KVZ_ERR_ALIGNMENT = 3,     /* a base pointer or leading dimension is not 16-byte aligned */
  KVZ_ERR_WORKSPACE = 4,     /* workspace missing or smaller than *_workspace_size() */
  KVZ_ERR_CUDA = 5,          /* a CUDA runtime/driver call or kernel launch failed */
  KVZ_ERR_INVALID_SCORE = 6, /* device: a score was NaN or negative (valid: +0 .. +inf) */
  KVZ_ERR_TIMEOUT = 7        /* device: a bounded wait inside a kernel expired */
} kvz_status;

typedef enum kvz_mode {
  KVZ_PER_HEAD = 0,          /* keep floor(ratio*n_c) keys in every head */
  KVZ_GLOBAL = 1             /* keep floor(ratio*B*n_c) keys across all B heads */
} kvz_mode;

/* Library version, as 10000*major + 100*minor + patch. */
int kvz_version(void);

/* Human-readable name of a kvz_status value (static string, never NULL). */
const char* kvz_status_string(int status);

/* ------------------------------------------------------------------------ */
/* Scoring.                                                                  */
/*                                                                          */
/* KVzip §3.2: for each KV head b, the repeat-prompt + context input of      */
/* n_in = n_prompt + n_c tokens gives grouped queries Q_b (G x n_in x d) and */
/* keys K_b = [K_ctx_b ; K_in_b] ((n_c + n_in) x d).  With                   */
/*     A_b = Softmax(scale * Q_b K_b^T)  (per query row, causal),            */
/* sliced to the n_c context-key columns, the score is                      */
/*     S_b[j] = max over g < G, i < n_in of A_b[g, i, j],   j < n_c.         */
/* Causality: input position i (0-based, prompt first) sees every context   */
/* key and the input keys 0..i (its own position included).  The softmax    */
/* is normalised over all visible keys (context and input) before slicing.  */
/* The attention matrix is never materialised.                              */
/*                                                                          */
/* Layouts (bf16):  Q     [B][G][n_in][d]                                    */
/*                  K_ctx [B][n_c][d]                                        */
/*                  K_in  [B][n_in][d]                                       */
/* Output:          S     [B][n_c] fp32, values in [0, 1] up to rounding.    */
/*                                                                          */
/* Work is done in row chunks of `row_chunk` input positions (0 = all rows  */
/* in one pass; otherwise a positive multiple of 256).  Chunks merge by an   */
/* exact max; row_chunk changes the result only in float rounding (where    */
/* pass 1 splits its partial last wave, see kvz_score_lse2) and sets the    */
/* workspace size.  Limits: d in {64,128}; G >= 1; n_c, n_in >= 1;          */
/* B*G <= 2^31-1; n_c, n_in <= 2^31-1; scale finite and > 0.                */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace kvz_score needs: B*G*P*4 rounded up to 256, where P is
 * the row count of one chunk, min(row_chunk or n_in, n_in), rounded up to a
 * multiple of 256, plus kvz_score_lse2_workspace_size() for pass 1's split
 * last wave.  Returns 0 for invalid arguments. */
size_t kvz_score_workspace_size(int64_t B, int G, int64_t n_in, int64_t row_chunk);

/* Full scoring: zero-fills S, then for each row chunk runs pass 1 (row
 * log-sum-exp) and pass 2 (context-key column max).  `workspace` holds the
 * per-row base-2 log-sum-exp of the current chunk. */
kvz_status kvz_score(const void* Q, const void* K_ctx, const void* K_in,
                     int64_t B, int G, int64_t n_c, int64_t n_in, int d,
                     float scale, int64_t row_chunk, float* S,
                     void* workspace, size_t workspace_bytes,
                     int32_t* d_status, cudaStream_t stream);

/* Pass 1 alone, for input rows i in [i_begin, i_end):
 *     lse2[(b*G + g)*ld_lse2 + (i - i_begin)] =
 *         log2( sum over visible u of 2^(scale*log2(e) * <q_{b,g,i}, k_{b,u}>) )
 * Entries for padding rows, i in [i_end, i_begin + roundup(i_end-i_begin,256)),
 * are set to +inf (they then never contribute in pass 2).
 * Requires i_begin % 256 == 0, 0 <= i_begin < i_end <= n_in,
 * ld_lse2 >= roundup(i_end - i_begin, 256) and ld_lse2 % 4 == 0.
 * `workspace` (nullable, kvz_score_lse2_workspace_size() bytes, 16-byte
 * aligned) lets the work units of the grid's partial last wave be split
 * over key ranges and merged exactly (max, then rescaled sums, in a fixed
 * order), so the last wave fills the GPU; NULL computes every unit whole.
 * The two differ only in float rounding, well inside the score tolerance. */
size_t kvz_score_lse2_workspace_size(void);

kvz_status kvz_score_lse2(const void* Q, const void* K_ctx, const void* K_in,
                          int64_t B, int G, int64_t n_c, int64_t n_in, int d,
                          float scale, int64_t i_begin, int64_t i_end,
                          float* lse2, int64_t ld_lse2,
                          void* workspace, size_t workspace_bytes,
                          int32_t* d_status, cudaStream_t stream);

/* Pass 2 alone, for the rows whose lse2 pass 1 produced (same i_begin,
 * i_end, ld_lse2):
 *     S[b*n_c + j] = max(S[b*n_c + j],
 *                        max over g, i of 2^(scale*log2(e)*<q_{b,g,i}, k_{b,j}> - lse2[b,g,i]))
 * If `accumulate` is 0, S is first set to 0 (so the call computes the
 * chunk's score alone); otherwise S must already hold values >= +0 and the
 * result is merged by max (exact).  Context keys are visible to every input
 * row, so this pass has no mask and never reads K_in. */
kvz_status kvz_score_colmax(const void* Q, const void* K_ctx,
                            int64_t B, int G, int64_t n_c, int64_t n_in, int d,
                            float scale, int64_t i_begin, int64_t i_end,
                            const float* lse2, int64_t ld_lse2,
                            float* S, int accumulate,
                            int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Scoring without any caller-provided or allocated scratch memory.          */
/*                                                                          */
/* The KVzip paper has no counterpart to this call; it exists for callers   */
/* that cannot allocate device memory at the point where they score: an     */
/* engine whose memory pool owns the whole GPU and forbids further          */
/* cudaMalloc, a plugin or callback that has no access to the host          */
/* program's allocator, or a latency-critical path that must not risk the   */
/* implicit device synchronisation a cudaMalloc/cudaFree can cause.         */
/*                                                                          */
/* It computes exactly what kvz_score computes (same arguments minus the    */
/* workspace and row_chunk; Q, K_ctx, K_in and S are still the caller's).   */
/* The per-row log-sum-exp scratch is a fixed static device array of        */
/* KVZ_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads */
/* the library holds until the process exits.  Rows are processed in        */
/* chunks of as many 256-row blocks as fit in it, which does not change the */
/* result.                                                                  */
/*                                                                          */
/* - Returns KVZ_ERR_WORKSPACE, launching nothing, when one 256-row block   */
/*   of every head and group does not fit: B*G*256*4 > KVZ_NOALLOC_SCRATCH_ */
/*   BYTES (B*G > 8192).  Other argument errors are those of kvz_score.     */
/* - The first call in each CUDA context (a device's primary context, or a */
/*   context the caller made current; a device reset makes a new one)      */
/*   looks up the array's device address there (cudaGetSymbolAddress);     */
/*   make that first call before any stream capture that would contain a   */
/*   later one.                                                             */
/* - Every call on a device uses the same array and leaves its contents     */
/*   behind.  Nothing in it needs to start at zero (each call writes every  */
/*   entry before reading it), but calls that overlap on the GPU (two       */
/*   streams, or two host threads) race on it: keep them ordered, e.g. on   */
/*   one stream.                                                             */
/* ------------------------------------------------------------------------ */
#define KVZ_NOALLOC_SCRATCH_BYTES (8u << 20)

kvz_status kvz_score_noalloc(const void* Q, const void* K_ctx, const void* K_in,
                             int64_t B, int G, int64_t n_c, int64_t n_in, int d,
                             float scale, float* S,
                             int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Selection.                                                                */
/*                                                                          */
/* KVzip §4.1 keeps the r% highest-scoring KV pairs across all heads         */
/* (KVZ_GLOBAL); KVZ_PER_HEAD keeps r% of every head.  The keep count of a   */
/* segment of N scores is k = floor(ratio * N) computed in IEEE double.      */
/* The kept set is unique: the k largest scores, ties at the threshold       */
/* going to the lower flattened index (b*n_c + j).  Equivalently, it is the  */
/* first k entries of a stable sort by descending score.                     */
/*                                                                          */
/* Input:  S [B][n_c] fp32, every value in [+0, +inf] (+inf forces a key to  */
/*         be kept; -0 counts as +0).  A NaN or negative score sets          */
/*         KVZ_ERR_INVALID_SCORE in d_status and is treated as +0.           */
/* Output: counts[b]   number kept in head b (int32, B entries)              */
/*         offsets[b]  sum of counts[0..b-1] (int64, B+1 entries)            */
/*         idx[offsets[b] + p], p < counts[b]: kept key positions j of head  */
/*                     b, strictly ascending (int32).                        */
/* idx_capacity must be at least B*floor(ratio*n_c) (per head) or            */
/* floor(ratio*B*n_c) (global).  ratio must lie in [0, 1].                   */
/* ------------------------------------------------------------------------ */

/* Number kept from a segment of n scores: floor(ratio * n) in IEEE double. */
int64_t kvz_keep_count(int64_t n, double ratio);

/* Bytes of workspace kvz_select needs (0 for invalid arguments). */
size_t kvz_select_workspace_size(int64_t B, int64_t n_c, int mode);

kvz_status kvz_select(const float* S, int64_t B, int64_t n_c, double ratio,
                      int mode, int32_t* idx, int64_t idx_capacity,
                      int32_t* counts, int64_t* offsets,
                      void* workspace, size_t workspace_bytes,
                      int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Global selection with the heads of one context split over ranks          */
/* (KVzip §4.1: the r% budget spans all heads of all layers, so a context    */
/* whose layers sit on several GPUs needs one exchange per radix digit).     */
/*                                                                          */
/* The result equals kvz_select(KVZ_GLOBAL) on the concatenation of every    */
/* rank's S in rank order (rank r holds B_local heads that come after those */
/* of ranks 0..r-1): k = floor(ratio * B_total * n_c), ties to the lower     */
/* flattened index across ranks.  Each rank gets the CSR form of its own     */
/* heads (counts, offsets from 0, idx ascending per head).                   */
/*                                                                          */
/* Sequence on every rank, the caller doing the exchanges in between:       */
/*   kvz_select_dist_begin      writes this rank's first-digit histogram     */
/*   for pass 0, 1, 2:                                                       */
/*     (caller) hist <- sum of hist over ranks (in place, uint32 [2048])     */
/*     kvz_select_dist_step(pass)  picks the digit; for pass < 2 writes the  */
/*                                 next local histogram, for pass 2 writes   */
/*                                 eq_total[0] = keys of this rank equal to  */
/*                                 the threshold (uint64)                    */
/*   (caller) eq_ranks[r] <- eq_total of rank r, for every rank (all-gather) */
/*   kvz_select_dist_finish      writes counts, offsets and idx              */
/* Layout: S [B_local][n_c] fp32 (as kvz_select); hist: 2048 uint32 of      */
/* device memory, 16-byte aligned, owned by the caller and left zeroed by   */
/* the last step; eq_total: one uint64; eq_ranks: world uint64.  All calls  */
/* take the same workspace (kvz_select_dist_workspace_size bytes, 16-byte   */
/* aligned), which carries the state from one call to the next.             */
/* idx_capacity >= min(k, B_local * n_c).  B_total >= B_local, 0 <= rank,  */
/* B_total * n_c < 2^32.                                                    */
/* Errors as kvz_select; every rank must make the same calls.               */
/* ------------------------------------------------------------------------ */
size_t kvz_select_dist_workspace_size(int64_t B_local, int64_t n_c);

kvz_status kvz_select_dist_begin(const float* S, int64_t B_local, int64_t n_c, int64_t B_total,
                                 double ratio, uint32_t* hist, void* workspace,
                                 size_t workspace_bytes, int32_t* d_status, cudaStream_t stream);

kvz_status kvz_select_dist_step(const float* S, int64_t B_local, int64_t n_c, int pass,
                                uint32_t* hist, uint64_t* eq_total, void* workspace,
                                size_t workspace_bytes, int32_t* d_status, cudaStream_t stream);

kvz_status kvz_select_dist_finish(const float* S, int64_t B_local, int64_t n_c, int64_t B_total,
                                  double ratio, const uint64_t* eq_ranks, int rank,
                                  int32_t* idx, int64_t idx_capacity, int32_t* counts,
                                  int64_t* offsets, void* workspace, size_t workspace_bytes,
                                  int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Context-independent head scores and head-level eviction (KVzip §4.2,     */
/* "context-independent eviction": one static importance per head, the pair  */
/* scores aggregated by a max along the sequence).                           */
/*                                                                          */
/* kvz_head_score: S_head[b] = max_j S[b][j].  S [B][n_c] fp32 (>= 0),      */
/*   S_head [B] fp32 (overwritten).  NaN or negative scores are reported    */
/*   (KVZ_ERR_INVALID_SCORE) and counted as +0.                              */
/* kvz_select_heads: keep the floor(ratio * B) heads with the highest head   */
/*   score (ties to the lower head index); a kept head keeps all its n_c     */
/*   pairs, an evicted head none.  Output in kvz_select's CSR form, ready    */
/*   for kvz_compact: counts[b] in {0, n_c}, offsets [B+1], idx = 0..n_c-1   */
/*   for each kept head in head order (capacity floor(ratio*B) * n_c).       */
/*   Workspace: kvz_select_heads_workspace_size(B) bytes.  B <= 65535.       */
/* ------------------------------------------------------------------------ */
kvz_status kvz_head_score(const float* S, int64_t B, int64_t n_c, float* S_head, int32_t* d_status,
                          cudaStream_t stream);

size_t kvz_select_heads_workspace_size(int64_t B);

kvz_status kvz_select_heads(const float* S_head, int64_t B, int64_t n_c, double ratio, int32_t* idx,
                            int64_t idx_capacity, int32_t* counts, int64_t* offsets, void* workspace,
                            size_t workspace_bytes, int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Selection with a protected prefix (KVzip §4.1: the initial system         */
/* prompt's KV pairs are kept intact).                                       */
/*                                                                          */
/* As kvz_select, except that positions j < n_protect of every head are      */
/* always kept and the ratio applies to the other positions: per head        */
/* n_protect + floor(ratio * (n_c - n_protect)) kept; globally               */
/* B * n_protect + floor(ratio * B * (n_c - n_protect)).  Ties among the     */
/* unprotected positions go to the lower flattened index.  idx capacity as   */
/* those totals (times B per head).  0 <= n_protect <= n_c; same workspace   */
/* as kvz_select.                                                            */
/* ------------------------------------------------------------------------ */
kvz_status kvz_select_protected(const float* S, int64_t B, int64_t n_c, double ratio, int mode,
                                int64_t n_protect, int32_t* idx, int64_t idx_capacity, int32_t* counts,
                                int64_t* offsets, void* workspace, size_t workspace_bytes,
                                int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Compaction into an int8 cache (KVzip §4.2, "KV quantization": the pruned  */
/* cache composes with a quantised one).                                     */
/*                                                                          */
/* Out-of-place kvz_compact whose destination rows are symmetric int8 codes */
/* with one fp32 scale per row: with a = max |x| over the row's d values,   */
/* scale = a / 127 and code = rint(x * (127 / a)) clamped to [-127, 127]    */
/* (round half to even; single IEEE float32 operations in that order); a    */
/* row of zeros gets code 0 and scale 0.  x ~= code * scale.                */
/* Layout: Kq, Vq [rows][d] int8 (16-byte aligned); K_scale, V_scale [rows] */
/* fp32; row of head b's p-th kept key = (out_offsets ? out_offsets[b] :    */
/* offsets[b]) + p.  Device-detected errors as kvz_compact.                 */
/* ------------------------------------------------------------------------ */
kvz_status kvz_compact_int8(const void* K, const void* V, int64_t B, int64_t n_c, int d,
                            const int32_t* idx, const int32_t* counts, const int64_t* offsets,
                            const int64_t* out_offsets, int8_t* Kq, int8_t* Vq, float* K_scale,
                            float* V_scale, int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Compaction.                                                               */
/*                                                                          */
/* KVzip §2.1: the pruned cache K_p is a subset of the full cache K_c that   */
/* is reused for every later query.  For p < counts[b]:                      */
/*     K_out[dst_b + p] = K[b*n_c + idx[offsets[b] + p]]   (rows of d bf16)  */
/*     V_out[dst_b + p] = V[b*n_c + idx[offsets[b] + p]]                     */
/* Key order is preserved because idx is ascending within a head.            */
/*                                                                          */
/* Out of place (K_out != K): dst_b = out_offsets[b] if out_offsets is not   */
/*   NULL, else offsets[b] (a packed CSR cache).  K_out/V_out must hold every */
/*   destination row and must not overlap K or V.  No workspace is needed   */
/*   (workspace may be NULL).                                                */
/* In place (K_out == K and V_out == V): dst_b = b*n_c, i.e. each head's     */
/*   kept rows are packed to the front of its own region; rows at and after  */
/*   counts[b] keep stale data.  out_offsets must be NULL.  Needs a          */
/*   workspace of kvz_compact_workspace_size(B, n_c) bytes (chunk claims,   */
/*   "sources read" flags and each chunk's first reader slot, all rebuilt by */
/*   the call).  Safe because a kept row never moves to a higher position: a */
/*   chunk of slots writes only after every earlier chunk that reads one of  */
/*   its destination rows has read (a bounded wait; if it ever expires,      */
/*   KVZ_ERR_TIMEOUT is set and that head's remaining chunks are left        */
/*   unwritten).                                                             */
/* Layout: K, V [B][n_c][d] bf16; idx/counts/offsets as kvz_select writes.   */
/* Device-detected errors: idx out of [0, n_c), or idx[p] < p in place       */
/* (not ascending) -> KVZ_ERR_INVALID_ARG, the offending slot is skipped.    */
/* ------------------------------------------------------------------------ */
size_t kvz_compact_workspace_size(int64_t B, int64_t n_c);

kvz_status kvz_compact(const void* K, const void* V, int64_t B, int64_t n_c,
                       int d, const int32_t* idx, const int32_t* counts,
                       const int64_t* offsets, const int64_t* out_offsets,
                       void* K_out, void* V_out,
                       void* workspace, size_t workspace_bytes,
                       int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Decode attention over the pruned cache (KVzip §2.1: every later query     */
/* reads the pruned cache in place of the full one).                         */
/*                                                                          */
/* One decode step for each KV head b with the G grouped queries of the new  */
/* token: out[b][g] = sum_j softmax_j(scale * <q[b][g], k_j>) v_j over head  */
/* b's kept rows j (rows offsets[b] .. offsets[b] + counts[b] of K_out and   */
/* V_out, as kvz_compact packs them).  lse2[b][g] (optional) is the base-2   */
/* log of the softmax denominator.  A head with counts[b] == 0 gives out = 0 */
/* and lse2 = -inf.                                                          */
/* Layout: q [B][G][d] bf16; K_out, V_out [n_rows][d] bf16; out [B][G][d]    */
/* fp32; lse2 [B][G] fp32.  n_c bounds every counts[b]; a count outside     */
/* [0, n_c] is reported (KVZ_ERR_INVALID_ARG in d_status) and that head is   */
/* skipped.  The rows are split over CTAs on the device from the counts, at  */
/* the same number of rows per CTA for every head, so uneven heads (global   */
/* selection) cost no more than even ones.                                  */
/* Limits: d in {64, 128}; 1 <= G <= 8 (else KVZ_ERR_UNSUPPORTED);          */
/* B <= 65535.  Workspace: kvz_decode_workspace_size(B, G, n_c, d) bytes,    */
/* 256-byte aligned (the work list and per-split partial results).           */
/* ------------------------------------------------------------------------ */
size_t kvz_decode_workspace_size(int64_t B, int G, int64_t n_c, int d);

kvz_status kvz_decode(const void* q, const void* K_out, const void* V_out, int64_t n_rows,
                      const int32_t* counts, const int64_t* offsets, int64_t B, int G, int64_t n_c,
                      int d, float scale, float* out, float* lse2, void* workspace,
                      size_t workspace_bytes, int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Chunked scoring (KVzip §3.4, "chunk-based scoring").                      */
/*                                                                          */
/* The context is cut into chunks of m tokens (the last one is n_c mod m     */
/* tokens when m does not divide n_c).  Chunk t, context positions           */
/* [c0, c1), m_t = c1 - c0, is appended to the repeat prompt and             */
/* reconstructed on its own: its input has n_in_t = n_prompt + m_t tokens    */
/* with their own grouped queries and input keys, and its rows see only the  */
/* chunk's m_t cache keys K_ctx[c0:c1] plus the input keys (causally), each  */
/* row normalised over exactly those keys: an n_in_t x (m_t + n_in_t)        */
/* attention matrix per chunk.  S[c0 + j] is the max over (g, i) of chunk    */
/* t's row values on its cache key j.  Cost is linear in n_c.                */
/* Layout (bf16; T = n_c / m full chunks, m_last = n_c % m):                 */
/*   Q         [B][T][G][n_prompt + m][d]       (NULL when T == 0)           */
/*   Q_tail    [B][G][n_prompt + m_last][d]     (NULL when m_last == 0)      */
/*   K_in      [B][T][n_prompt + m][d],  K_in_tail [B][n_prompt + m_last][d] */
/*   K_ctx     [B][n_c][d];  S [B][n_c] fp32 (overwritten).                  */
/* Workspace: kvz_score_chunked_workspace_size(...) bytes (per-row lse2).    */
/* Limits as kvz_score; n_prompt >= 0, m >= 1.                               */
/* ------------------------------------------------------------------------ */
size_t kvz_score_chunked_workspace_size(int64_t B, int G, int64_t n_c, int64_t n_prompt, int64_t m);

kvz_status kvz_score_chunked(const void* Q, const void* Q_tail, const void* K_ctx, const void* K_in,
                             const void* K_in_tail, int64_t B, int G, int64_t n_c, int64_t n_prompt,
                             int64_t m, int d, float scale, float* S, void* workspace,
                             size_t workspace_bytes, int32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* End to end from host memory.                                              */
/*                                                                          */
/* The whole path of one context (kvz_score, then kvz_select, then an        */
/* out-of-place kvz_compact into a packed cache) with inputs read from and   */
/* results written to HOST buffers, for callers whose KV cache and queries   */
/* come from the host.  The host->device copies go by head chunks (at most   */
/* 8) on `copy_stream`; each chunk is scored on `stream` as soon as it has   */
/* landed, so the copies overlap the scoring.  V is copied last (only the    */
/* compaction reads it).  The results come back on `stream`: h_counts[B],    */
/* h_offsets[B+1], h_idx[kept], hK_out[kept][d], hV_out[kept][d], where      */
/* kept = B*floor(ratio*n_c) per head or floor(ratio*B*n_c) globally.  The   */
/* call is asynchronous: the host outputs are valid once `stream` has        */
/* finished; page-locked host buffers are needed for the copies to overlap  */
/* (pageable ones work, serialised).  `stream` may equal `copy_stream`      */
/* (no overlap).  The pages have no counterpart; it composes the three      */
/* calls above.                                                              */
/* Layout: hQ [B][G][n_in][d], hK_ctx and hV [B][n_c][d], hK_in [B][n_in][d] */
/* bf16.  `workspace` is a device buffer of                                  */
/* kvz_compress_host_workspace_size(...) bytes, 256-byte aligned: device    */
/* copies of the inputs and outputs plus the scratch of the three calls.     */
/* Errors: as the three calls, plus KVZ_ERR_INVALID_ARG for a null host      */
/* pointer or idx_capacity < kept.                                           */
/* ------------------------------------------------------------------------ */
size_t kvz_compress_host_workspace_size(int64_t B, int G, int64_t n_c, int64_t n_in, int d, double ratio,
                                        int mode);

kvz_status kvz_compress_host(const void* hQ, const void* hK_ctx, const void* hK_in, const void* hV,
                             int64_t B, int G, int64_t n_c, int64_t n_in, int d, float scale,
                             double ratio, int mode, int32_t* h_idx, int64_t idx_capacity,
                             int32_t* h_counts, int64_t* h_offsets, void* hK_out, void* hV_out,
                             void* workspace, size_t workspace_bytes, int32_t* d_status,
                             cudaStream_t stream, cudaStream_t copy_stream);

#ifdef __cplusplus
}
#endif

#endif /* KVZ_H_ */
