// Launchers shared between the C ABI (kvz_api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace kvz {

// Raise a kernel's dynamic shared-memory limit once per device (the launch
// paths call this before every launch; the attribute call itself is a host
// round trip worth skipping).  `bytes` is a constant of the kernel.
template <auto Kernel>
cudaError_t smem_limit_once(int bytes) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Pass 1 (row log-sum-exp) arguments.  Rows i in [i_begin, i_end) are
// computed; rows_pad = roundup(i_end - i_begin, 256) entries per (b, g) are
// written at lse2[(b*G + g)*ld + (i - i_begin)], padding rows set to +inf.
// A call scores B independent problems (query groups against context keys).
// Problem p reads context-key block (p % T) of head (p / T): T = 1 for the
// plain score, T = chunks per head for chunked scoring (the context-key map
// is 4-D: columns, rows of a block, block, head).
// Grid: one CTA per (head, group, 256-row block) unit, longest first; the
// last r units (the partial last wave) may each be split into `nsplit`
// CTAs over consecutive key-tile ranges.  CTA x < n_full computes unit x
// whole; CTA n_full + t computes part t % nsplit of unit n_full + t / nsplit
// and writes its rows' partial (reference m, sum of 2^(c2 s - m)) to
// part[t * 256 + row]; a merge kernel then combines the parts of each unit
// in order.
struct LseArgs {
  int B, G, T;
  int64_t n_c, n_in;
  float c2;                 // scale * log2(e)
  int64_t i_begin, i_end, rows_pad, ld;
  float* lse2;
  int32_t* status;
  int n_full;               // CTAs that compute a whole unit (set by launch_lse)
  int nsplit;               // parts per split unit, 1 = none (set by launch_lse)
  float2* part;             // [split CTAs][256] partial (reference, sum); null = no split
  int head_major;           // unit order: 0 = row block, then (head, group); 1 = head, then row block, then
                            // group (set by launch_lse)
  int wave;                 // CTAs resident at once (the SM count; 0 = unknown) (set by launch_lse)
};
// Scratch for split units: at most this many split CTAs, 256 rows of
// (max, sum) each.
constexpr int kLseMaxSplitCtas = 256;
constexpr size_t kLsePartBytes = static_cast<size_t>(kLseMaxSplitCtas) * 256 * 8;

// Pass 2 (context-key column max) arguments; lse2 as pass 1 wrote it.
struct ColArgs {
  int B, G, T;
  int64_t n_c;
  float c2;
  int64_t i_begin, rows_pad, ld;
  const float* lse2;
  float* S;                 // problem p writes S[(p / T) * ldS + (p % T) * s_block + j], j < n_c
  int64_t ldS, s_block;
  int n_kblk;               // key blocks per head (set by launch_colmax)
  int nsplit;               // row-tile ranges per (head, key block) (set by launch_colmax)
  int tiles_per_split;      // (set by launch_colmax)
  int32_t* status;
};

cudaError_t launch_lse(int d, const CUtensorMap& tmQ, const CUtensorMap& tmKc, const CUtensorMap& tmKi,
                       const LseArgs& a, cudaStream_t stream);
cudaError_t launch_colmax(int d, const CUtensorMap& tmQ, const CUtensorMap& tmKc, const ColArgs& a,
                          cudaStream_t stream);
cudaError_t launch_fill_f32(float* x, int64_t n, float v, cudaStream_t stream);

// Decode attention over the pruned cache (a device-built work list of equal
// splits; split-KV partials merged by a two-level tree).
constexpr int kDecGMax = 8;                 // grouped queries per KV head
// One CTA of the decode kernel: split sp of head b, tiles t0 .. t0+n-1 of
// the head's 64-key tiles; its partial is written at the item's index, the
// head's nsp partials at indices (index - sp) .. (index - sp + nsp - 1).
struct __align__(16) DecItem {
  int b, sp, t0, n;                         // n == 0: nothing to do
  int count, nsp;                           // the head's kept rows and splits
  long long off;                            // the head's first row in K_out / V_out
};
static_assert(sizeof(DecItem) == 32, "two 16-byte loads");

struct DecArgs {
  int B, G;
  int64_t n_c;                              // upper bound of counts[b]
  float c2;                                 // scale * log2(e)
  const uint16_t* q;                        // bf16 [B][G][d]
  const int32_t* counts;
  const int64_t* offsets;
  int n_items;                              // decode CTAs (grid.x): kDecWave + B bounds the splits
  DecItem* items;                           // [n_items], written by the plan kernel
  float2* part_ml;                          // [n_items][G] (running max, sum), base 2
  float* part_o;                            // [n_items][G][d]
  unsigned* done;                           // [B] split groups merged per head (zeroed by the plan kernel)
  unsigned* gdone;                          // [n_items] splits finished per group, at the group's first item
  int32_t* status;
};
constexpr int kDecWave = 148 * 3;           // about 1.5 waves of two decode CTAs per SM (best of 2, 3, 4, 6 per SM)
inline int decode_items(int64_t B) { return static_cast<int>(kDecWave + B); }
cudaError_t launch_decode(int d, const CUtensorMap& tmK, const CUtensorMap& tmV, const DecArgs& a, float* out,
                          float* lse2, cudaStream_t stream);

// Head scores (segmented max of S) and the CSR form of a head-level selection.
cudaError_t launch_head_max(const float* S, int64_t B, int64_t n_c, float* S_head, int32_t* status,
                            cudaStream_t stream);
cudaError_t launch_head_expand(const int32_t* kept, int64_t k, int64_t B, int64_t n_c, int32_t* idx,
                               int32_t* counts, int64_t* offsets, cudaStream_t stream);

// Selection.  Workspace layout is computed by select_workspace().
struct SelWorkspace {
  size_t bytes;
  size_t off_state, off_hist, off_cg, off_ce, off_eqb, off_cbase, off_head_eq, off_head_base;
};
SelWorkspace select_workspace(int64_t B, int64_t n_c, int mode);
cudaError_t launch_select(const float* S, int64_t B, int64_t n_c, int64_t n_protect, int mode, int64_t k,
                          int32_t* idx, int32_t* counts, int64_t* offsets, void* ws, const SelWorkspace& lay,
                          int32_t* status, cudaStream_t stream);
cudaError_t launch_select_dist_begin(const float* S, int64_t B, int64_t n_c, int64_t k, uint32_t* hist, void* ws,
                                     const SelWorkspace& lay, int32_t* status, cudaStream_t stream);
cudaError_t launch_select_dist_step(const float* S, int64_t B, int64_t n_c, int pass, uint32_t* hist,
                                    unsigned long long* eq_total, void* ws, const SelWorkspace& lay,
                                    int32_t* status, cudaStream_t stream);
cudaError_t launch_select_dist_finish(const float* S, int64_t B, int64_t n_c, const unsigned long long* eq_ranks,
                                      int rank, int32_t* idx, int32_t* counts, int64_t* offsets, void* ws,
                                      const SelWorkspace& lay, cudaStream_t stream);

// Compaction.
cudaError_t launch_compact_gather(const void* K, const void* V, int64_t B, int64_t n_c, int d,
                                  const int32_t* idx, const int64_t* offsets, const int64_t* out_offsets,
                                  void* K_out, void* V_out, int32_t* status, cudaStream_t stream);
// In place: `ws` holds B + B*ceil(n_c/chunk) uint32 (per-head chunk claims and
// per-chunk "sources read" flags); the launcher zeroes it on `stream`.
// `wait_ns` bounds each ordering wait (kInplaceWaitNs normally); when hold_b
// and hold_c are both >= 0, chunk hold_c of head hold_b never publishes that
// its sources were read, so a chunk waiting on it times out (test use only).
constexpr uint64_t kInplaceWaitNs = 1000ull * 1000ull * 1000ull;   // 1 s: far beyond any legitimate wait
cudaError_t launch_compact_inplace(void* K, void* V, int64_t B, int64_t n_c, int d, const int32_t* idx,
                                   const int32_t* counts, const int64_t* offsets, uint32_t* ws, int32_t* status,
                                   cudaStream_t stream, uint64_t wait_ns = kInplaceWaitNs, int64_t hold_b = -1,
                                   int64_t hold_c = -1);
size_t compact_workspace_bytes(int64_t B, int64_t n_c);
// Out-of-place compaction into int8 codes with one fp32 scale per row.
cudaError_t launch_compact_int8(const void* K, const void* V, int64_t B, int64_t n_c, int d, const int32_t* idx,
                                const int32_t* counts, const int64_t* offsets, const int64_t* out_offsets,
                                int8_t* Kq, int8_t* Vq, float* K_scale, float* V_scale, int32_t* status,
                                cudaStream_t stream);

}  // namespace kvz
