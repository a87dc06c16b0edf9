// Top-ratio selection of KV pairs by score (KVzip analysis report, §4.1
// "eviction structure": keep the r% highest-scoring pairs across all heads,
// or per head), with the keep count floor(ratio * n) (SelKV page, §3.1).
//
// The kept set is the k largest scores with ties at the threshold going to
// the lower flattened index.  Scores are non-negative fp32, so their bit
// patterns (with -0 folded onto +0) order exactly like their values and the
// k-th largest bit pattern T is found by a three-digit radix select
// (11 + 11 + 10 bits, one histogram pass each).  With GT = #(s > T) and
// r_t = k - GT ties to take, a key is kept iff s > T, or s == T and fewer
// than r_t equal keys precede it in flattened order.  Output positions come
// from exclusive scans, so idx is ascending within each head.
#include <cuda_runtime.h>

#include <cstdint>

#include "kvz.h"
#include "kvz_internal.h"

namespace kvz {

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelItems = 16;
constexpr int kSelChunk = kSelThreads * kSelItems;  // scores per chunk (one CTA)
constexpr int kBins = 2048;

struct SelState {
  uint32_t prefix;               // bits of T fixed so far
  uint32_t mask;                 // which bits of prefix are fixed
  unsigned long long k_rem;      // keys still to take among those matching prefix
  int done;                      // 1 when nothing is selected (k == 0)
  int pad;
};

__device__ __forceinline__ void report_err(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Order-preserving 32-bit key of a valid score; NaN and negative scores are
// reported and ranked as +0.
__device__ __forceinline__ uint32_t score_key(float s, int32_t* status) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;
  if (u > 0x7F800000u) {
    report_err(status, KVZ_ERR_INVALID_SCORE);
    u = 0u;
  }
  return u;
}

// Key of position j of a head: the first n_protect positions rank above
// every score (their key exceeds +inf's pattern), the rest as score_key.
__device__ __forceinline__ uint32_t select_key(const float* src, int64_t j, int64_t n_protect, int32_t* status) {
  return j < n_protect ? 0xFFFFFFFFu : score_key(__ldg(src + j), status);
}

__device__ __forceinline__ int digit_shift(int pass) { return pass == 0 ? 21 : (pass == 1 ? 10 : 0); }
__device__ __forceinline__ uint32_t digit_mask(int pass) { return pass == 2 ? 0x3FFu : 0x7FFu; }

// Inclusive sum over the block (blockDim.x a multiple of 32, <= 1024).
template <typename T>
__device__ __forceinline__ T block_inclusive_sum(T v, T* warp_buf) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) warp_buf[w] = v;
  __syncthreads();
  if (w == 0) {
    T t = lane < nw ? warp_buf[lane] : T(0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      T y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) warp_buf[lane] = t;
  }
  __syncthreads();
  if (w > 0) v += warp_buf[w - 1];
  __syncthreads();   // warp_buf may be reused by the caller
  return v;
}

__global__ void sel_init(SelState* st, int nseg, unsigned long long k, uint32_t* hist) {
  const int64_t tid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t e = tid; e < static_cast<int64_t>(nseg) * kBins; e += stride) hist[e] = 0u;
  for (int64_t e = tid; e < nseg; e += stride) {
    SelState s;
    s.pad = 0;
    if (k == 0ull) {
      s.prefix = 0xFFFFFFFFu;        // no key equals or exceeds it
      s.mask = 0xFFFFFFFFu;
      s.k_rem = 0ull;
      s.done = 1;
    } else {
      s.prefix = 0u;
      s.mask = 0u;
      s.k_rem = k;
      s.done = 0;
    }
    st[e] = s;
  }
}

// Histogram of the current digit over keys that match the prefix.
__global__ void __launch_bounds__(kSelThreads) sel_hist(const float* S, int64_t n_c, int64_t n_protect, int mode,
                                                        int pass, const SelState* st, uint32_t* hist,
                                                        int32_t* status) {
  __shared__ uint32_t h[kBins];
  const int b = blockIdx.y;
  const int seg = mode == KVZ_GLOBAL ? 0 : b;
  const SelState s = st[seg];
  if (s.done) return;
  for (int e = threadIdx.x; e < kBins; e += kSelThreads) h[e] = 0u;
  __syncthreads();
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kSelChunk;
  const int lim = static_cast<int>(min(static_cast<int64_t>(kSelChunk), n_c - c0));
  const float* src = S + static_cast<int64_t>(b) * n_c + c0;
  const int sh = digit_shift(pass);
  const uint32_t dm = digit_mask(pass);
  int32_t* st_ptr = pass == 0 ? status : nullptr;
  for (int e = threadIdx.x; e < lim; e += kSelThreads) {
    const uint32_t key = select_key(src - c0, c0 + e, n_protect, st_ptr);
    if ((key & s.mask) == s.prefix) atomicAdd(&h[(key >> sh) & dm], 1u);
  }
  __syncthreads();
  uint32_t* gh = hist + static_cast<int64_t>(seg) * kBins;
  for (int e = threadIdx.x; e < kBins; e += kSelThreads)
    if (h[e] != 0u) atomicAdd(&gh[e], h[e]);
}

// Pick the digit holding the k_rem-th largest key; clear the histogram.
__global__ void __launch_bounds__(1024) sel_pick(int pass, SelState* st, uint32_t* hist) {
  __shared__ unsigned long long wbuf[32];
  const int seg = blockIdx.x;
  const SelState s = st[seg];
  if (s.done) return;
  const int nb = pass == 2 ? 1024 : 2048;
  uint32_t* gh = hist + static_cast<int64_t>(seg) * kBins;
  // position x = 0 is the highest digit; thread t owns positions 2t, 2t+1
  const int x0 = 2 * static_cast<int>(threadIdx.x);
  const unsigned long long c0 = x0 < nb ? gh[nb - 1 - x0] : 0ull;
  const unsigned long long c1 = x0 + 1 < nb ? gh[nb - 2 - x0] : 0ull;
  const unsigned long long incl = block_inclusive_sum<unsigned long long>(c0 + c1, wbuf);
  const unsigned long long excl = incl - c0 - c1;
  gh[x0] = 0u;
  gh[x0 + 1] = 0u;
  const unsigned long long k_rem = s.k_rem;
  int x = -1;
  unsigned long long above = 0ull;
  if (excl < k_rem && excl + c0 >= k_rem) {
    x = x0;
    above = excl;
  } else if (excl + c0 < k_rem && excl + c0 + c1 >= k_rem) {
    x = x0 + 1;
    above = excl + c0;
  }
  if (x >= 0) {
    const uint32_t digit = static_cast<uint32_t>(nb - 1 - x);
    const int sh = digit_shift(pass);
    SelState n = s;
    n.prefix = s.prefix | (digit << sh);
    n.mask = s.mask | (digit_mask(pass) << sh);
    n.k_rem = k_rem - above;
    st[seg] = n;
  }
}

// Per chunk: number of keys above T and equal to T.
__global__ void __launch_bounds__(kSelThreads) sel_count(const float* S, int64_t n_c, int64_t n_protect, int mode,
                                                         int nchunk, const SelState* st, uint32_t* cg,
                                                         uint32_t* ce) {
  __shared__ unsigned long long wbuf[32];
  const int b = blockIdx.y;
  const int seg = mode == KVZ_GLOBAL ? 0 : b;
  const uint32_t T = st[seg].prefix;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kSelChunk;
  const int lim = static_cast<int>(min(static_cast<int64_t>(kSelChunk), n_c - c0));
  const float* src = S + static_cast<int64_t>(b) * n_c + c0;
  uint32_t gt = 0u, eq = 0u;
  for (int e = threadIdx.x; e < lim; e += kSelThreads) {
    const uint32_t key = select_key(src - c0, c0 + e, n_protect, nullptr);
    gt += key > T ? 1u : 0u;
    eq += key == T ? 1u : 0u;
  }
  // pack both counts (each <= 4096) into one 64-bit sum
  const unsigned long long both =
      block_inclusive_sum<unsigned long long>((static_cast<unsigned long long>(gt) << 32) | eq, wbuf);
  if (threadIdx.x == kSelThreads - 1) {
    const int64_t x = static_cast<int64_t>(b) * nchunk + blockIdx.x;
    cg[x] = static_cast<uint32_t>(both >> 32);
    ce[x] = static_cast<uint32_t>(both & 0xFFFFFFFFull);
  }
}

// Single CTA: tie quota per chunk, per-head output bases, counts, offsets.
__global__ void __launch_bounds__(1024) sel_scan(int64_t B, int nchunk, int mode, const SelState* st,
                                                 const uint32_t* cg, const uint32_t* ce,
                                                 unsigned long long* eqb, uint32_t* cbase,
                                                 unsigned long long* head_eq, unsigned long long* head_base,
                                                 int32_t* counts, int64_t* offsets,
                                                 const unsigned long long* eq_ranks, int rank) {
  __shared__ unsigned long long wbuf[32];
  __shared__ unsigned long long carry;
  // 1. equal keys before each chunk, within its head
  for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
    unsigned long long run = 0ull;
    for (int c = 0; c < nchunk; ++c) {
      const int64_t x = b * nchunk + c;
      eqb[x] = run;
      run += ce[x];
    }
    head_eq[b] = run;
  }
  __syncthreads();
  // 2. equal keys in earlier heads (global mode: one segment spans all heads,
  //    and with the heads split over ranks, those of lower ranks come first)
  if (threadIdx.x == 0) {
    unsigned long long lower = 0ull;
    if (eq_ranks != nullptr)
      for (int r = 0; r < rank; ++r) lower += eq_ranks[r];
    carry = lower;
  }
  __syncthreads();
  for (int64_t t0 = 0; t0 < B; t0 += blockDim.x) {
    const int64_t b = t0 + threadIdx.x;
    const unsigned long long v = (mode == KVZ_GLOBAL && b < B) ? head_eq[b] : 0ull;
    const unsigned long long incl = block_inclusive_sum<unsigned long long>(v, wbuf);
    if (b < B) head_base[b] = carry + incl - v;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry += incl;
    __syncthreads();
  }
  // 3. kept keys per chunk and per head
  for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
    const int seg = mode == KVZ_GLOBAL ? 0 : static_cast<int>(b);
    const unsigned long long r_t = st[seg].k_rem;
    unsigned long long run = 0ull;
    for (int c = 0; c < nchunk; ++c) {
      const int64_t x = b * nchunk + c;
      const unsigned long long e = head_base[b] + eqb[x];
      const unsigned long long take = r_t > e ? min(r_t - e, static_cast<unsigned long long>(ce[x])) : 0ull;
      eqb[x] = e;
      cbase[x] = static_cast<uint32_t>(run);
      run += cg[x] + take;
    }
    counts[b] = static_cast<int32_t>(run);
  }
  __syncthreads();
  // 4. offsets = exclusive prefix sum of counts
  if (threadIdx.x == 0) carry = 0ull;
  __syncthreads();
  for (int64_t t0 = 0; t0 < B; t0 += blockDim.x) {
    const int64_t b = t0 + threadIdx.x;
    const unsigned long long v = b < B ? static_cast<unsigned long long>(counts[b]) : 0ull;
    const unsigned long long incl = block_inclusive_sum<unsigned long long>(v, wbuf);
    if (b < B) offsets[b] = static_cast<int64_t>(carry + incl - v);
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry += incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) offsets[B] = static_cast<int64_t>(carry);
}

// Per chunk: write the kept positions in ascending order.
__global__ void __launch_bounds__(kSelThreads) sel_write(const float* S, int64_t n_c, int64_t n_protect, int mode,
                                                         int nchunk, const SelState* st,
                                                         const unsigned long long* eqb, const uint32_t* cbase,
                                                         const int64_t* offsets, int32_t* idx) {
  __shared__ uint32_t wbuf[32];
  const int b = blockIdx.y;
  const int seg = mode == KVZ_GLOBAL ? 0 : b;
  const uint32_t T = st[seg].prefix;
  const unsigned long long r_t = st[seg].k_rem;
  const int64_t x = static_cast<int64_t>(b) * nchunk + blockIdx.x;
  const unsigned long long e0 = eqb[x];
  const int64_t out0 = offsets[b] + cbase[x];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kSelChunk;
  const int lim = static_cast<int>(min(static_cast<int64_t>(kSelChunk), n_c - c0));
  const float* src = S + static_cast<int64_t>(b) * n_c + c0;
  const int l0 = threadIdx.x * kSelItems;          // this thread's items, in order
  uint32_t key[kSelItems];
  uint32_t neq = 0u;
#pragma unroll
  for (int it = 0; it < kSelItems; ++it) {
    const int l = l0 + it;
    key[it] = l < lim ? select_key(src - c0, c0 + l, n_protect, nullptr) : 0u;
    neq += (l < lim && key[it] == T) ? 1u : 0u;
  }
  const uint32_t eq_incl = block_inclusive_sum<uint32_t>(neq, wbuf);
  unsigned long long e = e0 + (eq_incl - neq);
  uint32_t keep_bits = 0u, nkeep = 0u;
#pragma unroll
  for (int it = 0; it < kSelItems; ++it) {
    const int l = l0 + it;
    bool keep = false;
    if (l < lim) {
      if (key[it] > T) {
        keep = true;
      } else if (key[it] == T) {
        keep = e < r_t;
        ++e;
      }
    }
    keep_bits |= keep ? (1u << it) : 0u;
    nkeep += keep ? 1u : 0u;
  }
  const uint32_t keep_incl = block_inclusive_sum<uint32_t>(nkeep, wbuf);
  int64_t pos = out0 + (keep_incl - nkeep);
#pragma unroll
  for (int it = 0; it < kSelItems; ++it) {
    if (keep_bits & (1u << it)) idx[pos++] = static_cast<int32_t>(c0 + l0 + it);
  }
}

// Single CTA: the number of keys equal to T over all chunks of all heads.
__global__ void __launch_bounds__(1024) sel_eq_total(const uint32_t* ce, int64_t nx, unsigned long long* out) {
  __shared__ unsigned long long wbuf[32];
  unsigned long long v = 0ull;
  for (int64_t i = threadIdx.x; i < nx; i += blockDim.x) v += ce[i];
  const unsigned long long incl = block_inclusive_sum<unsigned long long>(v, wbuf);
  if (threadIdx.x == blockDim.x - 1) *out = incl;
}

// Per-head mode, one CTA per head: the same radix select and stable write as
// the kernels above, with the histograms, the digit picks and the scans in
// shared memory, so the whole selection is one launch.  With STAGED the
// head's keys stay in shared memory after the first pass.
constexpr int kHeadThreads = 1024;
constexpr int kHeadItems = 8;                            // consecutive scores per thread when writing
constexpr int kHeadTile = kHeadThreads * kHeadItems;
constexpr int64_t kHeadStageMax = 49152;                 // scores staged in shared memory (192 KB)

template <bool STAGED>
__global__ void __launch_bounds__(kHeadThreads) sel_head_kernel(const float* S, int64_t B, int64_t n_c,
                                                                int64_t n_protect, int64_t k, int32_t* idx,
                                                                int32_t* counts, int64_t* offsets,
                                                                int32_t* status) {
  extern __shared__ uint32_t skey[];                     // STAGED: the head's keys
  __shared__ uint32_t hist[kBins];
  __shared__ unsigned long long wbuf[32];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ unsigned long long s_krem, s_keep, s_eq;
  const int64_t b = blockIdx.x;
  const float* src = S + b * n_c;
  if (threadIdx.x == 0) {
    counts[b] = static_cast<int32_t>(k);
    offsets[b] = b * k;
    if (b == B - 1) offsets[B] = B * k;
    s_prefix = 0u;
    s_mask = 0u;
    s_krem = static_cast<unsigned long long>(k);
    s_keep = 0ull;
    s_eq = 0ull;
  }
  if (k == 0) return;
  auto key_at = [&](int64_t j) -> uint32_t { return STAGED ? skey[j] : select_key(src, j, n_protect, nullptr); };

  for (int pass = 0; pass < 3; ++pass) {
    for (int e = threadIdx.x; e < kBins; e += kHeadThreads) hist[e] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    const int sh = digit_shift(pass);
    const uint32_t dm = digit_mask(pass);
    for (int64_t j = threadIdx.x; j < n_c; j += kHeadThreads) {
      uint32_t key;
      if (pass == 0) {
        key = select_key(src, j, n_protect, status);
        if (STAGED) skey[j] = key;
      } else {
        key = key_at(j);
      }
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> sh) & dm], 1u);
    }
    __syncthreads();
    const unsigned long long k_rem = s_krem;
    // position x = 0 is the highest digit; thread t owns positions 2t, 2t+1
    const int nb = pass == 2 ? 1024 : 2048;
    const int x0 = 2 * static_cast<int>(threadIdx.x);
    const unsigned long long c0 = x0 < nb ? hist[nb - 1 - x0] : 0ull;
    const unsigned long long c1 = x0 + 1 < nb ? hist[nb - 2 - x0] : 0ull;
    const unsigned long long incl = block_inclusive_sum<unsigned long long>(c0 + c1, wbuf);
    const unsigned long long excl = incl - c0 - c1;
    int x = -1;
    unsigned long long above = 0ull;
    if (excl < k_rem && excl + c0 >= k_rem) {
      x = x0;
      above = excl;
    } else if (excl + c0 < k_rem && excl + c0 + c1 >= k_rem) {
      x = x0 + 1;
      above = excl + c0;
    }
    if (x >= 0) {                                        // exactly one thread
      const uint32_t digit = static_cast<uint32_t>(nb - 1 - x);
      s_prefix = prefix | (digit << sh);
      s_mask = mask | (dm << sh);
      s_krem = k_rem - above;
    }
    __syncthreads();
  }

  const uint32_t T = s_prefix;
  const unsigned long long r_t = s_krem;                 // keys equal to T that are kept
  int32_t* out = idx + b * k;
  for (int64_t base = 0; base < n_c; base += kHeadTile) {
    const unsigned long long keep0 = s_keep, eq0 = s_eq; // kept / equal keys before this tile
    const int64_t j0 = base + static_cast<int64_t>(threadIdx.x) * kHeadItems;
    uint32_t key[kHeadItems];
    uint32_t neq = 0u;
#pragma unroll
    for (int it = 0; it < kHeadItems; ++it) {
      const int64_t j = j0 + it;
      key[it] = j < n_c ? key_at(j) : 0u;
      neq += (j < n_c && key[it] == T) ? 1u : 0u;
    }
    const unsigned long long eq_incl = block_inclusive_sum<unsigned long long>(neq, wbuf);
    unsigned long long e = eq0 + eq_incl - neq;
    uint32_t keep_bits = 0u, nkeep = 0u;
#pragma unroll
    for (int it = 0; it < kHeadItems; ++it) {
      bool keep = false;
      if (j0 + it < n_c) {
        if (key[it] > T) {
          keep = true;
        } else if (key[it] == T) {
          keep = e < r_t;
          ++e;
        }
      }
      keep_bits |= keep ? (1u << it) : 0u;
      nkeep += keep ? 1u : 0u;
    }
    const unsigned long long keep_incl = block_inclusive_sum<unsigned long long>(nkeep, wbuf);
    int64_t pos = static_cast<int64_t>(keep0 + keep_incl - nkeep);
#pragma unroll
    for (int it = 0; it < kHeadItems; ++it)
      if (keep_bits & (1u << it)) out[pos++] = static_cast<int32_t>(j0 + it);
    if (threadIdx.x == kHeadThreads - 1) {               // after every thread read the carries
      s_keep = keep0 + keep_incl;
      s_eq = eq0 + eq_incl;
    }
    __syncthreads();
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

SelWorkspace select_workspace(int64_t B, int64_t n_c, int mode) {
  SelWorkspace w{};
  const int64_t nseg = mode == KVZ_GLOBAL ? 1 : B;
  const int64_t nchunk = (n_c + kSelChunk - 1) / kSelChunk;
  const int64_t nx = B * nchunk;
  size_t o = 0;
  w.off_state = o;     o = align256(o + sizeof(SelState) * nseg);
  w.off_hist = o;      o = align256(o + sizeof(uint32_t) * kBins * nseg);
  w.off_cg = o;        o = align256(o + sizeof(uint32_t) * nx);
  w.off_ce = o;        o = align256(o + sizeof(uint32_t) * nx);
  w.off_eqb = o;       o = align256(o + sizeof(unsigned long long) * nx);
  w.off_cbase = o;     o = align256(o + sizeof(uint32_t) * nx);
  w.off_head_eq = o;   o = align256(o + sizeof(unsigned long long) * B);
  w.off_head_base = o; o = align256(o + sizeof(unsigned long long) * B);
  w.bytes = o;
  return w;
}

cudaError_t launch_select(const float* S, int64_t B, int64_t n_c, int64_t n_protect, int mode, int64_t k,
                          int32_t* idx, int32_t* counts, int64_t* offsets, void* ws, const SelWorkspace& lay,
                          int32_t* status, cudaStream_t stream) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  SelState* st = reinterpret_cast<SelState*>(base + lay.off_state);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + lay.off_hist);
  uint32_t* cg = reinterpret_cast<uint32_t*>(base + lay.off_cg);
  uint32_t* ce = reinterpret_cast<uint32_t*>(base + lay.off_ce);
  unsigned long long* eqb = reinterpret_cast<unsigned long long*>(base + lay.off_eqb);
  uint32_t* cbase = reinterpret_cast<uint32_t*>(base + lay.off_cbase);
  unsigned long long* head_eq = reinterpret_cast<unsigned long long*>(base + lay.off_head_eq);
  unsigned long long* head_base = reinterpret_cast<unsigned long long*>(base + lay.off_head_base);
  if (mode == KVZ_PER_HEAD && (n_c <= kHeadStageMax || B >= 128)) {
    if (n_c <= kHeadStageMax) {
      const int smem = static_cast<int>(n_c * 4);
      cudaError_t e = smem_limit_once<sel_head_kernel<true>>(static_cast<int>(kHeadStageMax * 4));
      if (e != cudaSuccess) return e;
      sel_head_kernel<true><<<static_cast<unsigned>(B), kHeadThreads, smem, stream>>>(S, B, n_c, n_protect, k, idx,
                                                                                    counts, offsets, status);
    } else {
      sel_head_kernel<false><<<static_cast<unsigned>(B), kHeadThreads, 0, stream>>>(S, B, n_c, n_protect, k, idx,
                                                                                   counts, offsets, status);
    }
    return cudaGetLastError();
  }
  const int nseg = mode == KVZ_GLOBAL ? 1 : static_cast<int>(B);
  const int nchunk = static_cast<int>((n_c + kSelChunk - 1) / kSelChunk);
  const dim3 grid(static_cast<unsigned>(nchunk), static_cast<unsigned>(B));
  int64_t init_blocks = (static_cast<int64_t>(nseg) * kBins + 255) / 256;
  if (init_blocks > 1184) init_blocks = 1184;
  sel_init<<<static_cast<unsigned>(init_blocks), 256, 0, stream>>>(st, nseg, static_cast<unsigned long long>(k), hist);
  for (int pass = 0; pass < 3; ++pass) {
    sel_hist<<<grid, kSelThreads, 0, stream>>>(S, n_c, n_protect, mode, pass, st, hist, status);
    sel_pick<<<nseg, 1024, 0, stream>>>(pass, st, hist);
  }
  sel_count<<<grid, kSelThreads, 0, stream>>>(S, n_c, n_protect, mode, nchunk, st, cg, ce);
  sel_scan<<<1, 1024, 0, stream>>>(B, nchunk, mode, st, cg, ce, eqb, cbase, head_eq, head_base, counts, offsets,
                                   nullptr, 0);
  sel_write<<<grid, kSelThreads, 0, stream>>>(S, n_c, n_protect, mode, nchunk, st, eqb, cbase, offsets, idx);
  return cudaGetLastError();
}

// Global selection with the heads of one context split over ranks (rank r
// holds a contiguous range of heads, lower ranks first).  The kernels are
// those of launch_select in global mode; between the steps the caller sums
// `hist` over ranks (three times) and gathers every rank's equal-key total.
namespace {
struct DistPtrs {
  SelState* st;
  uint32_t *cg, *ce, *cbase;
  unsigned long long *eqb, *head_eq, *head_base;
};
DistPtrs dist_ptrs(void* ws, const SelWorkspace& lay) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  return DistPtrs{reinterpret_cast<SelState*>(base + lay.off_state),
                  reinterpret_cast<uint32_t*>(base + lay.off_cg),
                  reinterpret_cast<uint32_t*>(base + lay.off_ce),
                  reinterpret_cast<uint32_t*>(base + lay.off_cbase),
                  reinterpret_cast<unsigned long long*>(base + lay.off_eqb),
                  reinterpret_cast<unsigned long long*>(base + lay.off_head_eq),
                  reinterpret_cast<unsigned long long*>(base + lay.off_head_base)};
}
}  // namespace

cudaError_t launch_select_dist_begin(const float* S, int64_t B, int64_t n_c, int64_t k, uint32_t* hist, void* ws,
                                     const SelWorkspace& lay, int32_t* status, cudaStream_t stream) {
  const DistPtrs w = dist_ptrs(ws, lay);
  const int nchunk = static_cast<int>((n_c + kSelChunk - 1) / kSelChunk);
  const dim3 grid(static_cast<unsigned>(nchunk), static_cast<unsigned>(B));
  sel_init<<<8, 256, 0, stream>>>(w.st, 1, static_cast<unsigned long long>(k), hist);
  sel_hist<<<grid, kSelThreads, 0, stream>>>(S, n_c, 0, KVZ_GLOBAL, 0, w.st, hist, status);
  return cudaGetLastError();
}

cudaError_t launch_select_dist_step(const float* S, int64_t B, int64_t n_c, int pass, uint32_t* hist,
                                    unsigned long long* eq_total, void* ws, const SelWorkspace& lay,
                                    int32_t* status, cudaStream_t stream) {
  const DistPtrs w = dist_ptrs(ws, lay);
  const int nchunk = static_cast<int>((n_c + kSelChunk - 1) / kSelChunk);
  const dim3 grid(static_cast<unsigned>(nchunk), static_cast<unsigned>(B));
  sel_pick<<<1, 1024, 0, stream>>>(pass, w.st, hist);
  if (pass < 2) {
    sel_hist<<<grid, kSelThreads, 0, stream>>>(S, n_c, 0, KVZ_GLOBAL, pass + 1, w.st, hist, status);
  } else {
    sel_count<<<grid, kSelThreads, 0, stream>>>(S, n_c, 0, KVZ_GLOBAL, nchunk, w.st, w.cg, w.ce);
    sel_eq_total<<<1, 1024, 0, stream>>>(w.ce, B * nchunk, eq_total);
  }
  return cudaGetLastError();
}

cudaError_t launch_select_dist_finish(const float* S, int64_t B, int64_t n_c, const unsigned long long* eq_ranks,
                                      int rank, int32_t* idx, int32_t* counts, int64_t* offsets, void* ws,
                                      const SelWorkspace& lay, cudaStream_t stream) {
  const DistPtrs w = dist_ptrs(ws, lay);
  const int nchunk = static_cast<int>((n_c + kSelChunk - 1) / kSelChunk);
  const dim3 grid(static_cast<unsigned>(nchunk), static_cast<unsigned>(B));
  sel_scan<<<1, 1024, 0, stream>>>(B, nchunk, KVZ_GLOBAL, w.st, w.cg, w.ce, w.eqb, w.cbase, w.head_eq,
                                   w.head_base, counts, offsets, eq_ranks, rank);
  sel_write<<<grid, kSelThreads, 0, stream>>>(S, n_c, 0, KVZ_GLOBAL, nchunk, w.st, w.eqb, w.cbase, offsets, idx);
  return cudaGetLastError();
}

}  // namespace kvz
