// Compaction of the kept KV rows into the pruned cache (KVzip analysis
// report, §2.1: the pruned cache K_p is a subset of the full cache K_c).
// Rows move as 16-byte vectors; key order is kept because idx ascends
// within each head.  HBM-bound: every kept row is read once and written once.
#include <cuda_runtime.h>

#include <cstdint>

#include "kvz.h"
#include "kvz_internal.h"

namespace kvz {

namespace {

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 4;
constexpr int kInplaceThreads = 512;
constexpr int kInplaceUnroll = 4;

__device__ __forceinline__ void report_err(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Read-only streaming load (inputs are never written by this kernel).
__device__ __forceinline__ int4 ld_stream(const int4* p) {
  int4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Out of place.  Grid-stride over blocks of output slots; the head of a
// block's first slot is found by binary search over offsets, later slots
// walk forward (slots are in head order).
__global__ void __launch_bounds__(kGatherThreads)
    compact_gather_kernel(const int4* __restrict__ K, const int4* __restrict__ V, int64_t B, int64_t n_c,
                          int vpr, const int32_t* __restrict__ idx, const int64_t* __restrict__ offsets,
                          const int64_t* __restrict__ out_offsets, int4* __restrict__ Ko,
                          int4* __restrict__ Vo, int32_t* status) {
  __shared__ int64_t s_head;
  const int64_t total = offsets[B];
  const int rows_per_step = kGatherThreads / vpr;               // rows one pass of the CTA covers
  const int rows_per_blk = rows_per_step * kGatherUnroll;
  const int my_row = threadIdx.x / vpr;
  const int vec = threadIdx.x % vpr;
  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_blk; r0 < total;
       r0 += static_cast<int64_t>(gridDim.x) * rows_per_blk) {
    __syncthreads();
    if (threadIdx.x == 0) {
      int64_t lo = 0, hi = B - 1;                                 // largest b with offsets[b] <= r0
      while (lo < hi) {
        const int64_t mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= r0) lo = mid; else hi = mid - 1;
      }
      s_head = lo;
    }
    __syncthreads();
    int64_t hb = s_head;
    int4 kv[kGatherUnroll], vv[kGatherUnroll];
    int64_t dst[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int64_t slot = r0 + u * rows_per_step + my_row;
      dst[u] = -1;
      if (slot < total) {
        while (hb + 1 < B && offsets[hb + 1] <= slot) ++hb;
        const int64_t j = idx[slot];
        if (j < 0 || j >= n_c) {
          report_err(status, KVZ_ERR_INVALID_ARG);
        } else {
          const int64_t src = (hb * n_c + j) * vpr + vec;
          const int64_t base = out_offsets != nullptr ? out_offsets[hb] : offsets[hb];
          dst[u] = (base + (slot - offsets[hb])) * vpr + vec;
          kv[u] = ld_stream(K + src);
          vv[u] = ld_stream(V + src);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      if (dst[u] >= 0) {
        Ko[dst[u]] = kv[u];
        Vo[dst[u]] = vv[u];
      }
    }
  }
}

// In place.  One CTA owns one column segment (vps vectors) of every row of
// one head of one tensor and walks the kept slots in increasing order, a
// batch at a time.  Slot p moves row idx[p] >= p down to row p.  The loads of
// batch t+1 read rows >= the first slot of batch t+1, which batch t never
// writes; the barrier orders every load of batches <= t before the stores
// of batch t, so no row is overwritten before it has been read.
__global__ void __launch_bounds__(kInplaceThreads)
    compact_inplace_kernel(int4* K, int4* V, int64_t n_c, int vpr, int cs, const int32_t* __restrict__ idx,
                           const int32_t* __restrict__ counts, const int64_t* __restrict__ offsets,
                           int32_t* status) {
  const int64_t b = blockIdx.x;
  const int tsel = blockIdx.y / cs;
  const int part = blockIdx.y % cs;
  const int vps = vpr / cs;
  int4* X = (tsel == 0 ? K : V) + b * n_c * vpr + part * vps;
  const int64_t count = counts[b];
  const int64_t base = offsets[b];
  const int rows_per_batch = kInplaceThreads * kInplaceUnroll / vps;
  const int64_t nb = (count + rows_per_batch - 1) / rows_per_batch;
  if (count < 0 || count > n_c) {
    if (threadIdx.x == 0) report_err(status, KVZ_ERR_INVALID_ARG);
    return;
  }
  int4 cur[kInplaceUnroll], nxt[kInplaceUnroll];
  bool cur_ok[kInplaceUnroll], nxt_ok[kInplaceUnroll];
  auto load = [&](int64_t t, int4 (&v)[kInplaceUnroll], bool (&ok)[kInplaceUnroll]) {
#pragma unroll
    for (int u = 0; u < kInplaceUnroll; ++u) {
      const int item = threadIdx.x + u * kInplaceThreads;
      const int64_t p = t * rows_per_batch + item / vps;
      ok[u] = false;
      if (p < count) {
        const int64_t j = idx[base + p];
        if (j < p || j >= n_c) {             // ascending idx guarantees j >= p
          report_err(status, KVZ_ERR_INVALID_ARG);
        } else {
          v[u] = __ldcg(X + j * vpr + item % vps);
          ok[u] = true;
        }
      }
    }
  };
  if (nb > 0) load(0, cur, cur_ok);
  for (int64_t t = 0; t < nb; ++t) {
    if (t + 1 < nb) load(t + 1, nxt, nxt_ok);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kInplaceUnroll; ++u) {
      const int item = threadIdx.x + u * kInplaceThreads;
      const int64_t p = t * rows_per_batch + item / vps;
      if (cur_ok[u]) X[p * vpr + item % vps] = cur[u];
    }
#pragma unroll
    for (int u = 0; u < kInplaceUnroll; ++u) {
      cur[u] = nxt[u];
      cur_ok[u] = nxt_ok[u];
    }
  }
}

}  // namespace

cudaError_t launch_compact_gather(const void* K, const void* V, int64_t B, int64_t n_c, int d,
                                  const int32_t* idx, const int64_t* offsets, const int64_t* out_offsets,
                                  void* K_out, void* V_out, int32_t* status, cudaStream_t stream) {
  const int vpr = d / 8;                       // 16-byte vectors per row
  const int rows_per_blk = (kGatherThreads / vpr) * kGatherUnroll;
  int64_t blocks = (B * n_c + rows_per_blk - 1) / rows_per_blk;
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  compact_gather_kernel<<<static_cast<unsigned>(blocks), kGatherThreads, 0, stream>>>(
      static_cast<const int4*>(K), static_cast<const int4*>(V), B, n_c, vpr, idx, offsets, out_offsets,
      static_cast<int4*>(K_out), static_cast<int4*>(V_out), status);
  return cudaGetLastError();
}

cudaError_t launch_compact_inplace(void* K, void* V, int64_t B, int64_t n_c, int d, const int32_t* idx,
                                   const int32_t* counts, const int64_t* offsets, int32_t* status,
                                   cudaStream_t stream) {
  const int vpr = d / 8;
  const int cs = vpr / 8;                      // 128-byte column segments
  const dim3 grid(static_cast<unsigned>(B), static_cast<unsigned>(2 * cs));
  compact_inplace_kernel<<<grid, kInplaceThreads, 0, stream>>>(static_cast<int4*>(K), static_cast<int4*>(V),
                                                               n_c, vpr, cs, idx, counts, offsets, status);
  return cudaGetLastError();
}

}  // namespace kvz
