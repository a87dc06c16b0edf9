// Context-independent head scores and head-level eviction (KVzip analysis
// report, §4.2: one static importance per head, the pair scores aggregated
// by a max along the sequence; heads are then kept or evicted whole).
//
// head_max_kernel is a segmented max over S, HBM-bound (4 bytes per score).
// Scores are non-negative, so their fp32 bit patterns (-0 folded onto +0)
// order like the values and partial maxima merge with an integer atomicMax.
#include <cuda_runtime.h>

#include <cstdint>

#include "kvz.h"
#include "kvz_internal.h"

namespace kvz {

namespace {

constexpr int kHeadMaxThreads = 256;
constexpr int kHeadMaxItems = 32;                           // scores per thread per CTA
constexpr int kHeadMaxSpan = kHeadMaxThreads * kHeadMaxItems;

__device__ __forceinline__ void report_err(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__global__ void __launch_bounds__(kHeadMaxThreads)
    head_max_kernel(const float* __restrict__ S, int64_t n_c, uint32_t* S_head, int32_t* status) {
  __shared__ uint32_t wmax[kHeadMaxThreads / 32];
  const int64_t b = blockIdx.y;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kHeadMaxSpan;
  const float* src = S + b * n_c;
  uint32_t best = 0u;
#pragma unroll 8
  for (int it = 0; it < kHeadMaxItems; ++it) {
    const int64_t j = j0 + it * kHeadMaxThreads + threadIdx.x;    // coalesced
    if (j < n_c) {
      uint32_t u = __float_as_uint(__ldg(src + j));
      if (u == 0x80000000u) u = 0u;
      if (u > 0x7F800000u) {                                       // NaN or negative
        report_err(status, KVZ_ERR_INVALID_SCORE);
        u = 0u;
      }
      best = u > best ? u : best;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t y = __shfl_xor_sync(0xffffffffu, best, o);
    best = y > best ? y : best;
  }
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kHeadMaxThreads / 32; ++w) best = wmax[w] > best ? wmax[w] : best;
    atomicMax(&S_head[b], best);
  }
}

// counts[b] = n_c for a kept head, 0 otherwise; offsets from the rank of b
// among the kept heads (kept is ascending, so the rank is a lower bound).
__global__ void head_csr_kernel(const int32_t* __restrict__ kept, int64_t k, int64_t B, int64_t n_c,
                                int32_t* counts, int64_t* offsets) {
  const int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (b > B) return;
  int64_t lo = 0, hi = k;                                   // first r with kept[r] >= b
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (kept[mid] < b) lo = mid + 1; else hi = mid;
  }
  offsets[b] = lo * n_c;
  if (b < B) counts[b] = (lo < k && kept[lo] == b) ? static_cast<int32_t>(n_c) : 0;
}

// idx of a kept head is every position 0..n_c-1.
__global__ void head_idx_kernel(int64_t total, int64_t n_c, int32_t* idx) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x)
    idx[e] = static_cast<int32_t>(e % n_c);
}

}  // namespace

cudaError_t launch_head_max(const float* S, int64_t B, int64_t n_c, float* S_head, int32_t* status,
                            cudaStream_t stream) {
  cudaError_t e = launch_fill_f32(S_head, B, 0.0f, stream);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((n_c + kHeadMaxSpan - 1) / kHeadMaxSpan), static_cast<unsigned>(B));
  head_max_kernel<<<grid, kHeadMaxThreads, 0, stream>>>(S, n_c, reinterpret_cast<uint32_t*>(S_head), status);
  return cudaGetLastError();
}

cudaError_t launch_head_expand(const int32_t* kept, int64_t k, int64_t B, int64_t n_c, int32_t* idx,
                               int32_t* counts, int64_t* offsets, cudaStream_t stream) {
  head_csr_kernel<<<static_cast<unsigned>((B + 1 + 255) / 256), 256, 0, stream>>>(kept, k, B, n_c, counts, offsets);
  const int64_t total = k * n_c;
  if (total > 0) {
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    head_idx_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(total, n_c, idx);
  }
  return cudaGetLastError();
}

}  // namespace kvz
