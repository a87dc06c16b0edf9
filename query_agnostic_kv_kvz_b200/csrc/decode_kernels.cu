// Decode attention over the pruned KV cache (KVzip analysis report, §2.1:
// every later query reads the pruned cache K_p, V_p in place of the full
// one).  For KV head b with n_b kept rows and the G grouped queries of the
// new token:  out[b, g] = sum_j softmax_j(scale * <q_g, k_j>) v_j.
//
// HBM-bound: each step reads every kept key and value once (4*d bytes per
// kept row).  Split-KV on CUDA cores: a CTA takes a contiguous run of 64-key
// tiles of one head, brought in by TMA (three-stage ring, 128-byte swizzle so
// that one thread per key row reads shared memory without bank conflicts),
// keeps a running (max, sum, output) per query and writes it as a partial;
// decode_combine_kernel merges the partials of each (head, query).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kvz.h"
#include "kvz_internal.h"
#include "kvz_sm100.cuh"

namespace kvz {

namespace {

constexpr int kDecThreads = 128;
constexpr int kDecKeys = 64;                 // keys per tile (TMA box rows)
constexpr int kDecStages = 3;

template <int D>
struct DecLay {
  static constexpr int KB = D / 64;                          // 64-column blocks per row
  static constexpr int BLK = kDecKeys * 128;                 // 64 keys x 64 bf16 columns (8 KB)
  static constexpr int TILE = KB * BLK;                      // 64 keys of K (or of V)
  static constexpr int STAGE = 2 * TILE;                     // K then V
  static constexpr int Q_OFF = kDecStages * STAGE;           // float [G][D], times c2
  static constexpr int P_OFF = Q_OFF + kDecGMax * D * 4;     // float [G][kDecKeys]
  static constexpr int RED_OFF = P_OFF + kDecGMax * kDecKeys * 4;   // float [2][4 warps][G]
  static constexpr int O_OFF = RED_OFF + 2 * 4 * kDecGMax * 4;      // float [G][D] (second key group)
  static constexpr int BAR_OFF = O_OFF + kDecGMax * D * 4;
  static constexpr int SMEM = BAR_OFF + 64 + 1024;           // + alignment slack
};
static_assert(DecLay<128>::SMEM <= 113 * 1024, "two CTAs per SM");

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D>
__global__ void __launch_bounds__(kDecThreads)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        DecArgs p) {
  using L = DecLay<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  float* sQ = reinterpret_cast<float*>(smem + L::Q_OFF);
  float* sP = reinterpret_cast<float*>(smem + L::P_OFF);
  float* sRed = reinterpret_cast<float*>(smem + L::RED_OFF);
  float* sO = reinterpret_cast<float*>(smem + L::O_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + kDecStages);

  const int b = blockIdx.y, sp = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int count = p.counts[b];
  const int64_t off = p.offsets[b];
  if (count < 0 || count > p.n_c) {                           // the splits cover n_c keys at most
    if (sp == 0 && tid == 0 && p.status != nullptr) atomicCAS(p.status, 0, KVZ_ERR_INVALID_ARG);
    return;
  }
  const int ntile = (count + kDecKeys - 1) / kDecKeys;
  const int t0 = sp * p.cps;
  const int n = min(ntile, t0 + p.cps) - t0;                  // tiles of this split
  if (n <= 0) return;                                         // uniform: the combine skips it
  const int G = p.G;

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int e = tid; e < G * D; e += kDecThreads) {
    const uint16_t h = p.q[static_cast<int64_t>(b) * G * D + e];
    sQ[e] = __uint_as_float(static_cast<uint32_t>(h) << 16) * p.c2;
  }
  __syncthreads();
  auto issue = [&](int i) {
    const int s = i % kDecStages;
    mbar_arrive_expect_tx(&full[s], L::STAGE);
    const int row = static_cast<int>(off + static_cast<int64_t>(t0 + i) * kDecKeys);
    uint8_t* st = smem + s * L::STAGE;
    for (int kb = 0; kb < L::KB; ++kb) {
      tma_load_3d(st + kb * L::BLK, &tmK, &full[s], kb * 64, row, 0);
      tma_load_3d(st + L::TILE + kb * L::BLK, &tmV, &full[s], kb * 64, row, 0);
    }
  };
  if (tid == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    for (int i = 0; i < n && i < kDecStages; ++i) issue(i);
  }

  float m_run[kDecGMax], l_run[kDecGMax], o[kDecGMax];
#pragma unroll
  for (int g = 0; g < kDecGMax; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.0f;
    o[g] = 0.0f;
  }
  const int key = tid >> 1, half = tid & 1;                   // scores: two threads per key
  constexpr int kGroups = kDecThreads / D;                    // P.V: key groups (1 at d=128, 2 at d=64)
  const int dim = tid % D, kg = tid / D;
  int done = 0;
  for (int i = 0; i < n; ++i) {
    const int s = i % kDecStages;
    const bool got = mbar_wait(&full[s], static_cast<uint32_t>(i / kDecStages) & 1u, abort_flag, p.status);
    if (!__syncthreads_and(got)) break;                       // every thread leaves together
    const uint8_t* sK = smem + s * L::STAGE;
    const uint8_t* sV = sK + L::TILE;
    const int rows = min(kDecKeys, count - (t0 + i) * kDecKeys);

    // ---- scores of this thread's key over half of the dimensions
    float sc[kDecGMax];
#pragma unroll
    for (int g = 0; g < kDecGMax; ++g) sc[g] = 0.0f;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      const int d0 = half * (D / 2) + c * 8;
      const int kb = d0 / 64, cc = (d0 % 64) / 8;
      const uint4 kw = *reinterpret_cast<const uint4*>(sK + kb * L::BLK + key * 128 + ((cc ^ (key & 7)) * 16));
      const float k0 = bf16lo(kw.x), k1 = bf16hi(kw.x), k2 = bf16lo(kw.y), k3 = bf16hi(kw.y);
      const float k4 = bf16lo(kw.z), k5 = bf16hi(kw.z), k6 = bf16lo(kw.w), k7 = bf16hi(kw.w);
#pragma unroll
      for (int g = 0; g < kDecGMax; ++g) {
        if (g < G) {
          const float4 qa = *reinterpret_cast<const float4*>(sQ + g * D + d0);
          const float4 qb = *reinterpret_cast<const float4*>(sQ + g * D + d0 + 4);
          sc[g] = fmaf(k0, qa.x, fmaf(k1, qa.y, fmaf(k2, qa.z, fmaf(k3, qa.w, sc[g]))));
          sc[g] = fmaf(k4, qb.x, fmaf(k5, qb.y, fmaf(k6, qb.z, fmaf(k7, qb.w, sc[g]))));
        }
      }
    }
    // ---- tile max and running max per query
#pragma unroll
    for (int g = 0; g < kDecGMax; ++g) {
      sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], 1);
      if (key >= rows) sc[g] = -INFINITY;
      float mx = sc[g];
#pragma unroll
      for (int o2 = 16; o2 > 1; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      if (lane == 0 && g < G) sRed[warp * kDecGMax + g] = mx;
    }
    __syncthreads();
    float alpha[kDecGMax];
#pragma unroll
    for (int g = 0; g < kDecGMax; ++g) {
      const float mt = fmaxf(fmaxf(sRed[g], sRed[kDecGMax + g]), fmaxf(sRed[2 * kDecGMax + g], sRed[3 * kDecGMax + g]));
      const float mn = fmaxf(m_run[g], mt);                   // finite: the tile has a key
      alpha[g] = ex2_approx(m_run[g] - mn);                   // 0 on the first tile
      m_run[g] = mn;
      const float pv = ex2_approx(sc[g] - mn);
      if (half == 0 && g < G) sP[g * kDecKeys + key] = pv;
      float sm = half == 0 ? pv : 0.0f;
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o2);
      if (lane == 0 && g < G) sRed[4 * kDecGMax + warp * kDecGMax + g] = sm;
    }
    __syncthreads();
    // ---- running sum and P.V for this thread's output dimension
    const int kb = dim / 64, cc = (dim % 64) / 8, ee = dim % 8;
#pragma unroll
    for (int g = 0; g < kDecGMax; ++g) {
      const float ts = (sRed[4 * kDecGMax + g] + sRed[5 * kDecGMax + g]) +
                       (sRed[6 * kDecGMax + g] + sRed[7 * kDecGMax + g]);
      l_run[g] = fmaf(l_run[g], alpha[g], ts);
      o[g] *= alpha[g];
    }
    for (int k = kg; k < rows; k += kGroups) {
      const uint16_t vh = *reinterpret_cast<const uint16_t*>(sV + kb * L::BLK + k * 128 + ((cc ^ (k & 7)) * 16) +
                                                              ee * 2);
      const float v = __uint_as_float(static_cast<uint32_t>(vh) << 16);
#pragma unroll
      for (int g = 0; g < kDecGMax; ++g)
        if (g < G) o[g] = fmaf(sP[g * kDecKeys + k], v, o[g]);
    }
    __syncthreads();                                          // stage s, sP and sRed are free again
    if (tid == 0 && i + kDecStages < n) issue(i + kDecStages);
    done = i + 1;
  }
  if (done < n) {
    // a wait expired: let this CTA's own copies land (bounded) before leaving
    if (tid == 0)
      for (int i = done; i < n && i < done + kDecStages; ++i)
        mbar_wait_for(&full[i % kDecStages], static_cast<uint32_t>(i / kDecStages) & 1u, 20000000ull);
    return;
  }
  if (kGroups > 1) {                                          // fold the second key group's outputs
    if (kg == 1)
#pragma unroll
      for (int g = 0; g < kDecGMax; ++g)
        if (g < G) sO[g * D + dim] = o[g];
    __syncthreads();
    if (kg == 0)
#pragma unroll
      for (int g = 0; g < kDecGMax; ++g)
        if (g < G) o[g] += sO[g * D + dim];
  }
  const int64_t part = static_cast<int64_t>(b) * p.splits + sp;
#pragma unroll
  for (int g = 0; g < kDecGMax; ++g) {
    if (g < G) {
      if (tid == 0) p.part_ml[part * G + g] = make_float2(m_run[g], l_run[g]);
      if (kg == 0) p.part_o[(part * G + g) * D + dim] = o[g];
    }
  }
}

// Merge the partials of each (head, query): out = sum o_s 2^(m_s - M) / L.
template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_combine_kernel(DecArgs p, float* out, float* lse2) {
  const int b = blockIdx.x;
  const int count = p.counts[b];
  const int ntile = (count >= 0 && count <= p.n_c) ? (count + kDecKeys - 1) / kDecKeys : 0;
  const int nsp = min((ntile + p.cps - 1) / p.cps, p.splits);
  const int64_t base = static_cast<int64_t>(b) * p.splits;
  for (int g = 0; g < p.G; ++g) {
    float M = -INFINITY;
    for (int s = 0; s < nsp; ++s) M = fmaxf(M, p.part_ml[(base + s) * p.G + g].x);
    float Lsum = 0.0f;
    for (int s = 0; s < nsp; ++s) {
      const float2 ml = p.part_ml[(base + s) * p.G + g];
      Lsum += ml.y * exp2f(ml.x - M);
    }
    for (int d0 = threadIdx.x; d0 < D; d0 += blockDim.x) {
      float acc = 0.0f;
      for (int s = 0; s < nsp; ++s)
        acc += p.part_o[((base + s) * p.G + g) * D + d0] * exp2f(p.part_ml[(base + s) * p.G + g].x - M);
      out[(static_cast<int64_t>(b) * p.G + g) * D + d0] = nsp > 0 ? acc / Lsum : 0.0f;
    }
    if (threadIdx.x == 0 && lse2 != nullptr)
      lse2[static_cast<int64_t>(b) * p.G + g] = nsp > 0 ? M + log2f(Lsum) : -INFINITY;
  }
}

}  // namespace

void decode_plan(int64_t B, int64_t n_c, int* cps, int* splits) {
  const int64_t max_tiles = (n_c + kDecKeys - 1) / kDecKeys;
  const int64_t target = 148 * 2 * 4;                         // about four waves of two CTAs per SM
  int64_t c = (B * max_tiles + target - 1) / target;
  if (c < 1) c = 1;
  *cps = static_cast<int>(c);
  *splits = static_cast<int>((max_tiles + c - 1) / c);
}

cudaError_t launch_decode(int d, const CUtensorMap& tmK, const CUtensorMap& tmV, const DecArgs& a, float* out,
                          float* lse2, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(a.splits), static_cast<unsigned>(a.B));
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(decode_split_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecLay<128>::SMEM);
    if (e != cudaSuccess) return e;
    decode_split_kernel<128><<<grid, kDecThreads, DecLay<128>::SMEM, stream>>>(tmK, tmV, a);
    decode_combine_kernel<128><<<static_cast<unsigned>(a.B), kDecThreads, 0, stream>>>(a, out, lse2);
  } else {
    e = cudaFuncSetAttribute(decode_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecLay<64>::SMEM);
    if (e != cudaSuccess) return e;
    decode_split_kernel<64><<<grid, kDecThreads, DecLay<64>::SMEM, stream>>>(tmK, tmV, a);
    decode_combine_kernel<64><<<static_cast<unsigned>(a.B), kDecThreads, 0, stream>>>(a, out, lse2);
  }
  return cudaGetLastError();
}

}  // namespace kvz
