// Decode attention over the pruned KV cache (KVzip analysis report, §2.1:
// every later query reads the pruned cache K_p, V_p in place of the full
// one).  For KV head b with n_b kept rows and the G grouped queries of the
// new token:  out[b, g] = sum_j softmax_j(scale * <q_g, k_j>) v_j.
//
// HBM-bound: each step reads every kept key and value once (4*d bytes per
// kept row).  Split-KV: a CTA takes a contiguous run of 64-key tiles of one
// head, brought in by TMA (three-stage ring, 128-byte swizzle, read back with
// ldmatrix), keeps a running (max, sum, output) per query and writes it as a
// partial; the CTA that finishes a head's last split merges its partials.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kvz.h"
#include "kvz_internal.h"
#include "kvz_sm100.cuh"

namespace kvz {

namespace {

constexpr int kDecThreads = 128;            // 4 warps; warp w owns keys [16w, 16w+16) of every tile
constexpr int kDecKeys = 64;                 // keys per tile (TMA box rows)
constexpr int kDecStages = 3;
constexpr int kDecMaxSplits = 256;           // splits per head (shared-memory weights in the combine)
constexpr int kDecWarps = kDecThreads / 32;

template <int D>
struct DecLay {
  static constexpr int KB = D / 64;                          // 64-column blocks per row
  static constexpr int BLK = kDecKeys * 128;                 // 64 keys x 64 bf16 columns (8 KB)
  static constexpr int TILE = KB * BLK;                      // 64 keys of K (or of V)
  static constexpr int STAGE = 2 * TILE;                     // K then V
  static constexpr int Q_OFF = kDecStages * STAGE;           // bf16 [8][D]: the queries (rows >= G zero)
  static constexpr int M_OFF = Q_OFF + 8 * D * 2;            // float [warps][8] running max, then sum
  static constexpr int O_OFF = 0;                            // float [warps][8][D], over the idle stages
  static constexpr int BAR_OFF = M_OFF + 2 * kDecWarps * 8 * 4;
  static constexpr int SMEM = BAR_OFF + 64 + 1024;           // + alignment slack
};
static_assert(DecLay<128>::SMEM <= 113 * 1024, "two CTAs per SM");
static_assert(kDecWarps * 8 * 128 * 4 <= kDecStages * DecLay<128>::STAGE, "the warps' merge fits the stages");

// D = A * B + D for one 16x8x16 tile: A 16x16 bf16 (row), B 16x8 bf16 (col), D fp32.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// Two floats as a bf16x2 word (round to nearest even), low half = x.
__device__ __forceinline__ uint32_t pack_bf16x2(float x, float y) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y), "f"(x));
  return r;
}
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Shared-memory address of 16-byte chunk (dim / 8) of key row `key` in a
// swizzled 64-key tile (128-byte swizzle within each 64-column block).
template <int D>
__device__ __forceinline__ uint32_t tile_chunk(uint32_t tile, int key, int dim) {
  return tile + (dim / 64) * DecLay<D>::BLK + key * 128 + ((((dim % 64) / 8) ^ (key & 7)) * 16);
}

// Merge the partials of head b: out = sum_s o_s 2^(m_s - M) / L with
// L = sum_s l_s 2^(m_s - M), M = max_s m_s.  Run by the CTA that finishes the
// head's last split; the splits' partials are read from L2.
template <int D>
__device__ void combine_head(const DecArgs& p, int b, int nsp, float* out, float* lse2, float* s_w) {
  const int G = p.G;
  const int64_t base = static_cast<int64_t>(b) * p.splits;
  __shared__ float s_M[kDecGMax], s_L[kDecGMax];
  if (threadIdx.x < G) {
    const int g = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < nsp; ++s) M = fmaxf(M, __ldcg(&p.part_ml[(base + s) * G + g]).x);
    float Ls = 0.0f;
    for (int s = 0; s < nsp; ++s) {
      const float2 ml = __ldcg(&p.part_ml[(base + s) * G + g]);
      const float wgt = exp2f(ml.x - M);
      s_w[s * kDecGMax + g] = wgt;
      Ls += ml.y * wgt;
    }
    s_M[g] = M;
    s_L[g] = Ls;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += kDecThreads) {
    const int g = e / D;
    float acc = 0.0f;
#pragma unroll 8
    for (int s = 0; s < nsp; ++s) acc = fmaf(__ldcg(&p.part_o[((base + s) * G) * D + e]), s_w[s * kDecGMax + g], acc);
    out[static_cast<int64_t>(b) * G * D + e] = acc / s_L[g];
  }
  if (threadIdx.x < G && lse2 != nullptr)
    lse2[static_cast<int64_t>(b) * G + threadIdx.x] = s_M[threadIdx.x] + log2f(s_L[threadIdx.x]);
}

// Split-KV decode on the tensor cores (mma.sync m16n8k16, bf16 -> fp32): the
// G <= 8 queries of a KV head are the rows of the MMA (padded to 16), which
// is below the 64-row minimum of tcgen05; the kernel is HBM-bound and the
// MMAs only remove the per-key instruction cost of a CUDA-core dot product.
// S = Q K^T per 16-key slice of a warp; P = 2^(S - m) is split exactly into
// bf16 hi + lo parts (P - hi is representable to 2^-16 of P), so P.V keeps
// near-fp32 accuracy with two bf16 MMAs.
template <int D>
__global__ void __launch_bounds__(kDecThreads)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        DecArgs p, float* out, float* lse2) {
  using L = DecLay<D>;
  constexpr int KS = D / 16;                                  // k-steps of Q K^T
  constexpr int NT = D / 8;                                   // n-tiles of P V
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem + L::Q_OFF);
  float* sM = reinterpret_cast<float*>(smem + L::M_OFF);              // [warps][8]
  float* sL = sM + kDecWarps * 8;                                      // [warps][8]
  float* sO = reinterpret_cast<float*>(smem + L::O_OFF);              // [warps][8][D]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + kDecStages);

  const int b = blockIdx.y, sp = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int count = p.counts[b];
  const int64_t off = p.offsets[b];
  if (count < 0 || count > p.n_c) {                           // the splits cover n_c keys at most
    if (sp == 0 && tid == 0 && p.status != nullptr) atomicCAS(p.status, 0, KVZ_ERR_INVALID_ARG);
    return;
  }
  const int ntile = (count + kDecKeys - 1) / kDecKeys;
  const int cps = (ntile + p.splits - 1) / p.splits;          // this head's tiles spread over all its splits
  const int t0 = sp * cps;
  const int n = min(ntile, t0 + cps) - t0;                    // tiles of this split
  if (ntile == 0 && sp == 0) {                                // no kept rows: output 0, lse -inf
    for (int e = tid; e < G * D; e += kDecThreads) out[static_cast<int64_t>(b) * G * D + e] = 0.0f;
    if (tid < G && lse2 != nullptr) lse2[static_cast<int64_t>(b) * G + tid] = -INFINITY;
  }
  if (n <= 0) return;                                         // uniform: no partial from this split

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int e = tid; e < 8 * D; e += kDecThreads)
    sQ[e] = e / D < G ? p.q[static_cast<int64_t>(b) * G * D + e] : uint16_t(0);
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

  // A fragments of Q (rows = queries; rows 8..15 are padding and stay zero):
  // this thread's row r = lane/4, columns 2c, 2c+1 and 2c+8, 2c+9 of each k-step.
  const int r = lane >> 2, c = lane & 3;
  uint32_t qa0[KS], qa2[KS];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    qa0[ks] = *reinterpret_cast<const uint32_t*>(sQ + r * D + ks * 16 + 2 * c);
    qa2[ks] = *reinterpret_cast<const uint32_t*>(sQ + r * D + ks * 16 + 8 + 2 * c);
  }
  float o[NT][4];                                              // P.V accumulators (rows r and r+8)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f;                       // of query row r over this warp's keys
  const float c2 = p.c2;
  const int kw0 = warp * 16;                                   // this warp's keys within a tile
  // ldmatrix row addresses: lane l feeds row l % 8 of matrix l / 8
  const int lm = lane >> 3, lr = lane & 7;
  int done = 0;
  for (int i = 0; i < n; ++i) {
    const int s = i % kDecStages;
    const bool got = tid != 0 || mbar_wait(&full[s], static_cast<uint32_t>(i / kDecStages) & 1u, abort_flag,
                                           p.status);
    if (!__syncthreads_and(got)) break;
    const uint32_t sK = smem_u32(smem + s * L::STAGE);
    const uint32_t sV = sK + L::TILE;
    const int rows = min(kDecKeys, count - (t0 + i) * kDecKeys);

    if (kw0 < rows) {                                          // warp-uniform
      // ---- S = Q K^T for keys kw0 .. kw0+15 (two n-tiles of 8 keys)
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        // matrices: (keys 0-7, dims 0-7), (keys 0-7, dims 8-15), (keys 8-15, dims 0-7), (keys 8-15, dims 8-15)
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tile_chunk<D>(sK, kw0 + (lm >> 1) * 8 + lr, ks * 16 + (lm & 1) * 8), b0, b1, b2, b3);
        mma_bf16_16816(s0, qa0[ks], 0u, qa2[ks], 0u, b0, b1);
        mma_bf16_16816(s1, qa0[ks], 0u, qa2[ks], 0u, b2, b3);
      }
      // ---- online softmax of row r over these 16 keys (base 2)
      const int k0 = kw0 + 2 * c;                              // keys of s0[0], s0[1]; s1 holds k0+8, k0+9
      float x0 = k0 < rows ? s0[0] * c2 : -INFINITY;
      float x1 = k0 + 1 < rows ? s0[1] * c2 : -INFINITY;
      float x2 = k0 + 8 < rows ? s1[0] * c2 : -INFINITY;
      float x3 = k0 + 9 < rows ? s1[1] * c2 : -INFINITY;
      float mt = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
      const float mn = fmaxf(m_run, mt);                       // finite: key kw0 < rows is visible
      const float alpha = ex2_approx(m_run - mn);              // 0 on this warp's first keys
      m_run = mn;
      const float p0 = ex2_approx(x0 - mn), p1 = ex2_approx(x1 - mn);
      const float p2 = ex2_approx(x2 - mn), p3 = ex2_approx(x3 - mn);
      float ts = (p0 + p1) + (p2 + p3);
      ts += __shfl_xor_sync(0xffffffffu, ts, 1);
      ts += __shfl_xor_sync(0xffffffffu, ts, 2);
      l_run = fmaf(l_run, alpha, ts);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        o[nt][0] *= alpha;
        o[nt][1] *= alpha;
      }
      // ---- P as the A operand of P.V (keys are the k dimension): exact hi + lo split
      const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
      const uint32_t l01 = pack_bf16x2(p0 - bf16lo(h01), p1 - bf16hi(h01));
      const uint32_t l23 = pack_bf16x2(p2 - bf16lo(h23), p3 - bf16hi(h23));
      // ---- O += P V over the warp's 16 keys, two n-tiles (16 dims) per ldmatrix
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        // matrices: (keys 0-7, dims 0-7), (keys 8-15, dims 0-7), (keys 0-7, dims 8-15), (keys 8-15, dims 8-15)
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(tile_chunk<D>(sV, kw0 + (lm & 1) * 8 + lr, nt * 8 + (lm >> 1) * 8), v0, v1, v2, v3);
        mma_bf16_16816(o[nt], h01, 0u, h23, 0u, v0, v1);
        mma_bf16_16816(o[nt], l01, 0u, l23, 0u, v0, v1);
        mma_bf16_16816(o[nt + 1], h01, 0u, h23, 0u, v2, v3);
        mma_bf16_16816(o[nt + 1], l01, 0u, l23, 0u, v2, v3);
      }
    }
    __syncthreads();                                          // stage s is free again
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
  // ---- merge the four warps' states of each query row, write the split's partial
  // (sO lies over the stages: every issued tile has been consumed by now)
  if (c == 0) {
    sM[warp * 8 + r] = m_run;
    sL[warp * 8 + r] = l_run;
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    sO[(warp * 8 + r) * D + nt * 8 + 2 * c] = o[nt][0];
    sO[(warp * 8 + r) * D + nt * 8 + 2 * c + 1] = o[nt][1];
  }
  __syncthreads();
  const int64_t part = static_cast<int64_t>(b) * p.splits + sp;
  for (int e = tid; e < G * D; e += kDecThreads) {
    const int g = e / D, dd = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < kDecWarps; ++w2) M = fmaxf(M, sM[w2 * 8 + g]);
    float Ls = 0.0f, acc = 0.0f;
#pragma unroll
    for (int w2 = 0; w2 < kDecWarps; ++w2) {
      const float mw = sM[w2 * 8 + g];
      if (mw == -INFINITY) continue;                           // that warp saw no key of this split
      const float wgt = exp2f(mw - M);
      Ls += sL[w2 * 8 + g] * wgt;
      acc += sO[(w2 * 8 + g) * D + dd] * wgt;
    }
    p.part_o[(part * G + g) * D + dd] = acc;
    if (dd == 0) p.part_ml[part * G + g] = make_float2(M, Ls);
  }
  // ---- the CTA that finishes the head's last split merges all of them
  __shared__ int s_last;
  __threadfence();                                            // this partial before the count
  __syncthreads();
  const int nsp = (ntile + cps - 1) / cps;                    // splits of this head that have tiles
  if (tid == 0) s_last = atomicAdd(&p.done[b], 1u) == static_cast<unsigned>(nsp - 1);
  __syncthreads();
  if (s_last) {
    __threadfence();                                          // the other splits' partials before reading them
    __syncthreads();
    combine_head<D>(p, b, nsp, out, lse2, reinterpret_cast<float*>(smem));   // weights over the idle stages
  }
}

}  // namespace

// Splits per head: about two waves of two CTAs per SM over all heads, at
// most one split per 64-key tile of the longest possible head and at most
// kDecMaxSplits (each head's tiles are spread over its splits on the device,
// from its own count).
void decode_plan(int64_t B, int64_t n_c, int* cps, int* splits) {
  const int64_t max_tiles = (n_c + kDecKeys - 1) / kDecKeys;
  const int64_t target = 148 * 2 * 2;
  int64_t sp = (target + B - 1) / B;
  if (sp > max_tiles) sp = max_tiles;
  if (sp > kDecMaxSplits) sp = kDecMaxSplits;
  if (sp < 1) sp = 1;
  *splits = static_cast<int>(sp);
  *cps = static_cast<int>((max_tiles + sp - 1) / sp);
}

namespace {

template <int D>
cudaError_t launch_split(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecArgs& a, float* out, float* lse2,
                         cudaStream_t stream) {
  cudaError_t e = smem_limit_once<decode_split_kernel<D>>(DecLay<D>::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(a.splits), static_cast<unsigned>(a.B));
  decode_split_kernel<D><<<grid, kDecThreads, DecLay<D>::SMEM, stream>>>(tmK, tmV, a, out, lse2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(int d, const CUtensorMap& tmK, const CUtensorMap& tmV, const DecArgs& a, float* out,
                          float* lse2, cudaStream_t stream) {
  // per-head counts of finished splits start at zero (all-zero bits)
  cudaError_t e = launch_fill_f32(reinterpret_cast<float*>(a.done), a.B, 0.0f, stream);
  if (e != cudaSuccess) return e;
  return d == 128 ? launch_split<128>(tmK, tmV, a, out, lse2, stream)
                  : launch_split<64>(tmK, tmV, a, out, lse2, stream);
}

}  // namespace kvz
