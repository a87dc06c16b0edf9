// Decode attention over the pruned KV cache (KVzip analysis report, §2.1:
// every later query reads the pruned cache K_p, V_p in place of the full
// one).  For KV head b with n_b kept rows and the G grouped queries of the
// new token:  out[b, g] = sum_j softmax_j(scale * <q_g, k_j>) v_j.
//
// HBM-bound: each step reads every kept key and value once (4*d bytes per
// kept row).  Split-KV over a work list that a one-CTA plan kernel builds
// from the counts, with the same number of 64-key tiles in every split of
// every head.  A CTA takes one split, brings its tiles in by TMA (three-stage
// ring, 128-byte swizzle, read back with ldmatrix), keeps a running (max,
// sum, output) per query and writes it as a partial; the partials of a head
// merge in a two-level tree (the last CTA of each group of 16 splits, then
// the last group merger).
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
constexpr int kDecMaxSplits = 256;           // splits per head (two merge levels of 16)
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

// Splits are merged by a two-level tree: the last CTA to finish in each group
// of kDecGroup consecutive splits of a head merges that group, and the last
// group merger merges the groups.  A merge loads all its partials at once, so
// it costs about one L2 round trip per level, whatever the head's split count.
constexpr int kDecGroup = 16;
static_assert(kDecGroup * kDecGroup >= kDecMaxSplits, "two levels cover every head");
static_assert(kDecGMax * kDecGroup == kDecThreads, "one thread per (query, partial) in a merge");

// True in every thread of the CTA that arrives last of `total` at `counter`.
// Each arriving CTA's writes are ordered before its count; the last one
// orders the count before its reads of the others' writes.
__device__ __forceinline__ bool last_arrival(unsigned* counter, int total) {
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(counter, 1u) == static_cast<unsigned>(total - 1);
  __syncthreads();
  const bool last = s_last != 0;
  if (last) __threadfence();
  return last;
}

// Merge cnt <= kDecGroup partials (slots first, first + stride, ...), each a
// (max m_s, sum l_s, output o_s) with o_s relative to m_s, base 2:
// M = max_s m_s, L = sum_s l_s 2^(m_s - M), O = sum_s o_s 2^(m_s - M).
// final: out[b] = O / L and lse2[b] = M + log2 L; else (M, L, O) replaces
// the partial in slot `first` (each thread reads its own elements of that
// slot before writing them).
template <int D>
__device__ void merge_partials(const DecArgs& p, int64_t first, int stride, int cnt, bool final, int b, float* out,
                               float* lse2) {
  __shared__ float s_w[kDecGroup * kDecGMax];
  __shared__ float s_M[kDecGMax], s_L[kDecGMax];
  const int G = p.G, tid = threadIdx.x;
  {
    const int g = tid / kDecGroup, j = tid % kDecGroup;       // 16-lane group per query
    const bool on = g < G && j < cnt;
    float2 ml = make_float2(-INFINITY, 0.0f);
    if (on) ml = __ldcg(&p.part_ml[(first + static_cast<int64_t>(j) * stride) * G + g]);
    float M = ml.x;
#pragma unroll
    for (int o = kDecGroup / 2; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w = on ? exp2f(ml.x - M) : 0.0f;               // m_s is finite for every written partial
    float Ls = ml.y * w;
#pragma unroll
    for (int o = kDecGroup / 2; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    if (g < G) {
      s_w[j * kDecGMax + g] = w;
      if (j == 0) {
        s_M[g] = M;
        s_L[g] = Ls;
      }
    }
  }
  __syncthreads();
  const int E4 = G * D / 4;
  for (int e4 = tid; e4 < E4; e4 += kDecThreads) {
    const int g = (4 * e4) / D;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < kDecGroup; ++j) {
      if (j < cnt) {
        const float4 v =
            __ldcg(reinterpret_cast<const float4*>(p.part_o + (first + static_cast<int64_t>(j) * stride) * G * D) + e4);
        const float w = s_w[j * kDecGMax + g];
        acc.x = fmaf(v.x, w, acc.x);
        acc.y = fmaf(v.y, w, acc.y);
        acc.z = fmaf(v.z, w, acc.z);
        acc.w = fmaf(v.w, w, acc.w);
      }
    }
    if (final) {
      const float Lg = s_L[g];
      reinterpret_cast<float4*>(out + static_cast<int64_t>(b) * G * D)[e4] =
          make_float4(acc.x / Lg, acc.y / Lg, acc.z / Lg, acc.w / Lg);
    } else {
      reinterpret_cast<float4*>(p.part_o + first * G * D)[e4] = acc;
    }
  }
  if (tid < G) {
    if (final) {
      if (lse2 != nullptr) lse2[static_cast<int64_t>(b) * G + tid] = s_M[tid] + log2f(s_L[tid]);
    } else {
      p.part_ml[first * G + tid] = make_float2(s_M[tid], s_L[tid]);
    }
  }
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

  const DecItem it = p.items[blockIdx.x];
  const int n = it.n;                                         // tiles of this split
  if (n <= 0) return;                                         // uniform: no work in this item
  const int b = it.b, sp = it.sp, t0 = it.t0, count = it.count;
  const int64_t off = it.off;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;

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
  if (tid == 0) {                                             // the first tiles are in flight during the Q load
    for (int s = 0; s < kDecStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    for (int i = 0; i < n && i < kDecStages; ++i) issue(i);
  }
  for (int e = tid; e < D; e += kDecThreads) {                // 8 rows of 16-byte chunks; rows >= G zero
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if ((e * 8) / D < G) v = reinterpret_cast<const uint4*>(p.q + static_cast<int64_t>(b) * G * D)[e];
    reinterpret_cast<uint4*>(sQ)[e] = v;
  }
  __syncthreads();

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
  const int64_t part = blockIdx.x;
  const bool single = it.nsp == 1;                            // the split is the whole head: final output
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
    if (single) {
      out[(static_cast<int64_t>(b) * G + g) * D + dd] = acc / Ls;
      if (dd == 0 && lse2 != nullptr) lse2[static_cast<int64_t>(b) * G + g] = M + log2f(Ls);
    } else {
      p.part_o[(part * G + g) * D + dd] = acc;
      if (dd == 0) p.part_ml[part * G + g] = make_float2(M, Ls);
    }
  }
  if (single) return;
  // ---- merge tree: groups of kDecGroup consecutive splits, then the groups
  const int64_t base = part - sp;                             // the head's first split
  const int grp = sp / kDecGroup;
  const int ngrp = (it.nsp + kDecGroup - 1) / kDecGroup;
  const int64_t gfirst = base + static_cast<int64_t>(grp) * kDecGroup;
  if (!last_arrival(&p.gdone[gfirst], min(kDecGroup, it.nsp - grp * kDecGroup))) return;
  merge_partials<D>(p, gfirst, 1, min(kDecGroup, it.nsp - grp * kDecGroup), ngrp == 1, b, out, lse2);
  if (ngrp == 1) return;
  if (!last_arrival(&p.done[b], ngrp)) return;
  merge_partials<D>(p, base, kDecGroup, ngrp, true, b, out, lse2);
}

}  // namespace

namespace {

constexpr int kPlanThreads = 1024;

// Block-wide sums of one value per thread (kPlanThreads threads).
__device__ long long plan_sum(long long v, long long* s_red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
  __syncthreads();
  long long t = 0;
  for (int w = 0; w < kPlanThreads / 32; ++w) t += s_red[w];
  return t;
}

// Tiles of head h, or -1 for a count outside [0, n_c].
__device__ int plan_tiles(const DecArgs& p, int h) {
  const int c = p.counts[h];
  return (c < 0 || c > p.n_c) ? -1 : (c + kDecKeys - 1) / kDecKeys;
}

// The decode work list (one CTA).  Every split of every head takes the same
// number of 64-key tiles, cps, so the CTAs carry equal work whatever the
// heads' counts (a global selection leaves them uneven).  cps is the
// smallest value that fits all tiles into about kDecWave CTAs and gives no
// head more than kDecMaxSplits splits.  Then sum_b ceil(tiles_b / cps) <=
// kDecWave + B items, the grid size.  Heads with no kept rows are written
// here (out = 0, lse2 = -inf); the finished-split counters are zeroed.
template <int D>
__global__ void __launch_bounds__(kPlanThreads) decode_plan_kernel(DecArgs p, float* out, float* lse2) {
  __shared__ long long s_red[kPlanThreads / 32];
  __shared__ int s_scan[kPlanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  long long tot = 0, mx = 0;
  for (int h = tid; h < p.B; h += kPlanThreads) {
    const int t = plan_tiles(p, h);
    if (t > 0) {
      tot += t;
      mx = max(mx, static_cast<long long>(t));
    }
  }
  tot = plan_sum(tot, s_red);
  long long m = mx;
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __syncthreads();
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  for (int w = 0; w < kPlanThreads / 32; ++w) mx = max(mx, s_red[w]);
  long long cps = (tot + kDecWave - 1) / kDecWave;
  cps = max(cps, (mx + kDecMaxSplits - 1) / kDecMaxSplits);
  cps = max(cps, 1ll);

  const int c32 = static_cast<int>(cps);                      // <= ceil(n_c / 64)
  __shared__ int s_base[kPlanThreads], s_nsp[kPlanThreads], s_t[kPlanThreads];

  // exclusive scan of the heads' split counts, kPlanThreads heads at a time;
  // then one warp per head writes the head's items, a lane per split
  int carry = 0;
  for (int h0 = 0; h0 < p.B; h0 += kPlanThreads) {
    const int h = h0 + tid;
    const int t = h < p.B ? plan_tiles(p, h) : 0;
    const int nsp = t > 0 ? (t + c32 - 1) / c32 : 0;
    int inc = nsp;                                            // inclusive scan in the warp
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    __syncthreads();                                          // the previous chunk's shared arrays are read
    if (lane == 31) s_scan[warp] = inc;
    __syncthreads();
    int before = carry;
    for (int w = 0; w < warp; ++w) before += s_scan[w];
    int chunk = 0;
    for (int w = 0; w < kPlanThreads / 32; ++w) chunk += s_scan[w];
    s_base[tid] = before + inc - nsp;
    s_nsp[tid] = nsp;
    s_t[tid] = t;
    if (h < p.B) {
      p.done[h] = 0u;
      if (t < 0 && p.status != nullptr) atomicCAS(p.status, 0, KVZ_ERR_INVALID_ARG);
    }
    __syncthreads();
    const int nh = min(kPlanThreads, p.B - h0);
    for (int hh = warp; hh < nh; hh += kPlanThreads / 32) {
      const int hb = h0 + hh, th = s_t[hh], nb = s_nsp[hh], base = s_base[hh];
      if (th == 0) {                                          // no kept rows: out = 0, lse2 = -inf
        for (int e = lane; e < p.G * D; e += 32) out[static_cast<int64_t>(hb) * p.G * D + e] = 0.0f;
        if (lse2 != nullptr && lane < p.G) lse2[static_cast<int64_t>(hb) * p.G + lane] = -INFINITY;
      }
      if (nb <= 0) continue;
      const int cnt = p.counts[hb];
      const long long offb = p.offsets[hb];
      for (int sp = lane; sp < nb && base + sp < p.n_items; sp += 32) {   // the bound always holds; a guard
        DecItem it;
        it.b = hb;
        it.sp = sp;
        it.t0 = sp * c32;
        it.n = min(c32, th - sp * c32);
        it.count = cnt;
        it.nsp = nb;
        it.off = offb;
        p.items[base + sp] = it;
      }
    }
    carry += chunk;
  }
  for (int i = tid; i < p.n_items; i += kPlanThreads) p.gdone[i] = 0u;   // group counters
  // the items past the last split do nothing
  for (int i = carry + tid; i < p.n_items; i += kPlanThreads) {
    DecItem it{};
    it.b = -1;
    p.items[i] = it;
  }
}

template <int D>
cudaError_t launch_split(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecArgs& a, float* out, float* lse2,
                         cudaStream_t stream) {
  decode_plan_kernel<D><<<1, kPlanThreads, 0, stream>>>(a, out, lse2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = smem_limit_once<decode_split_kernel<D>>(DecLay<D>::SMEM);
  if (e != cudaSuccess) return e;
  decode_split_kernel<D><<<a.n_items, kDecThreads, DecLay<D>::SMEM, stream>>>(tmK, tmV, a, out, lse2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(int d, const CUtensorMap& tmK, const CUtensorMap& tmV, const DecArgs& a, float* out,
                          float* lse2, cudaStream_t stream) {
  return d == 128 ? launch_split<128>(tmK, tmV, a, out, lse2, stream)
                  : launch_split<64>(tmK, tmV, a, out, lse2, stream);
}

}  // namespace kvz
