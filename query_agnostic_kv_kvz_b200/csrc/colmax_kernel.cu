// KVzip scoring, pass 2: the context-key column max (KVzip analysis report,
// §3.2: S[j] = max over the grouped queries g and input rows i of the
// softmax row values A[g, i, j], sliced to the n_c context keys).
//
// With pass 1's per-row lse2_r = log2 sum_{u visible} 2^(c2 <q_r,k_u>) and
// c2 = scale * log2(e):
//     S[j] = 2^( c2 * max_r ( <q_r, k_j> - lse2_r / c2 ) ).
// Context keys are visible to every input row, so there is no mask.
//
// The per-row subtraction is folded into the MMA.  Besides the d/16 k-steps
// of <q, k>, each row tile gets one extra K=16 step: the query side holds
// x_r = -lse2_r / c2 split exactly into three bf16 parts (h + m + l = x_r),
// the key side holds ones in the same three columns.  The accumulator then
// is <q_r, k_j> + x_r, and the epilogue is a plain running max.  This keeps
// the per-(row, key) work off the load/store unit: broadcasting lse2 from
// shared memory costs one wavefront per 32 pairs, as much as the tensor
// core's whole pair rate.
//
// CTA = (head b, 256 context keys as two resident 128-key A tiles, a range
// of 256-row query tiles).  MMA: M = 128 keys, N = 256 rows, K = 16, bf16 ->
// fp32 in TMEM; keys are TMEM lanes, so each epilogue thread owns one key.
// Warps: 0 TMA producer, 1 MMA issuer, 2 TMEM owner, 3 builds the -lse2/c2
// block of each tile, 4..19 epilogue (two warpgroups per accumulator, each
// reading half of its 256 columns).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kvz_internal.h"
#include "kvz_sm100.cuh"

namespace kvz {

namespace {

constexpr int kThreads = 640;
constexpr int kKeys = 128;                 // keys per A tile (MMA M)
constexpr int kRows = 256;                 // query rows per tile (MMA N)
constexpr int kNumA = 2;                   // A tiles per CTA
constexpr int kBlk64 = 64 * 2;             // bytes of one 64-column bf16 row slice
constexpr uint32_t kIdesc = idesc_bf16_f32(kKeys, kRows);
constexpr int kK16Bytes = 32;              // one K=16 row slice of the extra block
constexpr int kOnesBytes = kKeys * kK16Bytes;   // 4 KB
constexpr int kAugBytes = kRows * kK16Bytes;    // 8 KB

template <int D>
struct Lay {
  static constexpr int KB = D / 64;                          // 64-column blocks
  static constexpr int A_BLK = kKeys * kBlk64;               // 16 KB: one A k-block
  static constexpr int A_TILE = KB * A_BLK;
  static constexpr int Q_BLK = kRows * kBlk64;               // 32 KB: one Q k-block
  static constexpr int Q_TILE = KB * Q_BLK;
  static constexpr int QST = D == 128 ? 2 : 4;               // Q-tile ring depth
  static constexpr int LST = 4;                              // lse2-slice ring depth
  static constexpr int A_OFF = 0;
  static constexpr int ONES_OFF = A_OFF + kNumA * A_TILE;
  static constexpr int Q_OFF = ONES_OFF + kOnesBytes;
  static constexpr int AUG_OFF = Q_OFF + QST * Q_TILE;
  static constexpr int L_OFF = AUG_OFF + QST * kAugBytes;
  static constexpr int BAR_OFF = L_OFF + LST * kRows * 4;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM = BAR_OFF + BAR_BYTES + 1024;
};
static_assert(Lay<128>::SMEM <= 232448, "shared memory budget");
static_assert(Lay<64>::SMEM <= 232448, "shared memory budget");

// k-step k (16 bf16 of K) of a K-major tile with 128-byte swizzle whose
// 64-column blocks are `blk` bytes apart.
__device__ __forceinline__ uint64_t kstep(const uint8_t* tile, int blk, int k) {
  return sdesc_kmajor_sw128(smem_u32(tile + (k >> 2) * blk + (k & 3) * 32));
}

// Row r's first 16-byte chunk in a no-swizzle K=16 block.
__device__ __forceinline__ int k16_row_offset(int r) { return (r >> 3) * 256 + (r & 7) * 16; }

__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    colmax_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc, ColArgs p) {
  using L = Lay<D>;
  const int u = blockIdx.x;
  const int kblk = u % p.n_kblk;
  const int rest = u / p.n_kblk;
  const int sp = rest % p.nsplit;
  const int b = rest / p.nsplit;
  const int tpg = static_cast<int>(p.rows_pad / kRows);   // row tiles per group
  const int T = p.G * tpg;
  const int t_begin = sp * p.tiles_per_split;
  const int t_end = min(T, t_begin + p.tiles_per_split);
  const int ntile = t_end - t_begin;
  if (ntile <= 0) return;                                  // uniform for the CTA

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem + L::A_OFF;
  uint8_t* sOnes = smem + L::ONES_OFF;
  uint8_t* sQ = smem + L::Q_OFF;
  uint8_t* sAug = smem + L::AUG_OFF;
  float* sL = reinterpret_cast<float*>(smem + L::L_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* a_full = bars + 0;
  uint64_t* q_full = bars + 1;                   // [QST] Q tile landed (TMA)
  uint64_t* q_empty = q_full + L::QST;           // [QST] MMAs done with Q tile and its -lse2/c2 block
  uint64_t* aug_full = q_empty + L::QST;         // [QST] -lse2/c2 block written
  uint64_t* l_full = aug_full + L::QST;          // [LST] lse2 slice landed
  uint64_t* l_empty = l_full + L::LST;           // [LST] slice consumed
  uint64_t* acc_full = l_empty + L::LST;         // [2] accumulator a ready
  uint64_t* acc_empty = acc_full + 2;            // [2] accumulator a drained
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t key0 = static_cast<int64_t>(kblk) * (kNumA * kKeys);

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < L::QST; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&aug_full[s], 1);
    }
    for (int s = 0; s < L::LST; ++s) {
      mbar_init(&l_full[s], 1);
      mbar_init(&l_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);              // the 8 epilogue warps reading accumulator a
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // The key side of the extra k-step: ones in columns 0..2.  The query-side
  // blocks start as zeros; only their first three columns change per tile.
  {
    const uint4 ones = make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int r = threadIdx.x; r < kKeys; r += kThreads) {
      *reinterpret_cast<uint4*>(sOnes + k16_row_offset(r)) = ones;
      *reinterpret_cast<uint4*>(sOnes + k16_row_offset(r) + 128) = zero;
    }
    for (int e = threadIdx.x; e < L::QST * kAugBytes / 16; e += kThreads)
      reinterpret_cast<uint4*>(sAug)[e] = zero;
    fence_proxy_async_smem();
  }
  if (warp == 2) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  int issued = 0;     // Q tiles whose loads were issued (producer thread)
  int l_issued = 0;   // lse2 slices whose loads were issued
  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmKc);
      mbar_arrive_expect_tx(a_full, kNumA * L::A_TILE);
      for (int a = 0; a < kNumA; ++a)
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_4d(sA + a * L::A_TILE + kb * L::A_BLK, &tmKc, a_full, kb * 64,
                      static_cast<int>(key0 + a * kKeys), b % p.T, b / p.T);
      for (int n = 0; n < ntile; ++n) {
        const int s = n % L::QST;
        const uint32_t use = static_cast<uint32_t>(n / L::QST);
        const int sl = n % L::LST;
        const uint32_t luse = static_cast<uint32_t>(n / L::LST);
        const int tau = t_begin + n;
        const int g = tau / tpg;
        const int il = (tau % tpg) * kRows;
        const int bgq = b * p.G + g;
        if (!mbar_wait(&q_empty[s], (use & 1u) ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&q_full[s], L::Q_TILE);
        for (int kb = 0; kb < L::KB; ++kb)
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(sQ + s * L::Q_TILE + kb * L::Q_BLK + hf * (kRows / 2) * kBlk64, &tmQ, &q_full[s],
                        kb * 64, static_cast<int>(p.i_begin + il + hf * (kRows / 2)), bgq);
        issued = n + 1;
        if (!mbar_wait(&l_empty[sl], (luse & 1u) ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&l_full[sl], kRows * 4);
        bulk_load(sL + sl * kRows, p.lse2 + static_cast<int64_t>(bgq) * p.ld + il, kRows * 4, &l_full[sl]);
        l_issued = n + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(a_full, 0, abort_flag, p.status);
      tc_fence_after();
      const uint64_t ones_desc = sdesc_kmajor_k16_noswizzle(smem_u32(sOnes));
      for (int n = 0; ok && n < ntile; ++n) {
        const int s = n % L::QST;
        const uint32_t use = static_cast<uint32_t>(n / L::QST);
        if (!mbar_wait(&q_full[s], use & 1u, abort_flag, p.status)) break;
        if (!mbar_wait(&aug_full[s], use & 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint8_t* q_tile = sQ + s * L::Q_TILE;
        const uint64_t aug_desc = sdesc_kmajor_k16_noswizzle(smem_u32(sAug + s * kAugBytes));
        for (int a = 0; a < kNumA; ++a) {
          if (!mbar_wait(&acc_empty[a], (static_cast<uint32_t>(n) & 1u) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(a * kRows);
          const uint8_t* a_tile = sA + a * L::A_TILE;
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            tc_mma_bf16(d_tmem, kstep(a_tile, L::A_BLK, k), kstep(q_tile, L::Q_BLK, k), kIdesc, k > 0 ? 1u : 0u);
          tc_mma_bf16(d_tmem, ones_desc, aug_desc, kIdesc, 1u);     // + (-lse2_r / c2)
          tc_commit(&acc_full[a]);
        }
        if (!ok) break;
        tc_commit(&q_empty[s]);
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------ -lse2/c2 blocks
    const float inv_c2 = 1.0f / p.c2;
    for (int n = 0; n < ntile; ++n) {
      const int s = n % L::QST;
      const uint32_t use = static_cast<uint32_t>(n / L::QST);
      const int sl = n % L::LST;
      const uint32_t luse = static_cast<uint32_t>(n / L::LST);
      if (!mbar_wait_warp(&q_empty[s], (use & 1u) ^ 1u, abort_flag, p.status)) break;
      if (!mbar_wait_warp(&l_full[sl], luse & 1u, abort_flag, p.status)) break;
      uint8_t* aug = sAug + s * kAugBytes;
#pragma unroll
      for (int i = 0; i < kRows / 32; ++i) {
        const int r = lane + 32 * i;
        const float x = -sL[sl * kRows + r] * inv_c2;    // -inf for padding rows
        __nv_bfloat16 h, m, l;
        if (x == -INFINITY) {
          h = __float2bfloat16_rn(x);
          m = __float2bfloat16_rn(0.0f);
          l = m;
        } else {                                          // exact: h + m + l == x
          h = __float2bfloat16_rn(x);
          const float r1 = x - __bfloat162float(h);
          m = __float2bfloat16_rn(r1);
          l = __float2bfloat16_rn(r1 - __bfloat162float(m));
        }
        *reinterpret_cast<uint4*>(aug + k16_row_offset(r)) =
            make_uint4(pack_bf16x2(h, m), pack_bf16x2(l, __float2bfloat16_rn(0.0f)), 0u, 0u);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&aug_full[s]);
        mbar_arrive(&l_empty[sl]);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue: running max
    const int ew = warp - 4;
    const int a = ew >> 3;                     // accumulator (key tile)
    const int h = (ew >> 2) & 1;               // which 128 of the 256 row columns
    const int wq = warp & 3;
    const int64_t j = key0 + a * kKeys + wq * 32 + lane;     // context key == TMEM lane
    const uint32_t tbase = tmem + (static_cast<uint32_t>(wq * 32) << 16) + static_cast<uint32_t>(a * kRows + h * 128);
    float y0 = -INFINITY, y1 = -INFINITY;      // max over rows of <q_r, k_j> - lse2_r / c2
    bool ok = true;
    for (int n = 0; n < ntile; ++n) {
      if (!mbar_wait_warp(&acc_full[a], static_cast<uint32_t>(n) & 1u, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float v[64];
      tmem_ld64(tbase, v);
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        y0 = fmax3(y0, v[c], v[c + 1]);
        y1 = fmax3(y1, v[c + 2], v[c + 3]);
      }
      tmem_ld64(tbase + 64, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);   // the accumulator is free once read
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        y0 = fmax3(y0, v[c], v[c + 1]);
        y1 = fmax3(y1, v[c + 2], v[c + 3]);
      }
    }
    if (ok && j < p.n_c) {
      const float sj = exp2f(p.c2 * fmaxf(y0, y1));   // >= +0: its bit pattern orders like the value
      float* dst = p.S + static_cast<int64_t>(b / p.T) * p.ldS + static_cast<int64_t>(b % p.T) * p.s_block + j;
      atomicMax(reinterpret_cast<unsigned int*>(dst), __float_as_uint(sj));
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // Unwinding after a timeout: let this CTA's copies and MMAs finish (bounded).
    if (warp == 0 && lane == 0) {
      mbar_wait_for(a_full, 0, 20000000ull);
      for (int s = 0; s < L::QST && s < issued; ++s) {
        const int n_last = s + L::QST * ((issued - 1 - s) / L::QST);
        mbar_wait_for(&q_full[s], static_cast<uint32_t>(n_last / L::QST) & 1u, 20000000ull);
      }
      for (int s = 0; s < L::LST && s < l_issued; ++s) {
        const int n_last = s + L::LST * ((l_issued - 1 - s) / L::LST);
        mbar_wait_for(&l_full[s], static_cast<uint32_t>(n_last / L::LST) & 1u, 20000000ull);
      }
    }
    if (warp == 1 && lane == 0) {
      tc_commit(drain);
      mbar_wait_for(drain, 0, 20000000ull);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_colmax(int d, const CUtensorMap& tmQ, const CUtensorMap& tmKc, const ColArgs& args,
                          cudaStream_t stream) {
  ColArgs a = args;
  constexpr int kNumSMs = 148;
  a.n_kblk = static_cast<int>((a.n_c + kNumA * kKeys - 1) / (kNumA * kKeys));
  // Split each (head, key block)'s row tiles so the grid fills ~8 waves.
  const int64_t T = static_cast<int64_t>(a.G) * (a.rows_pad / kRows);
  const int64_t base_units = static_cast<int64_t>(a.B) * a.n_kblk;
  int64_t nsplit = (kNumSMs * 8 + base_units - 1) / base_units;
  const int64_t max_split = T / 4 > 1 ? T / 4 : 1;
  if (nsplit > max_split) nsplit = max_split;
  if (nsplit < 1) nsplit = 1;
  const int64_t tps = (T + nsplit - 1) / nsplit;
  nsplit = (T + tps - 1) / tps;
  const int64_t grid = base_units * nsplit;
  if (grid <= 0 || grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  a.nsplit = static_cast<int>(nsplit);
  a.tiles_per_split = static_cast<int>(tps);
  cudaError_t e;
  if (d == 128) {
    e = smem_limit_once<colmax_kernel<128>>(Lay<128>::SMEM);
    if (e != cudaSuccess) return e;
    colmax_kernel<128><<<static_cast<unsigned>(grid), kThreads, Lay<128>::SMEM, stream>>>(tmQ, tmKc, a);
  } else {
    e = smem_limit_once<colmax_kernel<64>>(Lay<64>::SMEM);
    if (e != cudaSuccess) return e;
    colmax_kernel<64><<<static_cast<unsigned>(grid), kThreads, Lay<64>::SMEM, stream>>>(tmQ, tmKc, a);
  }
  return cudaGetLastError();
}

}  // namespace kvz
