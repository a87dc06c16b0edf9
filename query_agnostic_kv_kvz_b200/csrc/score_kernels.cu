// KVzip context-reconstruction scoring on sm_100a (tcgen05 + TMEM + TMA):
// pass 1 and shared launch helpers; pass 2 lives in colmax_kernel.cu.
//
// KVzip (analysis report, §3.2 "KV importance scoring", equation for S_{l,h}):
//   A = Softmax(Q K^T) over the n_c + n_in keys of the repeat-prompt + context
//   input, sliced to the n_c context keys; S[j] = max_{g,i} A[g,i,j].
// With c2 = scale * log2(e) and lse2_r = log2 sum_{u visible} 2^(c2 <q_r,k_u>):
//   A[r, j] = 2^(c2 <q_r, k_j> - lse2_r)  and, exp2 being monotone,
//   S[j]    = 2^( max_r (c2 <q_r, k_j> - lse2_r) ).
// Two passes, neither materialising the G*n_in x (n_c+n_in) matrix:
//   pass 1 (lse_kernel):    one thread per query row, a running sum of
//                           exp2 against a per-row reference over key tiles
//                           (no P.V, no per-tile max);
//   pass 2 (colmax_kernel): keys in TMEM lanes, one thread per context key,
//                           running max over query-row columns; no mask
//                           because every row sees every context key.
// Both kernels: warp 0 issues TMA loads, warp 1 (one thread) issues
// tcgen05.mma into tensor memory, warp 2 owns the TMEM allocation, warps
// 4..19 (four warpgroups, each owning half of a tile's 128 TMEM columns)
// read TMEM and do the softmax / max arithmetic.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kvz_internal.h"
#include "kvz_sm100.cuh"

namespace kvz {

namespace {

constexpr int kThreads = 640;     // 4 control warps + 4 epilogue warpgroups
constexpr int kTile = 128;        // rows of a Q sub-tile / keys of a K tile
constexpr int kSubBytes64 = kTile * 128;  // one 128-row x 64-column bf16 block (16 KB)
constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128);

// Of every 16 exp2 evaluations in pass 1, how many run as a polynomial on
// the FMA pipe instead of the SFU (even, 0..16).
#ifndef KVZ_POLY_PER16
#define KVZ_POLY_PER16 2
#endif
constexpr int kPolyPer16 = KVZ_POLY_PER16;

// 1: each Q sub-tile's MMAs are issued by its own thread (warp 1: sub-tile
// 0, warp 3: sub-tile 1), so the two sub-tiles' softmax warpgroups are
// coupled only through the shared K ring; 0: one thread issues both.
#ifndef KVZ_LSE_SPLIT_ISSUE
#define KVZ_LSE_SPLIT_ISSUE 0
#endif
static_assert(kPolyPer16 % 2 == 0 && kPolyPer16 >= 0 && kPolyPer16 <= 16, "pairs of exp2");

template <int D>
struct LseLayout {
  static constexpr int KB = D / 64;                      // 64-column blocks per row
  static constexpr int TILE_BYTES = KB * kSubBytes64;    // 128 rows x D
  static constexpr int NQ = 2;                           // Q sub-tiles per CTA
  static constexpr int KST = 4;                          // K-tile pipeline depth
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NQ * TILE_BYTES;
  static constexpr int MERGE_OFF = K_OFF + KST * TILE_BYTES;  // (max, sum) of the second column half
  static constexpr int BAR_OFF = MERGE_OFF + NQ * kTile * 2 * 4;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = BAR_OFF + BAR_BYTES + 1024;  // + alignment slack
};



// Row block and (head, group) of pass-1 unit u.  Both orders put a head's
// later (longer) row blocks first.  Row-block-major is longest-first over
// the whole grid; head-major keeps the CTAs running at one time on one or
// two heads, so they share those heads' key tiles in L2 (chosen when the
// units are nearly equal in length).
__device__ __forceinline__ void lse_unit(const LseArgs& p, int u, int nblk, int& iblk, int& bg) {
  if (p.head_major) {
    const int per_head = nblk * p.G;
    const int b = u / per_head;
    const int rem = u - b * per_head;
    iblk = nblk - 1 - rem / p.G;
    bg = b * p.G + rem % p.G;
  } else {
    const int BG = p.B * p.G;
    iblk = nblk - 1 - u / BG;
    bg = u % BG;
  }
}

// Max of a thread's 64 logits of a tile (two independent chains of 3-input
// max).
__device__ __forceinline__ float tile_max64(const float (&v)[64]) {
  float mx[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    float a = v[32 * k];
#pragma unroll
    for (int c = 1; c < 31; c += 2) a = fmax3(a, v[32 * k + c], v[32 * k + c + 1]);
    mx[k] = fmaxf(a, v[32 * k + 31]);
  }
  return fmaxf(mx[0], mx[1]);
}

// Sum over a thread's 64 logits of 2^(c2 * s - m): 16 - kPolyPer16 of every
// 16 exp2 on the SFU, the rest on the FMA pipe as a polynomial, so neither
// unit limits the pass on its own.  `pmax` gets the largest polynomial
// input: the polynomial builds 2^n in the exponent bits and is only valid
// for inputs up to 127 (the SFU returns +inf above its range).
__device__ __forceinline__ float exp2_sum64(const float (&v)[64], float c2, float m, float& pmax) {
  const float2 c22 = make_float2(c2, c2);
  const float2 nm2 = make_float2(-m, -m);
  float2 s0 = make_float2(0.f, 0.f), s1 = s0, s2 = s0;
  float pm = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; c += 16) {
#pragma unroll
    for (int k = 0; k < 16 - kPolyPer16; k += 2) {
      const float2 x = __ffma2_rn(make_float2(v[c + k], v[c + k + 1]), c22, nm2);
      const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      if (k & 2) s0 = __fadd2_rn(s0, e); else s1 = __fadd2_rn(s1, e);
    }
#pragma unroll
    for (int k = 16 - kPolyPer16; k < 16; k += 2) {
      const float2 x = __ffma2_rn(make_float2(v[c + k], v[c + k + 1]), c22, nm2);
      pm = fmax3(pm, x.x, x.y);
      s2 = __fadd2_rn(s2, exp2_poly2(x));
    }
  }
  pmax = pm;
  return ((s0.x + s0.y) + (s1.x + s1.y)) + (s2.x + s2.y);
}

// 2^n for an integer-valued n <= 0, exactly (0 below the normal range).
__device__ __forceinline__ float exp2_int_nonpos(float n) {
  const int e = static_cast<int>(n) + 127;
  return e > 0 ? __int_as_float(e << 23) : 0.0f;
}

// Descriptor of k-step `k` (16 bf16 of K) of a 128-row tile at `tile`.
__device__ __forceinline__ uint64_t kstep_desc(const uint8_t* tile, int k) {
  return sdesc_kmajor_sw128(smem_u32(tile + (k >> 2) * kSubBytes64 + (k & 3) * 32));
}

// ============================================================================
// Pass 1: lse2 of every input row in [i_begin, i_end).
// Unit = (head b, group g, 256 input rows = two 128-row sub-tiles), numbered
// longest-first (rows late in the input see more keys).  A CTA computes a
// whole unit, or (units of the partial last wave) one of `nsplit`
// consecutive ranges of the unit's key tiles, writing its rows' partial
// (max, sum) for lse_merge_kernel.
// ============================================================================
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    lse_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
               const __grid_constant__ CUtensorMap tmKi, LseArgs p) {
  using Lay = LseLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + Lay::Q_OFF;
  uint8_t* sK = smem + Lay::K_OFF;
  float* sMerge = reinterpret_cast<float*>(smem + Lay::MERGE_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                  // [KST]
  uint64_t* k_empty = k_full + Lay::KST;        // [KST]
  uint64_t* s_full = k_empty + Lay::KST;        // [2 sub-tiles][2 buffers]
  uint64_t* s_empty = s_full + 4;               // [2][2]
  uint64_t* drain = s_empty + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit (longest first) and this CTA's range of its key tiles ----
  const int nblk = static_cast<int>(p.rows_pad / 256);
  const int x = blockIdx.x;
  const bool split = x >= p.n_full;
  const int u = split ? p.n_full + (x - p.n_full) / p.nsplit : x;
  const int part = split ? (x - p.n_full) % p.nsplit : 0;
  int iblk, bg;
  lse_unit(p, u, nblk, iblk, bg);
  const int b = bg / p.G;
  const int64_t i0 = p.i_begin + static_cast<int64_t>(iblk) * 256;
  const int64_t row_hi = p.i_end;               // rows >= row_hi are padding
  const int nq_valid = (i0 + kTile < row_hi) ? 2 : 1;
  const int NC = static_cast<int>((p.n_c + kTile - 1) / kTile);
  int nin[2];
  nin[0] = static_cast<int>(i0 / kTile) + 1;
  nin[1] = static_cast<int>((i0 + kTile) / kTile) + 1;
  const int NT = NC + nin[nq_valid - 1];                 // the unit's key tiles: context, then input
  const int t_lo = split ? static_cast<int>(static_cast<int64_t>(NT) * part / p.nsplit) : 0;
  const int NL = (split ? static_cast<int>(static_cast<int64_t>(NT) * (part + 1) / p.nsplit) : NT) - t_lo;
  // Head-major order: when a head's CTAs span several waves, each wave
  // walks the head's key tiles in the direction opposite to the wave before
  // it, so it starts on the tiles that wave read last, which are still in
  // L2.  Every loop below maps its local index j to tile tile_of(j).
  bool rev = false;
  if (p.head_major && p.wave > 0) {
    const int u0 = b * nblk * p.G;
    const int x0 = u0 < p.n_full ? u0 : p.n_full + (u0 - p.n_full) * p.nsplit;
    rev = ((x / p.wave - x0 / p.wave) & 1) != 0;
  }
  auto tile_of = [rev, t_lo, NL](int j) { return rev ? t_lo + NL - 1 - j : t_lo + j; };

  const int n_issuers = KVZ_LSE_SPLIT_ISSUE ? nq_valid : 1;   // threads that commit to k_empty / drain
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < Lay::KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], n_issuers);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 8);                // 8 softmax warps read each buffer
    }
    mbar_init(drain, n_issuers);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  int issued = 0;   // K tiles whose TMA loads were issued (producer thread)
  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmKc);
      prefetch_tmap(&tmKi);
      mbar_arrive_expect_tx(q_full, nq_valid * Lay::TILE_BYTES);
      for (int q = 0; q < nq_valid; ++q)
        for (int kb = 0; kb < Lay::KB; ++kb)
          tma_load_3d(sQ + q * Lay::TILE_BYTES + kb * kSubBytes64, &tmQ, q_full, kb * 64,
                      static_cast<int>(i0 + q * kTile), bg);
      for (int j = 0; j < NL; ++j) {                   // ring slots follow the local tile index j
        const int t = tile_of(j);
        const int s = j % Lay::KST;
        const uint32_t use = static_cast<uint32_t>(j / Lay::KST);
        if (!mbar_wait(&k_empty[s], (use & 1u) ^ 1u, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&k_full[s], Lay::TILE_BYTES);
        for (int kb = 0; kb < Lay::KB; ++kb) {
          if (t < NC)   // context keys: block (b % T) of head (b / T)
            tma_load_4d(sK + s * Lay::TILE_BYTES + kb * kSubBytes64, &tmKc, &k_full[s], kb * 64, t * kTile,
                        b % p.T, b / p.T);
          else
            tma_load_3d(sK + s * Lay::TILE_BYTES + kb * kSubBytes64, &tmKi, &k_full[s], kb * 64,
                        (t - NC) * kTile, b);
        }
        issued = j + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1 || (KVZ_LSE_SPLIT_ISSUE && warp == 3)) {
    // ------------------------------------------------ MMA issuer(s)
    const int q_lo = KVZ_LSE_SPLIT_ISSUE && warp == 3 ? 1 : 0;
    const int q_hi = KVZ_LSE_SPLIT_ISSUE ? q_lo + 1 : 2;
    if (lane == 0 && q_lo < nq_valid) {
      uint32_t cnt[2] = {0u, 0u};
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
      tc_fence_after();
      for (int j = 0; ok && j < NL; ++j) {
        const int t = tile_of(j);
        const int s = j % Lay::KST;
        const uint32_t use = static_cast<uint32_t>(j / Lay::KST);
        if (!mbar_wait(&k_full[s], use & 1u, abort_flag, p.status)) break;
        tc_fence_after();
        for (int q = q_lo; q < q_hi && q < nq_valid; ++q) {
          if (t >= NC && t - NC >= nin[q]) continue;
          const uint32_t buf = cnt[q] & 1u;
          const uint32_t bu = cnt[q] >> 1;
          if (!mbar_wait(&s_empty[q * 2 + buf], (bu & 1u) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>((q * 2 + buf) * kTile);
          const uint8_t* a_tile = sQ + q * Lay::TILE_BYTES;
          const uint8_t* b_tile = sK + s * Lay::TILE_BYTES;
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            tc_mma_bf16(d_tmem, kstep_desc(a_tile, k), kstep_desc(b_tile, k), kIdesc, k > 0 ? 1u : 0u);
          tc_commit(&s_full[q * 2 + buf]);
          ++cnt[q];
        }
        tc_commit(&k_empty[s]);
      }
    }
    __syncwarp();
  }

  // ------------------------------------------------ softmax warpgroups
  // Four warpgroups: (sub-tile q, column half h).  A thread owns one query
  // row (its TMEM lane) and 64 of the 128 key columns of every tile; the
  // two halves' (reference, sum) pairs merge exactly at the end.
  // No per-tile max: a row's reference m is the floor of its first tile's
  // max (an integer, so rebasing by powers of two keeps it exact); each
  // tile's exp2s are taken against m directly (the sum is exact for any
  // reference), the sum is renormalised to [1, 2) by an exact power of two
  // once it reaches 2^24, and only a tile with a logit about 100 or more
  // above m (log2 units: its terms overflow, or leave the polynomial's
  // range) is reloaded and redone against its own max.  The tile's
  // accumulator buffer is released after the tile.
  const int ew = warp - 4;
  const int q = (ew >> 3) & 1;
  const int h = (ew >> 2) & 1;
  const int rl = (warp & 3) * 32 + lane;            // row within the sub-tile == TMEM lane
  float m = -INFINITY, l = 0.0f;
  bool ok = true;
  if (warp >= 4 && q < nq_valid) {
    const int wq = warp & 3;
    const float c2 = p.c2;
    const int ctx_tail = static_cast<int>(p.n_c - static_cast<int64_t>(NC - 1) * kTile) - h * 64;
    const int diag_lim = rl - h * 64;                 // diagonal tile: column c visible iff c <= diag_lim
    uint32_t cnt = 0;
    for (int j = 0; j < NL; ++j) {
      const int t = tile_of(j);
      if (t >= NC && t - NC >= nin[q]) continue;
      const uint32_t buf = cnt & 1u;
      const uint32_t bu = cnt >> 1;
      if (!mbar_wait_warp(&s_full[q * 2 + buf], bu & 1u, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(wq * 32) << 16) +
                             static_cast<uint32_t>((q * 2 + buf) * kTile + h * 64);
      const bool tail_tile = t == NC - 1 && ctx_tail < 64;
      const bool diag_tile = t >= NC && t - NC == nin[q] - 1;
      float v[64];
      tmem_ld64(taddr, v);
      if (tail_tile) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= ctx_tail) v[c] = -INFINITY;
      }
      if (diag_tile) {                             // diagonal input tile
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c > diag_lim) v[c] = -INFINITY;
      }
      if (m == -INFINITY) {                        // no reference yet: this tile's max, floored
        const float mt = tile_max64(v) * c2;
        if (mt != -INFINITY) m = floorf(mt);
      }
      float pmax = -INFINITY;
      float l_new = m == -INFINITY ? l : l + exp2_sum64(v, c2, m, pmax);
      // A term overflowed, or a polynomial input left its range (a logit
      // ~100 or more above the row's reference): reload the tile
      // (warp-uniform: tcgen05.ld is a warp collective) and redo those rows
      // against the tile's own max.
      bool redo = !(l_new <= 0x1p100f) || pmax > 100.0f;
      if (__any_sync(0xffffffffu, redo)) {
        tmem_ld64(taddr, v);
        if (tail_tile) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= ctx_tail) v[c] = -INFINITY;
        }
        if (diag_tile) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c > diag_lim) v[c] = -INFINITY;
        }
        if (redo) {
          const float mn = floorf(tile_max64(v) * c2);
          l = l * exp2_int_nonpos(m - mn);
          m = mn;
          l_new = l + exp2_sum64(v, c2, m, pmax);   // inputs now at most 1
        }
      }
      l = l_new;
      if (l >= 0x1p24f) {                          // renormalise to [1, 2): exact
        const int k = ((__float_as_int(l) >> 23) & 0xff) - 127;
        l = __int_as_float(__float_as_int(l) - (k << 23));
        m += static_cast<float>(k);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[q * 2 + buf]);
      ++cnt;
    }
  }
  if (warp >= 4 && h == 1) {
    sMerge[(q * kTile + rl) * 2 + 0] = m;
    sMerge[(q * kTile + rl) * 2 + 1] = ok ? l : -1.0f;
  }

  __syncthreads();
  if (warp >= 4 && h == 0) {
    const int64_t i = i0 + q * kTile + rl;
    const float m1 = sMerge[(q * kTile + rl) * 2 + 0];
    const float l1 = sMerge[(q * kTile + rl) * 2 + 1];
    const bool good = ok && l1 >= 0.0f;
    const float mm = fmaxf(m, m1);
    const float ll = (m == -INFINITY ? 0.0f : l * exp2f(m - mm)) + (m1 == -INFINITY ? 0.0f : l1 * exp2f(m1 - mm));
    if (split) {
      // this range's (max, sum) of the row: (-inf, 0) if it saw no key of
      // the row, sum -1 if the CTA gave up
      p.part[static_cast<int64_t>(x - p.n_full) * 256 + q * kTile + rl] =
          !good ? make_float2(-INFINITY, -1.0f) : (mm == -INFINITY ? make_float2(-INFINITY, 0.0f)
                                                                   : make_float2(mm, ll));
    } else {
      float lse2 = INFINITY;
      if (q < nq_valid && good && i < row_hi) lse2 = mm + log2f(ll);   // finite: every row sees a key
      p.lse2[static_cast<int64_t>(bg) * p.ld + (i - p.i_begin)] = lse2;
    }
  }
  if (*abort_flag) {
    // Unwinding after a timeout: let this CTA's own copies and MMAs finish
    // (bounded) before shared and tensor memory are released.
    if (warp == 0 && lane == 0) {
      mbar_wait_for(q_full, 0, 20000000ull);
      for (int s = 0; s < Lay::KST && s < issued; ++s) {
        const int t_last = s + Lay::KST * ((issued - 1 - s) / Lay::KST);
        mbar_wait_for(&k_full[s], static_cast<uint32_t>(t_last / Lay::KST) & 1u, 20000000ull);
      }
    }
    if ((warp == 1 || (KVZ_LSE_SPLIT_ISSUE && warp == 3 && nq_valid == 2)) && lane == 0) {
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

// Merge the key-range parts of each split unit, in part order (so the
// result does not depend on which part finished first).  Block = one split
// unit, thread = one of its 256 rows.
__global__ void __launch_bounds__(256) lse_merge_kernel(LseArgs p) {
  const int t_unit = blockIdx.x;
  const int row = threadIdx.x;
  const int u = p.n_full + t_unit;
  const int nblk = static_cast<int>(p.rows_pad / 256);
  int iblk, bg;
  lse_unit(p, u, nblk, iblk, bg);
  const int64_t i = p.i_begin + static_cast<int64_t>(iblk) * 256 + row;
  const float2* pr = p.part + static_cast<int64_t>(t_unit) * p.nsplit * 256 + row;
  float mm = -INFINITY;
  bool bad = false;
  for (int k = 0; k < p.nsplit; ++k) {
    const float2 v = pr[static_cast<int64_t>(k) * 256];
    if (v.y < 0.0f) bad = true;
    else if (v.y > 0.0f) mm = fmaxf(mm, v.x);
  }
  float ll = 0.0f;
  for (int k = 0; k < p.nsplit; ++k) {
    const float2 v = pr[static_cast<int64_t>(k) * 256];
    if (v.y > 0.0f) ll += v.y * exp2f(v.x - mm);
  }
  const float lse2 = (bad || i >= p.i_end || !(ll > 0.0f)) ? INFINITY : mm + log2f(ll);
  p.lse2[static_cast<int64_t>(bg) * p.ld + (i - p.i_begin)] = lse2;
}

__global__ void fill_f32_kernel(float* x, int64_t n, float v) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x)
    x[e] = v;
}

}  // namespace

cudaError_t launch_lse(int d, const CUtensorMap& tmQ, const CUtensorMap& tmKc, const CUtensorMap& tmKi,
                       const LseArgs& a_in, cudaStream_t stream) {
  LseArgs a = a_in;
  const int64_t nblk = a.rows_pad / 256;
  const int64_t units = static_cast<int64_t>(a.B) * a.G * nblk;
  if (units <= 0 || units > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  a.n_full = static_cast<int>(units);
  a.nsplit = 1;
  // Head-major when a call's row blocks differ in key count by at most 1/8
  // of the context tiles (row passes much shorter than the context).
  a.head_major = (a.rows_pad / kTile) * 8 <= (a.n_c + kTile - 1) / kTile ? 1 : 0;
  int64_t grid = units, r = 0;
  cudaError_t e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  a.wave = sms;                                     // one CTA per SM
  if (a.part != nullptr) {
    // The units past the last full wave are split over key ranges so that
    // the last wave fills the SMs.  The tail holds the shortest units (row
    // block 0 of the call); a part keeps >= 8 tiles.
    r = sms > 0 ? units % sms : 0;
    if (r > 0) {
      // the shortest tail unit: row block 0 of the call in either order
      const int64_t nt_min = (a.n_c + kTile - 1) / kTile + a.i_begin / kTile + 1;
      int64_t s = sms / r;
      if (s > nt_min / 8) s = nt_min / 8;
      if (s * r > kLseMaxSplitCtas) s = kLseMaxSplitCtas / r;
      if (s >= 2) {
        a.n_full = static_cast<int>(units - r);
        a.nsplit = static_cast<int>(s);
        grid = a.n_full + r * s;
      }
    }
  }
  if (d == 128) {
    e = smem_limit_once<lse_kernel<128>>(LseLayout<128>::SMEM);
    if (e != cudaSuccess) return e;
    lse_kernel<128><<<static_cast<unsigned>(grid), kThreads, LseLayout<128>::SMEM, stream>>>(tmQ, tmKc, tmKi, a);
  } else {
    e = smem_limit_once<lse_kernel<64>>(LseLayout<64>::SMEM);
    if (e != cudaSuccess) return e;
    lse_kernel<64><<<static_cast<unsigned>(grid), kThreads, LseLayout<64>::SMEM, stream>>>(tmQ, tmKc, tmKi, a);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.nsplit > 1) {
    lse_merge_kernel<<<static_cast<unsigned>(r), 256, 0, stream>>>(a);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_fill_f32(float* x, int64_t n, float v, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  fill_f32_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, n, v);
  return cudaGetLastError();
}

}  // namespace kvz
