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

// Launch-shape tuning (measured on B200; override with -D for sweeps).
#ifndef KVZ_GATHER_UNROLL
#define KVZ_GATHER_UNROLL 4
#endif
#ifndef KVZ_GATHER_CTAS_PER_SM
#define KVZ_GATHER_CTAS_PER_SM 8
#endif
#ifndef KVZ_INPLACE_THREADS
#define KVZ_INPLACE_THREADS 128
#endif
#ifndef KVZ_INPLACE_ROWS
#define KVZ_INPLACE_ROWS 16
#endif
#ifndef KVZ_INPLACE_DEPTH
#define KVZ_INPLACE_DEPTH 2
#endif
#ifndef KVZ_INPLACE_OVERSUB
#define KVZ_INPLACE_OVERSUB 3
#endif
#ifndef KVZ_INPLACE_MIN_CTAS
#define KVZ_INPLACE_MIN_CTAS 3
#endif
constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = KVZ_GATHER_UNROLL;
constexpr int kInplaceThreads = KVZ_INPLACE_THREADS;
constexpr int kInplaceRows = KVZ_INPLACE_ROWS;           // slots per chunk (one warp moves a chunk)
constexpr int kInplaceDepth = KVZ_INPLACE_DEPTH;         // chunks in each warp's register ring
constexpr int kInplaceOversub = KVZ_INPLACE_OVERSUB;     // warps launched per resident warp slot
constexpr int kInplaceMinCtas = KVZ_INPLACE_MIN_CTAS;    // resident CTAs per SM the registers must allow
static_assert(kInplaceThreads % 32 == 0, "whole warps");
static_assert(kInplaceDepth >= 2, "a ring holds the chunk being stored and at least one loading");
static_assert(kInplaceRows % 4 == 0, "a warp-wide access covers 2 (d = 128) or 4 (d = 64) rows");
static_assert(kInplaceDepth * kInplaceRows / 2 <= 32, "one validity bit per row, lane and stage in 32 bits");

__device__ __forceinline__ void report_err(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Streaming load through the read-only path: no kernel here reads a row
// after writing it.
__device__ __forceinline__ int4 ld_stream(const int4* p) {
  int4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Coherent streaming load for the in-place kernel, which overwrites rows
// that other warps of the same launch read: a relaxed gpu-scope load stays
// inside the memory model the kernel's ordering argument rests on (the
// read-only .nc path is only for data no thread of the launch writes).
__device__ __forceinline__ int4 ld_coherent(const int4* p) {
  int4 v;
  asm volatile("ld.relaxed.gpu.global.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_relaxed_gpu_add(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// A zero computed from x that the compiler cannot fold: a value built with it
// carries a data dependency on the load that produced x.
__device__ __forceinline__ uint32_t dep_zero(uint32_t x) {
  uint32_t z;
  asm volatile("and.b32 %0, %1, 0;" : "=r"(z) : "r"(x));
  return z;
}
__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
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

// Out of place into int8 (KVzip analysis report, §4.2 "KV quantization": the
// pruned cache composes with a quantised one).  Symmetric per-row codes: with
// a = max |x| over the row, scale = a / 127 and code = rint(x * (127 / a)),
// clamped to [-127, 127]; a row of zeros has code 0 and scale 0.  The two
// divisions and the product are single IEEE float32 operations (no fused or
// approximate forms), so the codes are reproducible to the bit.
// HBM-bound: 4d bytes read, 2d + 8 written per row.
//
// Two threads per row.  A CTA of 256 threads takes units of 64 slots of one
// head: threads 0-127 own the unit's K rows, 128-255 its V rows, a pair of
// adjacent lanes per row, one half of the row each; a shuffle combines the
// pair's absmax.  The rows of the next units arrive by cp.async (coalesced,
// 16 bytes per thread) into a three-stage ring while the current unit is
// quantised.  Each unit's count, offsets and source indices are fetched a
// unit earlier still and carried in registers, and a CTA steps through its
// units without integer division, so nothing between the barriers waits on
// memory or on a 64-bit divide (these two cost 12% of the kernel's time).  A
// thread reads its half row from shared memory twice (absmax, then codes),
// writes the codes into a staging tile, and one bulk copy per tensor stores
// the unit's code rows, which are contiguous in the output.  The 16-byte
// chunks of a staged row are XOR-swizzled and each thread visits its chunks
// in a rotated order, chosen by exhaustive search so that at d = 128 no
// shared-memory access has a bank conflict (at d = 64 some are two-way).
constexpr int kQ8Rows = 64;                                     // slots per unit
constexpr int kQ8Threads = 256;
constexpr int kQ8Stages = 3;                                    // units in the ring: two in flight

template <int D>
struct Q8 {
  static constexpr int VPR = D / 8;                             // 16-byte chunks of a bf16 row
  static constexpr int NCO = D / 16;                            // 16-byte chunks of a code row
  static constexpr int CPH = VPR / 2;                           // input chunks per half row
  static constexpr int COH = NCO / 2;                           // code chunks per half row
  static constexpr int RPT = VPR / 4;                           // rows each thread loads, per tensor
  static constexpr int LSTRIDE = kQ8Threads / VPR;              // loader row stride
  static constexpr int ROWB = D * 2;
  static constexpr int STAGE = 2 * kQ8Rows * ROWB;              // K rows, then V rows
  static constexpr int OUT = 2 * kQ8Rows * D;                   // K codes, then V codes
  static constexpr int SMEM = kQ8Stages * STAGE + OUT;
  // chunk c of staged row r sits at chunk c ^ swz(r)
  __device__ static int swz(int r) { return r & (VPR - 1); }
  // step c of the absmax pass reads input chunk h*CPH + p1(c, r, h); step k
  // of the code pass writes code chunk h*COH + p2(k, r, h)
  __device__ static int p1(int c, int r, int h) { return D == 128 ? ((c + 4 * h) & 7) : c; }
  __device__ static int p2(int k, int r, int h) { return D == 128 ? ((k + r + 2 * h) & 3) : k; }
};

// Codes of 4 bf16 values (w0 = x1:x0, w1 = x3:x2), x0 in the low byte.
// v = x * inv is one IEEE product; adding 1.5 * 2^23 rounds v to the nearest
// integer (ties to even, |v| < 2^22) and leaves that integer in the low bits
// of the sum's pattern, so the code is its low byte.  |x| <= a gives |v| <=
// 127 (1 + 2^-24)^2 < 127.5: the code never leaves [-127, 127].
__device__ __forceinline__ uint32_t code4(uint32_t w0, uint32_t w1, float inv) {
  constexpr float kRound = 12582912.0f;                         // 1.5 * 2^23
  const uint32_t c0 = __float_as_uint(__fadd_rn(__fmul_rn(__uint_as_float(w0 << 16), inv), kRound));
  const uint32_t c1 = __float_as_uint(__fadd_rn(__fmul_rn(__uint_as_float(w0 & 0xFFFF0000u), inv), kRound));
  const uint32_t c2 = __float_as_uint(__fadd_rn(__fmul_rn(__uint_as_float(w1 << 16), inv), kRound));
  const uint32_t c3 = __float_as_uint(__fadd_rn(__fmul_rn(__uint_as_float(w1 & 0xFFFF0000u), inv), kRound));
  return __byte_perm(__byte_perm(c0, c1, 0x0040), __byte_perm(c2, c3, 0x0040), 0x5410);
}

// Magnitude patterns (sign cleared) of bf16 values order like the
// magnitudes, so two-lane 16-bit integer maxima find max |x|.
__device__ __forceinline__ uint32_t absmax_u2(const uint4& w, uint32_t m) {
  return __vmaxu2(__vmaxu2(m, __vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu)),
                  __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu));
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait2() { asm volatile("cp.async.wait_group 2;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// Bulk copy shared -> global (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_store(void* gmem_dst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
               "r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_src))), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// This thread's shared-memory writes, visible to the bulk copy (async proxy).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(kQ8Threads)
    compact_int8_kernel(const int4* __restrict__ K, const int4* __restrict__ V, int64_t B, int64_t n_c,
                        const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                        const int64_t* __restrict__ offsets, const int64_t* __restrict__ out_offsets,
                        int8_t* __restrict__ Kq, int8_t* __restrict__ Vq, float* __restrict__ Ks,
                        float* __restrict__ Vs, int32_t* status) {
  using L = Q8<D>;
  extern __shared__ __align__(128) uint8_t q8s[];               // [3 stages][K | V rows], [K | V codes]
  const int t = threadIdx.x;
  const int64_t bph = (n_c + kQ8Rows - 1) / kQ8Rows;            // units per head
  const int lc = t % L::VPR;                                    // loader: chunk lc of rows lr0 + j * LSTRIDE
  const int lr0 = t / L::VPR;
  const int tensor = t >> 7;                                    // quantiser: half h of row r of K (0) or V (1)
  const int r = (t & 127) >> 1, h = t & 1;

  // A unit is (head hb, 64-slot block blk); this CTA visits units blockIdx.x,
  // blockIdx.x + gridDim.x, ... in that order, stepping (hb, blk) without a
  // division.  Each queued unit carries what its processing needs (count,
  // offsets, this thread's source rows), fetched a unit ahead.
  struct Unit {
    int64_t hb, blk, cnt, in0, out0;                             // hb == B: none
    int32_t own;                                                 // source row of this thread's quantiser row
  };
  const int64_t step_hb = gridDim.x / bph, step_blk = gridDim.x % bph;
  auto advance = [&](Unit& x) {
    x.blk += step_blk;
    x.hb += step_hb;
    if (x.blk >= bph) {
      x.blk -= bph;
      ++x.hb;
    }
  };
  // the first unit at or after x (inclusive) that has slots; then its offsets and source rows
  auto next_active = [&](Unit& x, int32_t (&src)[L::RPT]) {
    for (; x.hb < B; advance(x)) {
      x.cnt = counts[x.hb];
      if (x.cnt < 0 || x.cnt > n_c) {
        if (x.blk == 0 && t == 0) report_err(status, KVZ_ERR_INVALID_ARG);
        continue;
      }
      if (x.blk * kQ8Rows < x.cnt) break;
    }
#pragma unroll
    for (int j = 0; j < L::RPT; ++j) src[j] = -1;
    x.own = -1;
    if (x.hb >= B) return;
    x.in0 = offsets[x.hb];
    x.out0 = (out_offsets != nullptr ? out_offsets[x.hb] : x.in0) + x.blk * kQ8Rows;
    const int64_t p0 = x.blk * kQ8Rows;
#pragma unroll
    for (int j = 0; j < L::RPT; ++j) {
      const int64_t pp = p0 + lr0 + j * L::LSTRIDE;
      if (pp < x.cnt) src[j] = idx[x.in0 + pp];
    }
    if (p0 + r < x.cnt) x.own = idx[x.in0 + p0 + r];
  };
  auto issue = [&](const Unit& x, int st, const int32_t (&src)[L::RPT]) {
    if (x.hb < B) {
      uint8_t* sk = q8s + st * L::STAGE;
      const int4* kb = K + x.hb * n_c * L::VPR + lc;
      const int4* vb = V + x.hb * n_c * L::VPR + lc;
#pragma unroll
      for (int j = 0; j < L::RPT; ++j) {
        const int64_t s = src[j];
        if (s >= 0 && s < n_c) {
          const int row = lr0 + j * L::LSTRIDE;
          const int off = row * L::ROWB + ((lc ^ L::swz(row)) * 16);
          cp_async16(sk + off, kb + s * L::VPR);
          cp_async16(sk + kQ8Rows * L::ROWB + off, vb + s * L::VPR);
        }
      }
    }
    cp_async_commit();
  };

  // ring of three stages: units x0 (quantised now), x1 and x2 (in flight)
  int32_t src[L::RPT];
  Unit x0{static_cast<int64_t>(blockIdx.x) / bph, static_cast<int64_t>(blockIdx.x) % bph, 0, 0, 0, -1};
  next_active(x0, src);
  issue(x0, 0, src);
  Unit x1 = x0;
  advance(x1);
  next_active(x1, src);
  issue(x1, 1, src);
  Unit x2 = x1;
  advance(x2);
  next_active(x2, src);
  int st = 0;
  while (x0.hb < B) {
    issue(x2, st == 0 ? 2 : st - 1, src);                       // stage (st + 2) % 3
    Unit x3 = x2;
    advance(x3);
    next_active(x3, src);                                       // the unit after, and its indices
    cp_async_wait2();                                           // this thread's copies into stage st
    __syncthreads();                                            // everyone's

    const int nvalid = static_cast<int>(x0.cnt - x0.blk * kQ8Rows < kQ8Rows ? x0.cnt - x0.blk * kQ8Rows : kQ8Rows);
    const int64_t out0 = x0.out0;
    const uint8_t* srow = q8s + st * L::STAGE + tensor * kQ8Rows * L::ROWB + r * L::ROWB;
    uint8_t* orow = q8s + kQ8Stages * L::STAGE + tensor * kQ8Rows * D + r * D;
    const bool live = r < nvalid;
    const bool ok = x0.own >= 0 && x0.own < n_c;
    uint32_t m2 = 0u;
    if (live) {
      if (!ok && h == 0) report_err(status, KVZ_ERR_INVALID_ARG);   // idx out of [0, n_c): zeros
#pragma unroll
      for (int c = 0; c < L::CPH; ++c)
        m2 = absmax_u2(*reinterpret_cast<const uint4*>(srow + (((h * L::CPH + L::p1(c, r, h)) ^ L::swz(r)) * 16)),
                       m2);
    }
    m2 = __vmaxu2(m2, __shfl_xor_sync(0xffffffffu, m2, 1));    // the row's other half
    const uint32_t hm = max(m2 >> 16, m2 & 0xFFFFu);
    const float a = ok ? __uint_as_float(hm << 16) : 0.0f;
    if (t == 0) bulk_wait_read0();                              // the code tile: the last store has read it
    __syncthreads();
    if (live) {
      const float inv = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
#pragma unroll
      for (int k = 0; k < L::COH; ++k) {
        const int cc = h * L::COH + L::p2(k, r, h);
        uint4 code = make_uint4(0u, 0u, 0u, 0u);
        if (ok) {
          const uint4 w0 = *reinterpret_cast<const uint4*>(srow + (((2 * cc) ^ L::swz(r)) * 16));
          const uint4 w1 = *reinterpret_cast<const uint4*>(srow + (((2 * cc + 1) ^ L::swz(r)) * 16));
          code = make_uint4(code4(w0.x, w0.y, inv), code4(w0.z, w0.w, inv), code4(w1.x, w1.y, inv),
                            code4(w1.z, w1.w, inv));
        }
        *reinterpret_cast<uint4*>(orow + cc * 16) = code;
      }
      if (h == 0) (tensor == 0 ? Ks : Vs)[out0 + r] = __fdiv_rn(a, 127.0f);
    }
    fence_proxy_async_smem();                                   // the code tile, to the bulk copy
    __syncthreads();                                            // stage st and the tile are complete
    if (t == 0) {
      const uint8_t* tile = q8s + kQ8Stages * L::STAGE;
      bulk_store(Kq + out0 * D, tile, static_cast<uint32_t>(nvalid * D));
      bulk_store(Vq + out0 * D, tile + kQ8Rows * D, static_cast<uint32_t>(nvalid * D));
      bulk_commit();
    }
    x0 = x1;
    x1 = x2;
    x2 = x3;
    st = st == 2 ? 0 : st + 1;
  }
  cp_async_wait0();
  if (t == 0) bulk_wait_all();
}

// Dependencies of in-place compaction.  Slot chunk c (slots [cC, (c+1)C))
// writes rows [cC, (c+1)C).  Because idx ascends within a head, the slots
// whose source rows lie in that range form one contiguous run
// [lo_slot[c], lo_slot[c+1]), where lo_slot[r] is the first slot whose
// source row is >= rC (count if none).  Only the chunks holding that run
// read what chunk c overwrites.  One thread per slot p fills lo_slot[r] for
// the row chunks r in (chunk(idx[p-1]), chunk(idx[p])], capped at nchunks;
// the last slot also fills the row chunks past its source.
__global__ void __launch_bounds__(256)
    inplace_deps_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                        const int64_t* __restrict__ offsets, int64_t n_c, int64_t blocks_per_head,
                        uint32_t* lo_slot, int64_t lo_stride) {
  const int64_t b = blockIdx.x / blocks_per_head;
  const int64_t p = (blockIdx.x % blocks_per_head) * 256 + threadIdx.x;
  const int64_t count = counts[b];
  if (count < 0 || count > n_c || p >= count) return;   // the compaction kernel reports a bad count
  const int64_t nchunks = (count + kInplaceRows - 1) / kInplaceRows;
  const int32_t* hidx = idx + offsets[b];
  auto row_chunk = [&](int64_t v) -> int64_t {
    return v < 0 ? -1 : (v / kInplaceRows < nchunks ? v / kInplaceRows : nchunks);
  };
  const int64_t r1 = p == 0 ? -1 : row_chunk(hidx[p - 1]);
  const int64_t r2 = row_chunk(hidx[p]);
  uint32_t* lo = lo_slot + b * lo_stride;
  for (int64_t r = r1 + 1; r <= r2; ++r) lo[r] = static_cast<uint32_t>(p);
  if (p == count - 1)
    for (int64_t r = (r2 > r1 ? r2 : r1) + 1; r <= nchunks; ++r) lo[r] = static_cast<uint32_t>(count);
}

// In place.  Slot p of head b moves row idx[p] >= p down to row p, in K and
// in V.  Slots are cut into chunks of kInplaceRows; chunk c writes rows
// [cC, (c+1)C).  A row q is the source of at most one slot p', with
// p' <= idx[p'] = q, so only chunks <= c read rows that chunk c writes, and
// of those only the chunks holding slots [lo_slot[c], lo_slot[c+1]).
// Each warp is an independent worker: it claims chunks of its head from a
// per-head counter (lower chunks are claimed first) and keeps kInplaceDepth
// of them in a register ring, loads issued kInplaceDepth - 1 chunks ahead.
// For its oldest (current) chunk c every lane of the warp
//   - reads the "sources read" counters of the chunks below c that read
//     chunk c's rows (at most two: each of chunk c's rows feeds at most one
//     slot) and waits, bounded, until each shows all 32 lanes,
//   - writes its part of chunk c's rows from registers, then adds
//     1 + (a zero computed from the rows it loaded) to chunk c's counter.
// The add's value depends on the lane's loads and each row store is
// control-dependent on the counters its lane read, so a load can only see a
// row's old contents; no fence is needed (a release fence would wait for
// every load in flight).  At a keep ratio rho the readers of chunk c sit
// near chunk rho*c, long finished, so warps rarely wait.  A warp's current
// chunk is its lowest unpublished one and waits only on lower chunks, so
// the lowest unpublished chunk of a head always belongs to a warp whose
// waits are satisfied: every wait ends.  Rows are loaded coherently (they
// are written later in the same launch).
// `wait_ns` bounds every wait; publication of chunk `hold_c` of head
// `hold_b` is skipped when both are >= 0 (only the test entry point sets
// them, to make a wait expire; the normal call passes -1).
template <int VPR>
__global__ void __launch_bounds__(kInplaceThreads, kInplaceMinCtas)
    compact_inplace_kernel(int4* K, int4* V, int64_t B, int64_t n_c, int64_t warps_per_head,
                           const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                           const int64_t* __restrict__ offsets, uint32_t* next_chunk, uint32_t* chunk_read,
                           int64_t chunks_per_head, const uint32_t* lo_slot, int32_t* status, uint64_t wait_ns,
                           int64_t hold_b, int64_t hold_c) {
  constexpr int kRowsPerAccess = 32 / VPR;                    // rows one warp-wide access covers
  constexpr int NR = kInplaceRows / kRowsPerAccess;           // rows of a chunk each lane moves
  constexpr int D = kInplaceDepth;
  constexpr uint32_t kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * kInplaceThreads + threadIdx.x) >> 5;
  const int64_t b = gw / warps_per_head;
  if (b >= B) return;                                         // warp-uniform
  const int64_t count = counts[b];
  if (count < 0 || count > n_c) {
    if (lane == 0 && gw % warps_per_head == 0) report_err(status, KVZ_ERR_INVALID_ARG);
    return;
  }
  const uint32_t nchunks = static_cast<uint32_t>((count + kInplaceRows - 1) / kInplaceRows);
  int4* const Xk = K + b * n_c * VPR;
  int4* const Xv = V + b * n_c * VPR;
  uint32_t* const flags = chunk_read + b * chunks_per_head;
  const uint32_t* const lo = lo_slot + b * (chunks_per_head + 1);
  const int32_t* const hidx = idx + offsets[b];
  const int col = lane % VPR;                                 // 16-byte vector within the row
  const int rsub = lane / VPR;                                // row within an access

  int4 dk[D][NR], dv[D][NR];                                  // the register ring
  uint32_t valid = 0;                                         // bit s*NR + k: element k of stage s
  int32_t jn[NR];                                             // source rows of the next chunk to load
  uint32_t cl[D];                                             // chunk held by each stage (warp-uniform)

  auto fetch_idx = [&](uint32_t c) {
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int64_t p = static_cast<int64_t>(c) * kInplaceRows + rsub + k * kRowsPerAccess;
      jn[k] = (c < nchunks && p < count) ? hidx[p] : -1;
    }
  };
  auto issue = [&](int st, uint32_t c) {
    uint32_t bits = 0;
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int64_t p = static_cast<int64_t>(c) * kInplaceRows + rsub + k * kRowsPerAccess;
      if (c >= nchunks || p >= count) continue;
      const int64_t j = jn[k];
      if (j >= p && j < n_c) {
        dk[st][k] = ld_coherent(Xk + j * VPR + col);
        dv[st][k] = ld_coherent(Xv + j * VPR + col);
        bits |= 1u << k;
      } else {
        report_err(status, KVZ_ERR_INVALID_ARG);              // ascending idx guarantees p <= j < n_c
      }
    }
    valid = (valid & ~(((1u << NR) - 1u) << (st * NR))) | (bits << (st * NR));
  };

  {
    uint32_t first[D];
#pragma unroll
    for (int s = 0; s < D; ++s) first[s] = lane == 0 ? atomicAdd(&next_chunk[b], 1u) : 0u;
#pragma unroll
    for (int s = 0; s < D; ++s) cl[s] = __shfl_sync(kFull, first[s], 0);
  }
#pragma unroll
  for (int s = 0; s < D - 1; ++s) {
    fetch_idx(cl[s]);
    issue(s, cl[s]);
  }
  fetch_idx(cl[D - 1]);                                       // issued at the first step
  uint32_t pend = lane == 0 ? atomicAdd(&next_chunk[b], 1u) : 0u;   // the claim after that

  // Readers of chunk c: chunks [k0, k_end) (see inplace_deps_kernel).  The
  // run bounds of a chunk are loaded two steps before it is current and its
  // first reader's counter one step before; anything not yet complete is
  // polled at the current step.
  auto reader_range = [&](uint32_t c, uint32_t run_lo, uint32_t run_hi, uint32_t& k0, uint32_t& k_end) {
    const uint32_t k_last = run_hi > run_lo ? (run_hi - 1) / kInplaceRows + 1 : 0u;
    k0 = run_lo / kInplaceRows;
    k_end = c < nchunks ? (k_last < c ? k_last : c) : 0u;
  };
  auto first_flag = [&](uint32_t k0, uint32_t k_end) -> uint32_t {
    return k0 < k_end ? ld_relaxed_gpu(&flags[k0]) : 32u;
  };
  uint32_t k0 = 0, k_end = 0, seen = 32;                      // the current chunk's readers
  uint32_t nlo = 0, nhi = 0;                                  // run bounds of the next chunk
  if (cl[0] < nchunks) {
    reader_range(cl[0], lo[cl[0]], lo[cl[0] + 1], k0, k_end);
    seen = first_flag(k0, k_end);
  }
  if (cl[1 % D] < nchunks) {
    nlo = lo[cl[1 % D]];
    nhi = lo[cl[1 % D] + 1];
  }
  bool done = false;
  while (!done) {
#pragma unroll
    for (int s = 0; s < D; ++s) {
      const uint32_t cur = cl[s];
      if (cur >= nchunks) {                                   // later claims are higher chunks
        done = true;
        break;
      }
      int ok = 1;
      for (uint32_t k = k0; k < k_end; ++k) {
        if (k == k0 && seen == 32u) continue;
        if (ld_relaxed_gpu(&flags[k]) == 32u) continue;
        const uint64_t t0 = now_ns();
        while (ld_relaxed_gpu(&flags[k]) != 32u) {
          if (now_ns() - t0 > wait_ns) {
            ok = 0;
            break;
          }
        }
        if (!ok) break;
      }
      if (!__all_sync(kFull, ok)) {                           // a reader never published: stop
        if (lane == 0) report_err(status, KVZ_ERR_TIMEOUT);
        done = true;
        break;
      }
      uint32_t got = 0;                                       // a word of every row this lane loaded
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        if (!((valid >> (s * NR + k)) & 1u)) continue;
        const int64_t p = static_cast<int64_t>(cur) * kInplaceRows + rsub + k * kRowsPerAccess;
        Xk[p * VPR + col] = dk[s][k];
        Xv[p * VPR + col] = dv[s][k];
        got |= static_cast<uint32_t>(dk[s][k].x) | static_cast<uint32_t>(dv[s][k].x);
      }
      if (b != hold_b || static_cast<int64_t>(cur) != hold_c)
        red_relaxed_gpu_add(&flags[cur], 1u + dep_zero(got));   // this lane's sources of cur are read
      const int sn = (s + D - 1) % D;                         // the stage written out last step
      issue(sn, cl[sn]);
      const uint32_t c_next = __shfl_sync(kFull, pend, 0);
      fetch_idx(c_next);
      if (lane == 0) pend = atomicAdd(&next_chunk[b], 1u);
      cl[s] = c_next;
      const uint32_t c1 = cl[(s + 1) % D], c2 = cl[(s + 2) % D];   // the next two steps' chunks
      reader_range(c1, nlo, nhi, k0, k_end);
      seen = first_flag(k0, k_end);
      if (c2 < nchunks) {
        nlo = lo[c2];
        nhi = lo[c2 + 1];
      }
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
  if (blocks > 148 * KVZ_GATHER_CTAS_PER_SM) blocks = 148 * KVZ_GATHER_CTAS_PER_SM;
  if (blocks < 1) blocks = 1;
  compact_gather_kernel<<<static_cast<unsigned>(blocks), kGatherThreads, 0, stream>>>(
      static_cast<const int4*>(K), static_cast<const int4*>(V), B, n_c, vpr, idx, offsets, out_offsets,
      static_cast<int4*>(K_out), static_cast<int4*>(V_out), status);
  return cudaGetLastError();
}

namespace {
template <int D>
cudaError_t launch_int8(const void* K, const void* V, int64_t B, int64_t n_c, const int32_t* idx,
                        const int32_t* counts, const int64_t* offsets, const int64_t* out_offsets, int8_t* Kq,
                        int8_t* Vq, float* K_scale, float* V_scale, int32_t* status, cudaStream_t stream) {
  cudaError_t e = smem_limit_once<compact_int8_kernel<D>>(Q8<D>::SMEM);
  if (e != cudaSuccess) return e;
  int64_t blocks = B * ((n_c + kQ8Rows - 1) / kQ8Rows);
  const int64_t cap = D == 128 ? 148 * 2 : 148 * 3;              // resident CTAs per SM by shared memory (112 / 56 KB)
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  compact_int8_kernel<D><<<static_cast<unsigned>(blocks), kQ8Threads, Q8<D>::SMEM, stream>>>(
      static_cast<const int4*>(K), static_cast<const int4*>(V), B, n_c, idx, counts, offsets, out_offsets, Kq, Vq,
      K_scale, V_scale, status);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_compact_int8(const void* K, const void* V, int64_t B, int64_t n_c, int d, const int32_t* idx,
                                const int32_t* counts, const int64_t* offsets, const int64_t* out_offsets,
                                int8_t* Kq, int8_t* Vq, float* K_scale, float* V_scale, int32_t* status,
                                cudaStream_t stream) {
  return d == 128 ? launch_int8<128>(K, V, B, n_c, idx, counts, offsets, out_offsets, Kq, Vq, K_scale, V_scale,
                                     status, stream)
                  : launch_int8<64>(K, V, B, n_c, idx, counts, offsets, out_offsets, Kq, Vq, K_scale, V_scale,
                                    status, stream);
}

size_t compact_workspace_bytes(int64_t B, int64_t n_c) {
  const int64_t chunks = (n_c + kInplaceRows - 1) / kInplaceRows;
  return static_cast<size_t>((B * (2 + 2 * chunks) * 4 + 255) / 256 * 256);
}

cudaError_t launch_compact_inplace(void* K, void* V, int64_t B, int64_t n_c, int d, const int32_t* idx,
                                   const int32_t* counts, const int64_t* offsets, uint32_t* ws, int32_t* status,
                                   cudaStream_t stream, uint64_t wait_ns, int64_t hold_b, int64_t hold_c) {
  const int64_t chunks = (n_c + kInplaceRows - 1) / kInplaceRows;
  // next_chunk[B] | chunk_read[B][chunks] | lo_slot[B][chunks + 1], all zeroed (all-zero bits)
  uint32_t* next_chunk = ws;
  uint32_t* chunk_read = next_chunk + B;
  uint32_t* lo_slot = chunk_read + B * chunks;
  cudaError_t e = launch_fill_f32(reinterpret_cast<float*>(ws), B * (2 + 2 * chunks), 0.0f, stream);
  if (e != cudaSuccess) return e;
  const int64_t blocks_per_head = (n_c + 255) / 256;
  if (B * blocks_per_head > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  inplace_deps_kernel<<<static_cast<unsigned>(B * blocks_per_head), 256, 0, stream>>>(
      idx, counts, offsets, n_c, blocks_per_head, lo_slot, chunks + 1);
  auto kern = d == 128 ? compact_inplace_kernel<16> : compact_inplace_kernel<8>;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kInplaceThreads, 0)) != cudaSuccess) return e;
  // Enough warp workers to fill every resident warp slot kInplaceOversub times,
  // spread evenly over the heads, at most one per chunk.
  const int64_t slots = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1) * (kInplaceThreads / 32);
  int64_t wph = (slots * kInplaceOversub + B - 1) / B;
  if (wph > chunks) wph = chunks;
  if (wph < 1) wph = 1;
  const int64_t warps_per_cta = kInplaceThreads / 32;
  const int64_t grid = (B * wph + warps_per_cta - 1) / warps_per_cta;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), kInplaceThreads, 0, stream>>>(
      static_cast<int4*>(K), static_cast<int4*>(V), B, n_c, wph, idx, counts, offsets, next_chunk, chunk_read, chunks,
      lo_slot, status, wait_ns, hold_b, hold_c);
  return cudaGetLastError();
}

}  // namespace kvz
