// C ABI of libkvz: argument validation, TMA descriptor encoding and launch
// planning for the KVzip scoring, selection and compaction kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "kvz.h"
#include "kvz_internal.h"
#include "kvz_testing.h"

namespace {

constexpr int64_t kMaxRows = (int64_t(1) << 31) - 1024;   // TMA coordinates are int32

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
int64_t roundup(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D view [batch][rows][d] of a bf16 tensor, read in 128-row x 64-column
// boxes with the 128-byte swizzle the UMMA descriptors expect.  Rows past
// `rows` read as zeros (and are masked or discarded by the kernels).
bool make_map(CUtensorMap* m, const void* base, int64_t d, int64_t rows, int64_t batch) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(rows * d * 2)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D view [head][block][rows][d] of the context keys: `T` blocks of `rows`
// keys per head, block b of head h starting at row h*head_stride +
// b*block_stride.  Rows past `rows` read as zeros, so a block never sees the
// next block's keys.
bool make_ctx_map(CUtensorMap* m, const void* base, int64_t d, int64_t rows, int64_t T, int64_t heads,
                  int64_t block_stride, int64_t head_stride) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(T),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(block_stride * d * 2),
                           static_cast<cuuint64_t>(head_stride * d * 2)};
  cuuint32_t box[4] = {64, 128, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Where the context keys of each problem live: T blocks per head (see
// LseArgs); the plain score is T = 1 with both strides n_c.
struct CtxGeom {
  int T;
  int64_t block_stride, head_stride;   // in rows
};
CtxGeom plain_geom(int64_t n_c) { return CtxGeom{1, n_c, n_c}; }

// Rows [rows][d] of a packed cache read in 64-row x 64-column boxes (128-byte
// swizzle) by the decode kernel.
bool make_rows_map(CUtensorMap* m, const void* base, int64_t d, int64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), 1};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(rows * d * 2)};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

float log2e_scale(float scale) { return static_cast<float>(static_cast<double>(scale) * 1.4426950408889634); }

kvz_status check_score_common(const void* Q, const void* K_ctx, int64_t B, int G, int64_t n_c, int64_t n_in,
                              int d, float scale) {
  if (Q == nullptr || K_ctx == nullptr) return KVZ_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVZ_ERR_UNSUPPORTED;
  if (B < 1 || G < 1 || n_c < 1 || n_in < 1) return KVZ_ERR_INVALID_ARG;
  if (B * static_cast<int64_t>(G) > 0x7FFFFFFF || B > 0x7FFFFFFF) return KVZ_ERR_INVALID_ARG;
  if (n_c > kMaxRows || n_in > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return KVZ_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K_ctx, 16)) return KVZ_ERR_ALIGNMENT;
  return KVZ_OK;
}

// `part`: kvz::kLsePartBytes of scratch for the split tail of pass 1's
// grid, or null (no split).
kvz_status run_lse(const void* Q, const void* K_ctx, const void* K_in, int64_t B, int G, int64_t n_c,
                   int64_t n_in, int d, float scale, int64_t i_begin, int64_t i_end, float* lse2, int64_t ld,
                   int32_t* status, cudaStream_t stream, CtxGeom geom, void* part) {
  CUtensorMap tmQ, tmKc, tmKi;
  if (!make_map(&tmQ, Q, d, n_in, B * G) ||
      !make_ctx_map(&tmKc, K_ctx, d, n_c, geom.T, B / geom.T, geom.block_stride, geom.head_stride) ||
      !make_map(&tmKi, K_in, d, n_in, B))
    return KVZ_ERR_CUDA;
  kvz::LseArgs a{};
  a.B = static_cast<int>(B);
  a.G = G;
  a.T = geom.T;
  a.n_c = n_c;
  a.n_in = n_in;
  a.c2 = log2e_scale(scale);
  a.i_begin = i_begin;
  a.i_end = i_end;
  a.rows_pad = roundup(i_end - i_begin, 256);
  a.ld = ld;
  a.lse2 = lse2;
  a.status = status;
  a.part = static_cast<float2*>(part);
  return kvz::launch_lse(d, tmQ, tmKc, tmKi, a, stream) == cudaSuccess ? KVZ_OK : KVZ_ERR_CUDA;
}

kvz_status run_colmax(const void* Q, const void* K_ctx, int64_t B, int G, int64_t n_c, int64_t n_in, int d,
                      float scale, int64_t i_begin, int64_t i_end, const float* lse2, int64_t ld, float* S,
                      int32_t* status, cudaStream_t stream, CtxGeom geom, int64_t ldS, int64_t s_block) {
  CUtensorMap tmQ, tmKc;
  if (!make_map(&tmQ, Q, d, n_in, B * G) ||
      !make_ctx_map(&tmKc, K_ctx, d, n_c, geom.T, B / geom.T, geom.block_stride, geom.head_stride))
    return KVZ_ERR_CUDA;
  kvz::ColArgs a{};
  a.B = static_cast<int>(B);
  a.G = G;
  a.T = geom.T;
  a.ldS = ldS;
  a.s_block = s_block;
  a.n_c = n_c;
  a.c2 = log2e_scale(scale);
  a.i_begin = i_begin;
  a.rows_pad = roundup(i_end - i_begin, 256);
  a.ld = ld;
  a.lse2 = lse2;
  a.S = S;
  a.status = status;
  return kvz::launch_colmax(d, tmQ, tmKc, a, stream) == cudaSuccess ? KVZ_OK : KVZ_ERR_CUDA;
}

}  // namespace

extern "C" {

int kvz_version(void) { return 100; }

const char* kvz_status_string(int status) {
  switch (status) {
    case KVZ_OK: return "KVZ_OK";
    case KVZ_ERR_INVALID_ARG: return "KVZ_ERR_INVALID_ARG";
    case KVZ_ERR_UNSUPPORTED: return "KVZ_ERR_UNSUPPORTED";
    case KVZ_ERR_ALIGNMENT: return "KVZ_ERR_ALIGNMENT";
    case KVZ_ERR_WORKSPACE: return "KVZ_ERR_WORKSPACE";
    case KVZ_ERR_CUDA: return "KVZ_ERR_CUDA";
    case KVZ_ERR_INVALID_SCORE: return "KVZ_ERR_INVALID_SCORE";
    case KVZ_ERR_TIMEOUT: return "KVZ_ERR_TIMEOUT";
    default: return "KVZ_ERR_UNKNOWN";
  }
}

// Bytes of one chunk's lse2 in a scoring workspace (the split-tail scratch
// of pass 1 follows it).
int64_t lse_area_bytes(int64_t B, int G, int64_t rows) { return roundup(B * G * roundup(rows, 256) * 4, 256); }

size_t kvz_score_workspace_size(int64_t B, int G, int64_t n_in, int64_t row_chunk) {
  if (B < 1 || G < 1 || n_in < 1 || row_chunk < 0 || (row_chunk % 256) != 0) return 0;
  const int64_t rows = row_chunk == 0 || row_chunk > n_in ? n_in : row_chunk;
  return static_cast<size_t>(lse_area_bytes(B, G, rows)) + kvz::kLsePartBytes;
}

size_t kvz_score_lse2_workspace_size(void) { return kvz::kLsePartBytes; }

kvz_status kvz_score_lse2(const void* Q, const void* K_ctx, const void* K_in, int64_t B, int G, int64_t n_c,
                          int64_t n_in, int d, float scale, int64_t i_begin, int64_t i_end, float* lse2,
                          int64_t ld_lse2, void* workspace, size_t workspace_bytes, int32_t* d_status,
                          cudaStream_t stream) {
  kvz_status st = check_score_common(Q, K_ctx, B, G, n_c, n_in, d, scale);
  if (st != KVZ_OK) return st;
  if (K_in == nullptr || lse2 == nullptr) return KVZ_ERR_INVALID_ARG;
  if (!aligned(K_in, 16) || !aligned(lse2, 16) || ld_lse2 % 4 != 0) return KVZ_ERR_ALIGNMENT;
  if (i_begin < 0 || i_begin % 256 != 0 || i_end <= i_begin || i_end > n_in) return KVZ_ERR_INVALID_ARG;
  if (ld_lse2 < roundup(i_end - i_begin, 256)) return KVZ_ERR_INVALID_ARG;
  if (workspace != nullptr && workspace_bytes < kvz::kLsePartBytes) return KVZ_ERR_WORKSPACE;
  if (workspace != nullptr && !aligned(workspace, 16)) return KVZ_ERR_ALIGNMENT;
  return run_lse(Q, K_ctx, K_in, B, G, n_c, n_in, d, scale, i_begin, i_end, lse2, ld_lse2, d_status, stream,
                 plain_geom(n_c), workspace);
}

kvz_status kvz_score_colmax(const void* Q, const void* K_ctx, int64_t B, int G, int64_t n_c, int64_t n_in, int d,
                            float scale, int64_t i_begin, int64_t i_end, const float* lse2, int64_t ld_lse2,
                            float* S, int accumulate, int32_t* d_status, cudaStream_t stream) {
  kvz_status st = check_score_common(Q, K_ctx, B, G, n_c, n_in, d, scale);
  if (st != KVZ_OK) return st;
  if (lse2 == nullptr || S == nullptr) return KVZ_ERR_INVALID_ARG;
  if (!aligned(lse2, 16) || ld_lse2 % 4 != 0 || !aligned(S, 4)) return KVZ_ERR_ALIGNMENT;
  if (i_begin < 0 || i_begin % 256 != 0 || i_end <= i_begin || i_end > n_in) return KVZ_ERR_INVALID_ARG;
  if (ld_lse2 < roundup(i_end - i_begin, 256)) return KVZ_ERR_INVALID_ARG;
  if (!accumulate && kvz::launch_fill_f32(S, B * n_c, 0.0f, stream) != cudaSuccess) return KVZ_ERR_CUDA;
  return run_colmax(Q, K_ctx, B, G, n_c, n_in, d, scale, i_begin, i_end, lse2, ld_lse2, S, d_status, stream,
                    plain_geom(n_c), n_c, n_c);
}

kvz_status kvz_score(const void* Q, const void* K_ctx, const void* K_in, int64_t B, int G, int64_t n_c,
                     int64_t n_in, int d, float scale, int64_t row_chunk, float* S, void* workspace,
                     size_t workspace_bytes, int32_t* d_status, cudaStream_t stream) {
  kvz_status st = check_score_common(Q, K_ctx, B, G, n_c, n_in, d, scale);
  if (st != KVZ_OK) return st;
  if (K_in == nullptr || S == nullptr) return KVZ_ERR_INVALID_ARG;
  if (!aligned(K_in, 16) || !aligned(S, 4)) return KVZ_ERR_ALIGNMENT;
  if (row_chunk < 0 || row_chunk % 256 != 0) return KVZ_ERR_INVALID_ARG;
  const size_t need = kvz_score_workspace_size(B, G, n_in, row_chunk);
  if (workspace == nullptr || workspace_bytes < need) return KVZ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return KVZ_ERR_ALIGNMENT;
  const int64_t chunk = (row_chunk == 0 || row_chunk > n_in) ? n_in : row_chunk;
  const int64_t ld = roundup(chunk, 256);
  float* lse2 = static_cast<float*>(workspace);
  void* part = static_cast<uint8_t*>(workspace) + lse_area_bytes(B, G, chunk);
  if (kvz::launch_fill_f32(S, B * n_c, 0.0f, stream) != cudaSuccess) return KVZ_ERR_CUDA;
  for (int64_t i0 = 0; i0 < n_in; i0 += chunk) {
    const int64_t i1 = i0 + chunk < n_in ? i0 + chunk : n_in;
    st = run_lse(Q, K_ctx, K_in, B, G, n_c, n_in, d, scale, i0, i1, lse2, ld, d_status, stream, plain_geom(n_c),
                 part);
    if (st != KVZ_OK) return st;
    st = run_colmax(Q, K_ctx, B, G, n_c, n_in, d, scale, i0, i1, lse2, ld, S, d_status, stream, plain_geom(n_c),
                    n_c, n_c);
    if (st != KVZ_OK) return st;
  }
  return KVZ_OK;
}

size_t kvz_score_chunked_workspace_size(int64_t B, int G, int64_t n_c, int64_t n_prompt, int64_t m) {
  if (B < 1 || G < 1 || n_c < 1 || n_prompt < 0 || m < 1) return 0;
  const int64_t T = n_c / m, m_last = n_c % m;
  const int64_t full = T > 0 ? B * T * G * roundup(n_prompt + m, 256) * 4 : 0;
  const int64_t tail = m_last > 0 ? B * G * roundup(n_prompt + m_last, 256) * 4 : 0;
  return static_cast<size_t>(roundup(full > tail ? full : tail, 256)) + kvz::kLsePartBytes;
}

kvz_status kvz_score_chunked(const void* Q, const void* Q_tail, const void* K_ctx, const void* K_in,
                             const void* K_in_tail, int64_t B, int G, int64_t n_c, int64_t n_prompt, int64_t m,
                             int d, float scale, float* S, void* workspace, size_t workspace_bytes,
                             int32_t* d_status, cudaStream_t stream) {
  if (K_ctx == nullptr || S == nullptr) return KVZ_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVZ_ERR_UNSUPPORTED;
  if (B < 1 || G < 1 || n_c < 1 || n_prompt < 0 || m < 1 || n_c > kMaxRows || n_prompt + m > kMaxRows)
    return KVZ_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return KVZ_ERR_INVALID_ARG;
  const int64_t T = n_c / m, m_last = n_c % m;
  if (T > 0 && (Q == nullptr || K_in == nullptr)) return KVZ_ERR_INVALID_ARG;
  if (m_last > 0 && (Q_tail == nullptr || K_in_tail == nullptr)) return KVZ_ERR_INVALID_ARG;
  if (B * T * static_cast<int64_t>(G) > 0x7FFFFFFF || B * static_cast<int64_t>(G) > 0x7FFFFFFF)
    return KVZ_ERR_INVALID_ARG;
  if (!aligned(K_ctx, 16) || !aligned(S, 4) || (Q && !aligned(Q, 16)) || (Q_tail && !aligned(Q_tail, 16)) ||
      (K_in && !aligned(K_in, 16)) || (K_in_tail && !aligned(K_in_tail, 16)))
    return KVZ_ERR_ALIGNMENT;
  if (workspace == nullptr || workspace_bytes < kvz_score_chunked_workspace_size(B, G, n_c, n_prompt, m))
    return KVZ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return KVZ_ERR_ALIGNMENT;
  float* lse2 = static_cast<float*>(workspace);
  void* part = static_cast<uint8_t*>(workspace) +
               (kvz_score_chunked_workspace_size(B, G, n_c, n_prompt, m) - kvz::kLsePartBytes);
  if (kvz::launch_fill_f32(S, B * n_c, 0.0f, stream) != cudaSuccess) return KVZ_ERR_CUDA;
  if (T > 0) {
    // the full chunks of every head as one batch of B*T problems
    const int64_t n_in = n_prompt + m, ld = roundup(n_in, 256);
    const CtxGeom geom{static_cast<int>(T), m, n_c};
    kvz_status st =
        run_lse(Q, K_ctx, K_in, B * T, G, m, n_in, d, scale, 0, n_in, lse2, ld, d_status, stream, geom, part);
    if (st != KVZ_OK) return st;
    st = run_colmax(Q, K_ctx, B * T, G, m, n_in, d, scale, 0, n_in, lse2, ld, S, d_status, stream, geom, n_c, m);
    if (st != KVZ_OK) return st;
  }
  if (m_last > 0) {
    // the shorter last chunk of every head
    const int64_t n_in = n_prompt + m_last, ld = roundup(n_in, 256);
    const void* K_last = static_cast<const uint8_t*>(K_ctx) + T * m * d * 2;
    const CtxGeom geom{1, m_last, n_c};
    kvz_status st = run_lse(Q_tail, K_last, K_in_tail, B, G, m_last, n_in, d, scale, 0, n_in, lse2, ld, d_status,
                            stream, geom, part);
    if (st != KVZ_OK) return st;
    st = run_colmax(Q_tail, K_last, B, G, m_last, n_in, d, scale, 0, n_in, lse2, ld, S + T * m, d_status, stream,
                    geom, n_c, m_last);
    if (st != KVZ_OK) return st;
  }
  return KVZ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free scoring: the lse2 scratch is this file-scope device array.
// In host code its name only stands in for the symbol; the device address
// comes from cudaGetSymbolAddress, looked up once per CUDA context.
// ---------------------------------------------------------------------------
static __device__ __align__(256) float kvz_noalloc_lse2[KVZ_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {

// Driver calls that name the current context by its process-unique id, so a
// context created after a device reset, or a non-primary context a caller
// made current, never reuses an address looked up in another context.
struct CtxIdFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};
const CtxIdFns& ctx_id_fns() {
  static CtxIdFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return f;
}

constexpr int kMaxContexts = 64;
std::mutex g_noalloc_mu;
unsigned long long g_noalloc_ctx[kMaxContexts] = {};   // context ids (0 = free slot)
float* g_noalloc_addr[kMaxContexts] = {};
int g_noalloc_next = 0;                                 // round-robin replacement when full

// Process-unique id of the calling thread's current context (0 if none).
unsigned long long current_ctx_id() {
  const CtxIdFns& f = ctx_id_fns();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (f.get_current == nullptr || f.get_id == nullptr || f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      f.get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the static scratch in the current context.  With no
// context current yet, the symbol lookup itself initialises the current
// device's primary context, and the id is read after it.
kvz_status noalloc_scratch(float** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long id = current_ctx_id();
  if (id != 0)
    for (int i = 0; i < kMaxContexts; ++i)
      if (g_noalloc_ctx[i] == id) {
        *out = g_noalloc_addr[i];
        return KVZ_OK;
      }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, kvz_noalloc_lse2) != cudaSuccess || p == nullptr) return KVZ_ERR_CUDA;
  if (id == 0 && (id = current_ctx_id()) == 0) return KVZ_ERR_CUDA;
  const int slot = g_noalloc_next;
  g_noalloc_next = (g_noalloc_next + 1) % kMaxContexts;
  g_noalloc_ctx[slot] = id;
  g_noalloc_addr[slot] = static_cast<float*>(p);
  *out = g_noalloc_addr[slot];
  return KVZ_OK;
}

}  // namespace

extern "C" {

kvz_status kvz_score_noalloc(const void* Q, const void* K_ctx, const void* K_in, int64_t B, int G, int64_t n_c,
                             int64_t n_in, int d, float scale, float* S, int32_t* d_status, cudaStream_t stream) {
  kvz_status st = check_score_common(Q, K_ctx, B, G, n_c, n_in, d, scale);
  if (st != KVZ_OK) return st;
  if (K_in == nullptr || S == nullptr) return KVZ_ERR_INVALID_ARG;
  if (!aligned(K_in, 16) || !aligned(S, 4)) return KVZ_ERR_ALIGNMENT;
  constexpr int64_t cap = KVZ_NOALLOC_SCRATCH_BYTES / sizeof(float);
  const int64_t per_block = B * G * 256;                 // floats for one 256-row block of every (b, g)
  if (per_block > cap) return KVZ_ERR_WORKSPACE;
  int64_t chunk = (cap / per_block) * 256;
  if (chunk >= n_in) chunk = n_in;
  const int64_t ld = roundup(chunk, 256);
  float* lse2 = nullptr;
  st = noalloc_scratch(&lse2);
  if (st != KVZ_OK) return st;
  if (kvz::launch_fill_f32(S, B * n_c, 0.0f, stream) != cudaSuccess) return KVZ_ERR_CUDA;
  for (int64_t i0 = 0; i0 < n_in; i0 += chunk) {
    const int64_t i1 = i0 + chunk < n_in ? i0 + chunk : n_in;
    st = run_lse(Q, K_ctx, K_in, B, G, n_c, n_in, d, scale, i0, i1, lse2, ld, d_status, stream, plain_geom(n_c),
                 nullptr);
    if (st != KVZ_OK) return st;
    st = run_colmax(Q, K_ctx, B, G, n_c, n_in, d, scale, i0, i1, lse2, ld, S, d_status, stream, plain_geom(n_c),
                    n_c, n_c);
    if (st != KVZ_OK) return st;
  }
  return KVZ_OK;
}

int64_t kvz_keep_count(int64_t n, double ratio) {
  if (n < 0 || !(ratio >= 0.0 && ratio <= 1.0)) return -1;
  return static_cast<int64_t>(std::floor(ratio * static_cast<double>(n)));
}

size_t kvz_select_workspace_size(int64_t B, int64_t n_c, int mode) {
  if (B < 1 || n_c < 1 || (mode != KVZ_PER_HEAD && mode != KVZ_GLOBAL)) return 0;
  return kvz::select_workspace(B, n_c, mode).bytes;
}

kvz_status kvz_select(const float* S, int64_t B, int64_t n_c, double ratio, int mode, int32_t* idx,
                      int64_t idx_capacity, int32_t* counts, int64_t* offsets, void* workspace,
                      size_t workspace_bytes, int32_t* d_status, cudaStream_t stream) {
  if (S == nullptr || counts == nullptr || offsets == nullptr) return KVZ_ERR_INVALID_ARG;
  if (mode != KVZ_PER_HEAD && mode != KVZ_GLOBAL) return KVZ_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || n_c < 1 || n_c > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (B * n_c >= (int64_t(1) << 32)) return KVZ_ERR_INVALID_ARG;
  if (!(ratio >= 0.0 && ratio <= 1.0)) return KVZ_ERR_INVALID_ARG;
  if (!aligned(S, 4) || !aligned(counts, 4) || !aligned(offsets, 8) || (idx && !aligned(idx, 4)))
    return KVZ_ERR_ALIGNMENT;
  const int64_t k = mode == KVZ_GLOBAL ? kvz_keep_count(B * n_c, ratio) : kvz_keep_count(n_c, ratio);
  const int64_t need = mode == KVZ_GLOBAL ? k : B * k;
  if (idx_capacity < need || (need > 0 && idx == nullptr)) return KVZ_ERR_INVALID_ARG;
  const kvz::SelWorkspace lay = kvz::select_workspace(B, n_c, mode);
  if (workspace == nullptr || workspace_bytes < lay.bytes) return KVZ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return KVZ_ERR_ALIGNMENT;
  return kvz::launch_select(S, B, n_c, 0, mode, k, idx, counts, offsets, workspace, lay, d_status, stream) ==
                 cudaSuccess
             ? KVZ_OK
             : KVZ_ERR_CUDA;
}

namespace {
// Host checks shared by the distributed selection calls.
kvz_status dist_check(const float* S, int64_t B_local, int64_t n_c, const void* ws, size_t ws_bytes,
                      kvz::SelWorkspace* lay) {
  if (S == nullptr) return KVZ_ERR_INVALID_ARG;
  if (B_local < 1 || B_local > 65535 || n_c < 1 || n_c > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (B_local * n_c >= (int64_t(1) << 32)) return KVZ_ERR_INVALID_ARG;
  if (!aligned(S, 4)) return KVZ_ERR_ALIGNMENT;
  *lay = kvz::select_workspace(B_local, n_c, KVZ_GLOBAL);
  if (ws == nullptr || ws_bytes < lay->bytes) return KVZ_ERR_WORKSPACE;
  if (!aligned(ws, 16)) return KVZ_ERR_ALIGNMENT;
  return KVZ_OK;
}
}  // namespace

size_t kvz_select_dist_workspace_size(int64_t B_local, int64_t n_c) {
  if (B_local < 1 || n_c < 1) return 0;
  return kvz::select_workspace(B_local, n_c, KVZ_GLOBAL).bytes;
}

kvz_status kvz_select_dist_begin(const float* S, int64_t B_local, int64_t n_c, int64_t B_total, double ratio,
                                 uint32_t* hist, void* workspace, size_t workspace_bytes, int32_t* d_status,
                                 cudaStream_t stream) {
  kvz::SelWorkspace lay;
  const kvz_status st = dist_check(S, B_local, n_c, workspace, workspace_bytes, &lay);
  if (st != KVZ_OK) return st;
  if (hist == nullptr) return KVZ_ERR_INVALID_ARG;
  if (!aligned(hist, 16)) return KVZ_ERR_ALIGNMENT;
  if (B_total < B_local || !(ratio >= 0.0 && ratio <= 1.0)) return KVZ_ERR_INVALID_ARG;
  if (B_total * n_c >= (int64_t(1) << 32)) return KVZ_ERR_INVALID_ARG;   // histogram bins are 32-bit
  const int64_t k = kvz_keep_count(B_total * n_c, ratio);
  return kvz::launch_select_dist_begin(S, B_local, n_c, k, hist, workspace, lay, d_status, stream) == cudaSuccess
             ? KVZ_OK
             : KVZ_ERR_CUDA;
}

kvz_status kvz_select_dist_step(const float* S, int64_t B_local, int64_t n_c, int pass, uint32_t* hist,
                                uint64_t* eq_total, void* workspace, size_t workspace_bytes, int32_t* d_status,
                                cudaStream_t stream) {
  kvz::SelWorkspace lay;
  const kvz_status st = dist_check(S, B_local, n_c, workspace, workspace_bytes, &lay);
  if (st != KVZ_OK) return st;
  if (pass < 0 || pass > 2 || hist == nullptr || (pass == 2 && eq_total == nullptr)) return KVZ_ERR_INVALID_ARG;
  if (!aligned(hist, 16) || (eq_total != nullptr && !aligned(eq_total, 8))) return KVZ_ERR_ALIGNMENT;
  return kvz::launch_select_dist_step(S, B_local, n_c, pass, hist,
                                      reinterpret_cast<unsigned long long*>(eq_total), workspace, lay, d_status,
                                      stream) == cudaSuccess
             ? KVZ_OK
             : KVZ_ERR_CUDA;
}

kvz_status kvz_select_dist_finish(const float* S, int64_t B_local, int64_t n_c, int64_t B_total, double ratio,
                                  const uint64_t* eq_ranks, int rank, int32_t* idx, int64_t idx_capacity,
                                  int32_t* counts, int64_t* offsets, void* workspace, size_t workspace_bytes,
                                  int32_t* d_status, cudaStream_t stream) {
  kvz::SelWorkspace lay;
  const kvz_status st = dist_check(S, B_local, n_c, workspace, workspace_bytes, &lay);
  if (st != KVZ_OK) return st;
  if (eq_ranks == nullptr || counts == nullptr || offsets == nullptr || rank < 0) return KVZ_ERR_INVALID_ARG;
  if (B_total < B_local || !(ratio >= 0.0 && ratio <= 1.0)) return KVZ_ERR_INVALID_ARG;
  if (B_total * n_c >= (int64_t(1) << 32)) return KVZ_ERR_INVALID_ARG;   // histogram bins are 32-bit
  if (!aligned(eq_ranks, 8) || !aligned(counts, 4) || !aligned(offsets, 8) || (idx && !aligned(idx, 4)))
    return KVZ_ERR_ALIGNMENT;
  const int64_t k = kvz_keep_count(B_total * n_c, ratio);
  const int64_t need = k < B_local * n_c ? k : B_local * n_c;
  if (idx_capacity < need || (need > 0 && idx == nullptr)) return KVZ_ERR_INVALID_ARG;
  (void)d_status;
  return kvz::launch_select_dist_finish(S, B_local, n_c, reinterpret_cast<const unsigned long long*>(eq_ranks),
                                        rank, idx, counts, offsets, workspace, lay, stream) == cudaSuccess
             ? KVZ_OK
             : KVZ_ERR_CUDA;
}

kvz_status kvz_select_protected(const float* S, int64_t B, int64_t n_c, double ratio, int mode, int64_t n_protect,
                                int32_t* idx, int64_t idx_capacity, int32_t* counts, int64_t* offsets,
                                void* workspace, size_t workspace_bytes, int32_t* d_status, cudaStream_t stream) {
  if (S == nullptr || counts == nullptr || offsets == nullptr) return KVZ_ERR_INVALID_ARG;
  if (mode != KVZ_PER_HEAD && mode != KVZ_GLOBAL) return KVZ_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || n_c < 1 || n_c > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (B * n_c >= (int64_t(1) << 32)) return KVZ_ERR_INVALID_ARG;
  if (!(ratio >= 0.0 && ratio <= 1.0) || n_protect < 0 || n_protect > n_c) return KVZ_ERR_INVALID_ARG;
  if (!aligned(S, 4) || !aligned(counts, 4) || !aligned(offsets, 8) || (idx && !aligned(idx, 4)))
    return KVZ_ERR_ALIGNMENT;
  // the protected positions rank above every score, so keeping them plus the
  // ratio's share of the rest is a top-k of k = protected + share
  const int64_t free = n_c - n_protect;
  const int64_t k = mode == KVZ_GLOBAL ? B * n_protect + kvz_keep_count(B * free, ratio)
                                       : n_protect + kvz_keep_count(free, ratio);
  const int64_t need = mode == KVZ_GLOBAL ? k : B * k;
  if (idx_capacity < need || (need > 0 && idx == nullptr)) return KVZ_ERR_INVALID_ARG;
  const kvz::SelWorkspace lay = kvz::select_workspace(B, n_c, mode);
  if (workspace == nullptr || workspace_bytes < lay.bytes) return KVZ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return KVZ_ERR_ALIGNMENT;
  return kvz::launch_select(S, B, n_c, n_protect, mode, k, idx, counts, offsets, workspace, lay, d_status,
                            stream) == cudaSuccess
             ? KVZ_OK
             : KVZ_ERR_CUDA;
}

kvz_status kvz_head_score(const float* S, int64_t B, int64_t n_c, float* S_head, int32_t* d_status,
                          cudaStream_t stream) {
  if (S == nullptr || S_head == nullptr) return KVZ_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || n_c < 1 || n_c > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (!aligned(S, 4) || !aligned(S_head, 4)) return KVZ_ERR_ALIGNMENT;
  return kvz::launch_head_max(S, B, n_c, S_head, d_status, stream) == cudaSuccess ? KVZ_OK : KVZ_ERR_CUDA;
}

size_t kvz_select_heads_workspace_size(int64_t B) {
  if (B < 1 || B > 65535) return 0;
  const size_t sel = kvz_select_workspace_size(1, B, KVZ_PER_HEAD);
  return ((sel + 255) & ~size_t(255)) + ((static_cast<size_t>(B) * 4 + 255) & ~size_t(255)) + 256;
}

kvz_status kvz_select_heads(const float* S_head, int64_t B, int64_t n_c, double ratio, int32_t* idx,
                            int64_t idx_capacity, int32_t* counts, int64_t* offsets, void* workspace,
                            size_t workspace_bytes, int32_t* d_status, cudaStream_t stream) {
  if (S_head == nullptr || counts == nullptr || offsets == nullptr) return KVZ_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || n_c < 1 || n_c > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (!(ratio >= 0.0 && ratio <= 1.0)) return KVZ_ERR_INVALID_ARG;
  const int64_t k = kvz_keep_count(B, ratio);
  if (idx_capacity < k * n_c || (k > 0 && idx == nullptr) || k * n_c > 0x7FFFFFFF) return KVZ_ERR_INVALID_ARG;
  if (!aligned(S_head, 4) || !aligned(counts, 4) || !aligned(offsets, 8) || (idx && !aligned(idx, 4)))
    return KVZ_ERR_ALIGNMENT;
  if (workspace == nullptr || workspace_bytes < kvz_select_heads_workspace_size(B)) return KVZ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return KVZ_ERR_ALIGNMENT;
  // the head scores as one segment of B scores: the kept heads, ascending
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t sel = (kvz_select_workspace_size(1, B, KVZ_PER_HEAD) + 255) & ~size_t(255);
  int32_t* kept = reinterpret_cast<int32_t*>(ws + sel);
  int32_t* cnt1 = reinterpret_cast<int32_t*>(ws + sel + ((static_cast<size_t>(B) * 4 + 255) & ~size_t(255)));
  int64_t* off2 = reinterpret_cast<int64_t*>(cnt1 + 4);
  kvz_status st = kvz_select(S_head, 1, B, ratio, KVZ_PER_HEAD, kept, k > 0 ? k : 1, cnt1, off2, ws, sel,
                             d_status, stream);
  if (st != KVZ_OK) return st;
  return kvz::launch_head_expand(kept, k, B, n_c, idx, counts, offsets, stream) == cudaSuccess ? KVZ_OK
                                                                                            : KVZ_ERR_CUDA;
}

size_t kvz_decode_workspace_size(int64_t B, int G, int64_t n_c, int d) {
  if (B < 1 || B > 65535 || G < 1 || G > kvz::kDecGMax || n_c < 1 || (d != 64 && d != 128)) return 0;
  const size_t items = static_cast<size_t>(kvz::decode_items(B));
  return ((items * sizeof(kvz::DecItem) + 255) & ~size_t(255)) + ((items * G * 8 + 255) & ~size_t(255)) +
         ((items * G * d * 4 + 255) & ~size_t(255)) + ((static_cast<size_t>(B) * 4 + 255) & ~size_t(255)) +
         ((items * 4 + 255) & ~size_t(255));
}

kvz_status kvz_decode(const void* q, const void* K_out, const void* V_out, int64_t n_rows, const int32_t* counts,
                      const int64_t* offsets, int64_t B, int G, int64_t n_c, int d, float scale, float* out,
                      float* lse2, void* workspace, size_t workspace_bytes, int32_t* d_status,
                      cudaStream_t stream) {
  if (q == nullptr || K_out == nullptr || V_out == nullptr || counts == nullptr || offsets == nullptr ||
      out == nullptr)
    return KVZ_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVZ_ERR_UNSUPPORTED;
  if (G < 1 || G > kvz::kDecGMax) return KVZ_ERR_UNSUPPORTED;
  if (B < 1 || B > 65535 || n_c < 1 || n_rows < 1 || n_rows > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return KVZ_ERR_INVALID_ARG;
  if (!aligned(K_out, 16) || !aligned(V_out, 16) || !aligned(q, 16) || !aligned(out, 16) || !aligned(counts, 4) ||
      !aligned(offsets, 8) || (lse2 && !aligned(lse2, 4)))
    return KVZ_ERR_ALIGNMENT;
  const size_t need = kvz_decode_workspace_size(B, G, n_c, d);
  if (workspace == nullptr || workspace_bytes < need) return KVZ_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return KVZ_ERR_ALIGNMENT;
  CUtensorMap tmK, tmV;
  if (!make_rows_map(&tmK, K_out, d, n_rows) || !make_rows_map(&tmV, V_out, d, n_rows)) return KVZ_ERR_CUDA;
  kvz::DecArgs a{};
  a.B = static_cast<int>(B);
  a.G = G;
  a.n_c = n_c;
  a.c2 = log2e_scale(scale);
  a.q = static_cast<const uint16_t*>(q);
  a.counts = counts;
  a.offsets = offsets;
  a.n_items = kvz::decode_items(B);
  const size_t items = static_cast<size_t>(a.n_items);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.items = reinterpret_cast<kvz::DecItem*>(w);
  w += (items * sizeof(kvz::DecItem) + 255) & ~size_t(255);
  a.part_ml = reinterpret_cast<float2*>(w);
  w += (items * G * 8 + 255) & ~size_t(255);
  a.part_o = reinterpret_cast<float*>(w);
  w += (items * G * d * 4 + 255) & ~size_t(255);
  a.done = reinterpret_cast<unsigned*>(w);
  w += (static_cast<size_t>(B) * 4 + 255) & ~size_t(255);
  a.gdone = reinterpret_cast<unsigned*>(w);
  a.status = d_status;
  return kvz::launch_decode(d, tmK, tmV, a, out, lse2, stream) == cudaSuccess ? KVZ_OK : KVZ_ERR_CUDA;
}

kvz_status kvz_compact_int8(const void* K, const void* V, int64_t B, int64_t n_c, int d, const int32_t* idx,
                            const int32_t* counts, const int64_t* offsets, const int64_t* out_offsets, int8_t* Kq,
                            int8_t* Vq, float* K_scale, float* V_scale, int32_t* d_status, cudaStream_t stream) {
  if (K == nullptr || V == nullptr || idx == nullptr || counts == nullptr || offsets == nullptr || Kq == nullptr ||
      Vq == nullptr || K_scale == nullptr || V_scale == nullptr)
    return KVZ_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVZ_ERR_UNSUPPORTED;
  if (B < 1 || B > 0x7FFFFFFF / 8 || n_c < 1 || n_c > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(Kq, 16) || !aligned(Vq, 16) || !aligned(K_scale, 4) ||
      !aligned(V_scale, 4) || !aligned(idx, 4) || !aligned(counts, 4) || !aligned(offsets, 8) ||
      (out_offsets && !aligned(out_offsets, 8)))
    return KVZ_ERR_ALIGNMENT;
  return kvz::launch_compact_int8(K, V, B, n_c, d, idx, counts, offsets, out_offsets, Kq, Vq, K_scale, V_scale,
                                  d_status, stream) == cudaSuccess
             ? KVZ_OK
             : KVZ_ERR_CUDA;
}

size_t kvz_compact_workspace_size(int64_t B, int64_t n_c) {
  if (B < 1 || n_c < 1) return 0;
  return kvz::compact_workspace_bytes(B, n_c);
}

kvz_status kvz_compact(const void* K, const void* V, int64_t B, int64_t n_c, int d, const int32_t* idx,
                       const int32_t* counts, const int64_t* offsets, const int64_t* out_offsets, void* K_out,
                       void* V_out, void* workspace, size_t workspace_bytes, int32_t* d_status, cudaStream_t stream) {
  if (K == nullptr || V == nullptr || K_out == nullptr || V_out == nullptr || counts == nullptr ||
      offsets == nullptr || idx == nullptr)
    return KVZ_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVZ_ERR_UNSUPPORTED;
  if (B < 1 || B > 0x7FFFFFFF / 8 || n_c < 1 || n_c > kMaxRows) return KVZ_ERR_INVALID_ARG;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(K_out, 16) || !aligned(V_out, 16) || !aligned(idx, 4) ||
      !aligned(counts, 4) || !aligned(offsets, 8) || (out_offsets && !aligned(out_offsets, 8)))
    return KVZ_ERR_ALIGNMENT;
  const bool k_same = K_out == K, v_same = V_out == V;
  if (k_same != v_same) return KVZ_ERR_INVALID_ARG;          // partial in-place aliasing
  if (K == V) return KVZ_ERR_INVALID_ARG;
  if (k_same) {
    if (out_offsets != nullptr) return KVZ_ERR_INVALID_ARG;
    if (workspace == nullptr || workspace_bytes < kvz::compact_workspace_bytes(B, n_c)) return KVZ_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return KVZ_ERR_ALIGNMENT;
    return kvz::launch_compact_inplace(K_out, V_out, B, n_c, d, idx, counts, offsets,
                                       static_cast<uint32_t*>(workspace), d_status, stream) == cudaSuccess
               ? KVZ_OK
               : KVZ_ERR_CUDA;
  }
  // Out of place: the outputs must not start inside either input.
  const uintptr_t span = static_cast<uintptr_t>(B * n_c * d * 2);
  const uintptr_t k0 = reinterpret_cast<uintptr_t>(K), v0 = reinterpret_cast<uintptr_t>(V);
  for (const void* o : {K_out, V_out}) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(o);
    if ((x >= k0 && x < k0 + span) || (x >= v0 && x < v0 + span)) return KVZ_ERR_INVALID_ARG;
  }
  return kvz::launch_compact_gather(K, V, B, n_c, d, idx, offsets, out_offsets, K_out, V_out, d_status,
                                    stream) == cudaSuccess
             ? KVZ_OK
             : KVZ_ERR_CUDA;
}

kvz_status kvz_testing_compact_in_place_withhold(void* K, void* V, int64_t B, int64_t n_c, int d,
                                                 const int32_t* idx, const int32_t* counts,
                                                 const int64_t* offsets, void* workspace,
                                                 size_t workspace_bytes, int64_t wait_ns, int64_t hold_head,
                                                 int64_t hold_chunk, int32_t* d_status, cudaStream_t stream) {
  if (K == nullptr || V == nullptr || counts == nullptr || offsets == nullptr || idx == nullptr)
    return KVZ_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVZ_ERR_UNSUPPORTED;
  if (B < 1 || B > 0x7FFFFFFF / 8 || n_c < 1 || n_c > kMaxRows || K == V) return KVZ_ERR_INVALID_ARG;
  if (wait_ns < 1000 || wait_ns > 1000000000 || hold_head < 0 || hold_head >= B || hold_chunk < 0)
    return KVZ_ERR_INVALID_ARG;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(idx, 4) || !aligned(counts, 4) || !aligned(offsets, 8))
    return KVZ_ERR_ALIGNMENT;
  if (workspace == nullptr || workspace_bytes < kvz::compact_workspace_bytes(B, n_c)) return KVZ_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return KVZ_ERR_ALIGNMENT;
  return kvz::launch_compact_inplace(K, V, B, n_c, d, idx, counts, offsets, static_cast<uint32_t*>(workspace),
                                     d_status, stream, static_cast<uint64_t>(wait_ns), hold_head,
                                     hold_chunk) == cudaSuccess
             ? KVZ_OK
             : KVZ_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// End to end from host memory: one context's inputs are copied in by head
// chunks on a copy stream, each chunk is scored as soon as it lands, then
// selection, compaction and the copies of the results back to the host run
// on the compute stream.
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t kHostChunks = 8;   // head chunks the input copies are split into

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct HostPlan {
  int64_t k, kept, chunk_heads;
  size_t off_q, off_kc, off_ki, off_v, off_s, off_lse, lse_bytes, off_sel, sel_bytes, off_idx, off_cnt, off_off,
      off_ko, off_vo, bytes;
};

bool host_plan(int64_t B, int G, int64_t n_c, int64_t n_in, int d, double ratio, int mode, HostPlan* p) {
  if (B < 1 || G < 1 || n_c < 1 || n_in < 1 || (d != 64 && d != 128)) return false;
  if (!(ratio >= 0.0 && ratio <= 1.0) || (mode != KVZ_PER_HEAD && mode != KVZ_GLOBAL)) return false;
  if (B > 65535 || n_c > kMaxRows || n_in > kMaxRows || B * n_c >= (int64_t(1) << 32)) return false;
  p->k = kvz_keep_count(mode == KVZ_GLOBAL ? B * n_c : n_c, ratio);
  p->kept = mode == KVZ_GLOBAL ? p->k : B * p->k;
  const int64_t nchunks = B < kHostChunks ? B : kHostChunks;
  p->chunk_heads = (B + nchunks - 1) / nchunks;
  const size_t row = static_cast<size_t>(d) * 2;
  const size_t kept1 = static_cast<size_t>(p->kept > 0 ? p->kept : 1);
  size_t o = 0;
  p->off_q = o;   o = align256(o + static_cast<size_t>(B * G * n_in) * row);
  p->off_kc = o;  o = align256(o + static_cast<size_t>(B * n_c) * row);
  p->off_ki = o;  o = align256(o + static_cast<size_t>(B * n_in) * row);
  p->off_v = o;   o = align256(o + static_cast<size_t>(B * n_c) * row);
  p->off_s = o;   o = align256(o + static_cast<size_t>(B * n_c) * 4);
  p->lse_bytes = kvz_score_workspace_size(p->chunk_heads, G, n_in, 0);
  p->off_lse = o; o = align256(o + p->lse_bytes);
  p->sel_bytes = kvz_select_workspace_size(B, n_c, mode);
  p->off_sel = o; o = align256(o + p->sel_bytes);
  p->off_idx = o; o = align256(o + kept1 * 4);
  p->off_cnt = o; o = align256(o + static_cast<size_t>(B) * 4);
  p->off_off = o; o = align256(o + static_cast<size_t>(B + 1) * 8);
  p->off_ko = o;  o = align256(o + kept1 * row);
  p->off_vo = o;  o = align256(o + kept1 * row);
  p->bytes = o;
  return true;
}

// Events of one call; released when the call returns (a recorded event may
// be destroyed before it completes).
struct CallEvents {
  cudaEvent_t ev[kHostChunks + 2] = {};
  int n = 0;
  cudaError_t make(int count) {
    for (; n < count; ++n) {
      cudaError_t e = cudaEventCreateWithFlags(&ev[n], cudaEventDisableTiming);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  ~CallEvents() {
    for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);
  }
};

}  // namespace

extern "C" {

size_t kvz_compress_host_workspace_size(int64_t B, int G, int64_t n_c, int64_t n_in, int d, double ratio,
                                        int mode) {
  HostPlan p;
  return host_plan(B, G, n_c, n_in, d, ratio, mode, &p) ? p.bytes : 0;
}

kvz_status kvz_compress_host(const void* hQ, const void* hK_ctx, const void* hK_in, const void* hV, int64_t B,
                             int G, int64_t n_c, int64_t n_in, int d, float scale, double ratio, int mode,
                             int32_t* h_idx, int64_t idx_capacity, int32_t* h_counts, int64_t* h_offsets,
                             void* hK_out, void* hV_out, void* workspace, size_t workspace_bytes,
                             int32_t* d_status, cudaStream_t stream, cudaStream_t copy_stream) {
  if (hQ == nullptr || hK_ctx == nullptr || hK_in == nullptr || hV == nullptr || h_counts == nullptr ||
      h_offsets == nullptr)
    return KVZ_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVZ_ERR_UNSUPPORTED;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return KVZ_ERR_INVALID_ARG;
  HostPlan p;
  if (!host_plan(B, G, n_c, n_in, d, ratio, mode, &p)) return KVZ_ERR_INVALID_ARG;
  if (idx_capacity < p.kept || (p.kept > 0 && (h_idx == nullptr || hK_out == nullptr || hV_out == nullptr)))
    return KVZ_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < p.bytes) return KVZ_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return KVZ_ERR_ALIGNMENT;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* dQ = ws + p.off_q;
  uint8_t* dKc = ws + p.off_kc;
  uint8_t* dKi = ws + p.off_ki;
  uint8_t* dV = ws + p.off_v;
  float* dS = reinterpret_cast<float*>(ws + p.off_s);
  int32_t* d_idx = reinterpret_cast<int32_t*>(ws + p.off_idx);
  int32_t* d_cnt = reinterpret_cast<int32_t*>(ws + p.off_cnt);
  int64_t* d_off = reinterpret_cast<int64_t*>(ws + p.off_off);
  const size_t row = static_cast<size_t>(d) * 2;
  const int64_t nchunks = (B + p.chunk_heads - 1) / p.chunk_heads;

  CallEvents evs;
  if (evs.make(static_cast<int>(nchunks) + 2) != cudaSuccess) return KVZ_ERR_CUDA;
  cudaEvent_t ev_start = evs.ev[0], ev_v = evs.ev[1];
  // the copies must not overwrite the workspace while earlier work on `stream` reads it
  if (cudaEventRecord(ev_start, stream) != cudaSuccess || cudaStreamWaitEvent(copy_stream, ev_start, 0) != cudaSuccess)
    return KVZ_ERR_CUDA;
  auto h2d = [&](uint8_t* dst, const void* src, size_t off, size_t bytes) {
    return cudaMemcpyAsync(dst + off, static_cast<const uint8_t*>(src) + off, bytes, cudaMemcpyHostToDevice,
                           copy_stream);
  };
  for (int64_t c = 0; c < nchunks; ++c) {
    const int64_t h0 = c * p.chunk_heads, nb = (h0 + p.chunk_heads <= B ? p.chunk_heads : B - h0);
    if (h2d(dQ, hQ, static_cast<size_t>(h0 * G * n_in) * row, static_cast<size_t>(nb * G * n_in) * row) ||
        h2d(dKc, hK_ctx, static_cast<size_t>(h0 * n_c) * row, static_cast<size_t>(nb * n_c) * row) ||
        h2d(dKi, hK_in, static_cast<size_t>(h0 * n_in) * row, static_cast<size_t>(nb * n_in) * row) ||
        cudaEventRecord(evs.ev[2 + c], copy_stream) != cudaSuccess)
      return KVZ_ERR_CUDA;
  }
  if (h2d(dV, hV, 0, static_cast<size_t>(B * n_c) * row) || cudaEventRecord(ev_v, copy_stream) != cudaSuccess)
    return KVZ_ERR_CUDA;

  for (int64_t c = 0; c < nchunks; ++c) {
    const int64_t h0 = c * p.chunk_heads, nb = (h0 + p.chunk_heads <= B ? p.chunk_heads : B - h0);
    if (cudaStreamWaitEvent(stream, evs.ev[2 + c], 0) != cudaSuccess) return KVZ_ERR_CUDA;
    kvz_status st = kvz_score(dQ + static_cast<size_t>(h0 * G * n_in) * row, dKc + static_cast<size_t>(h0 * n_c) * row,
                              dKi + static_cast<size_t>(h0 * n_in) * row, nb, G, n_c, n_in, d, scale, 0,
                              dS + h0 * n_c, ws + p.off_lse, p.lse_bytes, d_status, stream);
    if (st != KVZ_OK) return st;
  }
  kvz_status st = kvz_select(dS, B, n_c, ratio, mode, d_idx, p.kept > 0 ? p.kept : 1, d_cnt, d_off,
                             ws + p.off_sel, p.sel_bytes, d_status, stream);
  if (st != KVZ_OK) return st;
  if (cudaStreamWaitEvent(stream, ev_v, 0) != cudaSuccess) return KVZ_ERR_CUDA;
  st = kvz_compact(dKc, dV, B, n_c, d, d_idx, d_cnt, d_off, nullptr, ws + p.off_ko, ws + p.off_vo, nullptr, 0,
                   d_status, stream);
  if (st != KVZ_OK) return st;
  const size_t kept = static_cast<size_t>(p.kept);
  if (cudaMemcpyAsync(h_counts, d_cnt, static_cast<size_t>(B) * 4, cudaMemcpyDeviceToHost, stream) ||
      cudaMemcpyAsync(h_offsets, d_off, static_cast<size_t>(B + 1) * 8, cudaMemcpyDeviceToHost, stream))
    return KVZ_ERR_CUDA;
  if (kept > 0 &&
      (cudaMemcpyAsync(h_idx, d_idx, kept * 4, cudaMemcpyDeviceToHost, stream) ||
       cudaMemcpyAsync(hK_out, ws + p.off_ko, kept * row, cudaMemcpyDeviceToHost, stream) ||
       cudaMemcpyAsync(hV_out, ws + p.off_vo, kept * row, cudaMemcpyDeviceToHost, stream)))
    return KVZ_ERR_CUDA;
  return KVZ_OK;
}

}  // extern "C"
