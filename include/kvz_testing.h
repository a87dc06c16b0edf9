/*
 * kvz_testing.h — test-only entry points of libkvz.  Nothing on the
 * compression path calls them; they exist so that error paths which normal
 * inputs never reach can be exercised on a GPU without faulting it.
 */
#ifndef KVZ_TESTING_H_
#define KVZ_TESTING_H_

#include "kvz.h"

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------------ */
/* In-place compaction with its ordering wait made to expire.                */
/*                                                                          */
/* Same arguments, layout and result as kvz_compact in place (K_out == K,    */
/* V_out == V; KVzip §2.1 pruned cache packed to the front of each head's   */
/* region), except that                                                     */
/*   - every wait of a chunk for the chunks that read its destination rows   */
/*     gives up after wait_ns nanoseconds (kvz_compact: 1 s), and            */
/*   - chunk hold_chunk (slots [16*hold_chunk, 16*hold_chunk + 16)) of head  */
/*     hold_head is written but never reports its source rows as read.       */
/* A chunk that waits on it therefore times out: the kernel sets             */
/* KVZ_ERR_TIMEOUT in d_status, that warp stops (its own and later chunks    */
/* of that head stay unwritten or partly written), and the launch returns.  */
/* Every other head is compacted exactly as kvz_compact would.  The wait is  */
/* a bounded poll of a global counter on %globaltimer; nothing traps.       */
/* Limits: 1000 <= wait_ns <= 1e9; 0 <= hold_head < B; hold_chunk >= 0.     */
/* Workspace: kvz_compact_workspace_size(B, n_c) bytes.                     */
/* ------------------------------------------------------------------------ */
kvz_status kvz_testing_compact_in_place_withhold(void* K, void* V, int64_t B, int64_t n_c, int d,
                                                 const int32_t* idx, const int32_t* counts,
                                                 const int64_t* offsets, void* workspace,
                                                 size_t workspace_bytes, int64_t wait_ns,
                                                 int64_t hold_head, int64_t hold_chunk,
                                                 int32_t* d_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVZ_TESTING_H_ */
