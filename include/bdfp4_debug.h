/*
 * bdfp4_debug.h -- test hooks of libbdfp4.so.  Nothing here is part of the
 * method: these entry points exist so that tests can exercise paths a correct
 * run never takes.
 */
#ifndef BDFP4_DEBUG_H
#define BDFP4_DEBUG_H

#include "bdfp4.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * bdfp4_decode on the d = 128 tensor-core decode (H_q / H_kv = 8, static
 * probability pre-scale: the one shape compiled with this switch) with every
 * in-kernel wait bounded by wait_limit_cycles clock cycles instead of about two
 * seconds, and, when stall is nonzero, each CTA's first K tile never announced
 * to its MMA warp.  The MMA warp's wait for that tile then runs out: the CTA
 * unwinds -- its producer waits (bounded) until every copy it started has
 * landed, its MMA warp until every tensor-core operation it issued has
 * finished, and it frees its tensor memory -- and BDFP4_DEV_TIMEOUT is OR-ed
 * into *dev_status.  The output is then undefined; the device context stays
 * usable.  With stall = 0 the call is bdfp4_decode with the given wait bound.
 * Returns BDFP4_ERR_UNSUPPORTED for other shapes, BDFP4_ERR_ARG for a
 * non-positive bound, else as bdfp4_decode.
 */
BDFP4_API int bdfp4_debug_decode_wait_test(const void* q, const void* k_pages, const void* k_scales,
                                           const void* v_pages, const void* v_scales, const int32_t* block_table,
                                           const int32_t* seq_lens, int B, int H_q, int H_kv, int d_k, int d_v,
                                           int max_pages_per_seq, int64_t num_pages, bdfp4_fmt fmt, int flags,
                                           const bdfp4_kv_params* kv, float sm_scale, int chunk_tiles,
                                           void* workspace, size_t workspace_bytes, void* out, int32_t* dev_status,
                                           long long wait_limit_cycles, int stall, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BDFP4_DEBUG_H */
