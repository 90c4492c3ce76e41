/*
 * bdfp4_bf16.h -- the BF16-KV comparator of the FP4 decode path.
 *
 * The pages measure the FP4 cache against a BF16 KV cache ("BitDecoding-FP4
 * tests native 4-bit attention for long contexts", Key Takeaways: 2.4-3.0x
 * the peak throughput of a BF16 cache; "BitDecoding-FP4: Native FP4 KV Cache
 * Decoding via Algorithm-System Co-Design", Article Summary).  This is that
 * baseline built the same way as bdfp4_decode (64-slot pages, 128-token
 * tiles, bulk copies into shared memory, tcgen05 MMA with TMEM accumulators,
 * transposed online softmax, split-KV + merge), with bf16 K, V, Q and P and
 * no quantization, smoothing or rotation: plain softmax(q K^T * sm_scale) V.
 *
 * Cache layout per (page, KV head), d = 128, 16 KB each (bf16, 2 B/element):
 *   k_pages  [num_pages][H_kv][64 * d]: [slot/8][elem/8][slot%8][8 elements]
 *            (the K tile is the A operand of S^T = K q^T, K-major)
 *   v_pages  [num_pages][H_kv][d * 64]: [chan/8][slot/8][chan%8][8 slots]
 *            (V^T per page is the A operand of O^T = V^T P^T, K-major)
 * Slots that no append wrote may hold any bits: the decode masks their logits
 * and zeroes their value columns in shared memory before PV.
 *
 * Conventions are those of bdfp4.h: device pointers, caller-owned memory,
 * asynchronous on `stream` (a cudaStream_t, NULL = default stream), host
 * errors as return codes before any launch, device-found errors OR-ed into
 * *dev_status (BDFP4_DEV_* bits), no traps.  Supported: d = 128 and
 * G = H_q / H_kv in {1, 2, 4, 8, 16}; anything else returns
 * BDFP4_ERR_UNSUPPORTED.  Base pointers of the cache arrays and the workspace
 * must be 128-byte aligned, q/k/v/out 16-byte aligned (BDFP4_ERR_ALIGN).
 */
#ifndef BDFP4_BF16_H
#define BDFP4_BF16_H

#include "bdfp4.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Scatter T tokens of bf16 keys k [T][H_kv][d] and values v [T][H_kv][d] into
 * the pages at slot_mapping[t] = page * 64 + slot (negative = skip; a slot past
 * num_pages * 64 sets BDFP4_DEV_BAD_SLOT and is skipped).  No arithmetic.
 */
BDFP4_API int bdfp4_bf16_append(const void* k, const void* v, const int64_t* slot_mapping, int T, int H_kv, int d,
                                void* k_pages, void* v_pages, int64_t num_pages, int32_t* dev_status, void* stream);

/*
 * Decode one query token per sequence over the bf16 pages:
 *   out[b][h] = sum_t softmax_t(sm_scale q[b][h] . k_t) v_t,  t < seq_lens[b],
 * with query head h reading KV head h / G.  q [B][H_q][d] bf16, out
 * [B][H_q][d] bf16, block_table [B][max_pages_per_seq] int32, seq_lens [B]
 * int32.  Logits and the softmax are fp32; the probabilities enter PV as bf16.
 * chunk_tiles / workspace as in bdfp4_decode (same plan and workspace size,
 * bdfp4_decode_plan / bdfp4_decode_workspace_size).  An empty sequence gives
 * zeros.
 */
BDFP4_API int bdfp4_bf16_decode(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                                const int32_t* seq_lens, int B, int H_q, int H_kv, int d, int max_pages_per_seq,
                                int64_t num_pages, float sm_scale, int chunk_tiles, void* workspace,
                                size_t workspace_bytes, void* out, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BDFP4_BF16_H */
