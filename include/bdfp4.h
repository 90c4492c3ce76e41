/*
 * bdfp4.h -- C ABI of a B200 (sm_100a) library for decode-time attention over
 * a paged KV cache stored in native 4-bit microscaling formats.
 *
 * The method is BitDecoding-FP4 ("BitDecoding-FP4: Native FP4 KV Cache
 * Decoding via Algorithm-System Co-Design", Article Summary): NVFP4 / MXFP4 KV
 * cache; Outlier-Aware Key Quantization (static smoothing, Hadamard rotation,
 * scale search) under token-wise scaling; Dual-Residual Query Quantization
 * (q ~ q1 + q2, two FP4 tensors); Underflow-Aware Probability Scaling; a
 * transposed softmax with fused probability quantization and stacked-query
 * MMA on paged caches.  How each step is read where the pages leave it open
 * is stated next to the entry point that performs it.
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers unless the name says host_.  The
 *    caller owns and allocates all memory; the library keeps no state between
 *    calls and allocates nothing.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = the
 *    legacy default stream) and is asynchronous; the return code only reports
 *    errors found on the host before launch, or a launch failure.
 *  - Errors the kernels find (bad page index, bad sequence length, bad slot)
 *    are OR-ed into *dev_status (an int32 the caller zeroes and reads after
 *    synchronising); the offending token is skipped, never read or written
 *    out of bounds.  No kernel traps.
 *  - bf16 tensors are row-major with the last dimension contiguous.
 *  - Base pointers of cache arrays and the workspace must be 128-byte aligned;
 *    bf16 inputs 16-byte aligned.
 *
 * Cache layout (a "page" holds 64 token slots for every KV head; beta = 16
 * for NVFP4, 32 for MXFP4; FP4 values are E2M1 codes, two per byte, the
 * even-indexed element in the low nibble; scale codes are E4M3 (NVFP4) or
 * E8M0 (MXFP4) bytes):
 *   k_pages  [num_pages][H_kv][64 * d_k / 2] bytes; within (page, head):
 *            [slot/8][elem/32][slot%8][16 bytes holding elements 32*(elem/32)..+31]
 *   k_scales [num_pages][H_kv][256 * ceil(d_k / (4 beta))]; within (page, head),
 *            the scale of block blk (elements blk*beta..) of slot sits at
 *            [blk/4][slot%32][slot/32][blk%4] (256-byte chunks)
 *   v_pages  [num_pages][H_kv][d_v * 64 / 2]; within (page, head):
 *            [chan/8][slot/32][chan%8][16 bytes holding slots 32*(slot/32)..+31]
 *   v_scales [num_pages][H_kv][d_v * 64 / beta]; scale of the beta-slot block
 *            blk of channel chan: [chan/128][chan%32][(chan%128)/32][blk]
 * K blocks run along the head dim of one token (token-wise scaling); V blocks
 * run along beta consecutive slots of one page for one channel, because the
 * PV product reduces over tokens.  These are the tcgen05 block-scaled MMA
 * operand and scale-factor layouts: each page moves to shared memory with one
 * bulk copy per array and scale chunks move on into tensor memory with
 * tcgen05.cp (a 128-token tile takes MMA rows 0-63 from its first page and
 * 64-127 from its second; lane i of a K scale chunk holds the words of slots
 * i and 32 + i of both pages, 8 contiguous bytes per page).
 *
 * Supported shapes: (d_k, d_v) in {(128, 128), (576, 512)}; H_q / H_kv in
 * {1, 2, 4, 8, 16} or a multiple of 16 up to 128; anything else returns
 * BDFP4_ERR_UNSUPPORTED.
 */
#ifndef BDFP4_H
#define BDFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BDFP4_API __attribute__((visibility("default")))
#else
#define BDFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { BDFP4_NVFP4 = 0, BDFP4_MXFP4 = 1 } bdfp4_fmt;

/* host return codes */
#define BDFP4_OK 0
#define BDFP4_ERR_ARG (-1)         /* null pointer, negative size, bad enum       */
#define BDFP4_ERR_SHAPE (-2)       /* inconsistent sizes                           */
#define BDFP4_ERR_ALIGN (-3)       /* pointer alignment                            */
#define BDFP4_ERR_UNSUPPORTED (-4) /* shape outside the compiled set               */
#define BDFP4_ERR_CUDA (-5)        /* a CUDA launch or query failed                */
#define BDFP4_ERR_WORKSPACE (-6)   /* workspace too small for the split plan      */

/* bits OR-ed into *dev_status by the kernels */
#define BDFP4_DEV_BAD_PAGE 1       /* block_table entry outside [0, num_pages)     */
#define BDFP4_DEV_BAD_SEQLEN 2     /* seq_len < 0 or > max_pages_per_seq * 64      */
#define BDFP4_DEV_BAD_SLOT 4       /* slot_mapping entry >= num_pages * 64         */
#define BDFP4_DEV_TIMEOUT 8        /* a bounded in-kernel wait gave up (the CTA unwound) */

/* flags (ablation arms of the method; 0 = the method as described) */
#define BDFP4_FLAG_NO_HADAMARD 1     /* no rotation of K and q (must match between quantize and decode) */
#define BDFP4_FLAG_NO_SCALE_SEARCH 2 /* keys use the plain amax scale rule                               */
#define BDFP4_FLAG_SINGLE_QUERY 4    /* vanilla single-FP4 query (q2 = 0)                               */
#define BDFP4_FLAG_NO_UNDERFLOW 8    /* vanilla probability scaling (alpha = 1)                         */
/* Variant of the Underflow-Aware Probability Scaling (decode, NVFP4).  The
 * collapse it guards against sits at long contexts ("FP4 KV Cache Done Right",
 * What is actually new; "BitDecoding-FP4 : décodage natif du KV cache FP4",
 * Analyse approfondie).  The probability pre-scale alpha = 2^E is chosen per
 * 128-token tile and query head,
 * E the largest integer with p_max 2^E <= 2688 (p_max the tile's largest
 * probability relative to the running maximum), clamped to [11, 64]; each
 * tile's alpha is divided out of its quantized probabilities.  A tile that
 * raises the running maximum keeps the static 2^11.  Runs in every decode
 * kernel (the tensor-core decodes at d = 128 and for MLA shapes, the CUDA-core
 * decode); with MXFP4 it changes nothing; with BDFP4_FLAG_NO_UNDERFLOW it is
 * BDFP4_ERR_ARG. */
#define BDFP4_FLAG_DYNAMIC_ALPHA 32

/* Static per-layer quantization parameters (device pointers), produced by
 * bdfp4_calibrate (and bdfp4_key_weights) or supplied by the caller. */
typedef struct {
    const float* smooth;   /* [H_kv][d_k]: s_c, each a power of two; keys are divided by s_c, queries multiplied */
    const float* k_gscale; /* [H_kv]: NVFP4 FP32 tensor scale of keys (unused for MXFP4)   */
    const float* v_gscale; /* [H_kv]: NVFP4 FP32 tensor scale of values (unused for MXFP4) */
    /* [H_kv][d_k] channel weights of the attention-aware key scale search
     * (bdfp4_key_weights), or NULL for the plain objective.  Only the key
     * appends read it (bdfp4_quantize_kv, bdfp4_quantize_k, bdfp4_decode_step). */
    const float* k_weight;
} bdfp4_kv_params;

/*
 * Static calibration of the Outlier-Aware Key Quantization parameters
 * ("static smoothing", Article Summary), from a calibration draw.
 * k_cal [Tc][H_kv][d_k], v_cal [Tc][H_kv][d_v], q_cal [Tq][H_q][d_k] bf16.
 * Outputs smooth [H_kv][d_k], k_gscale [H_kv], v_gscale [H_kv] (fp32).
 * Reading: s_c = 2^n, n = round-half-up(log2(kmax_c / qmax_c) / 2) clamped to
 * [-20, 20] (0 when either maximum is 0), kmax over the calibration keys of
 * the head and qmax over the queries of its group; g_k = fp32(amax / 2688) of
 * the transformed calibration keys, g_v = fp32(amax / 2688) of the values
 * (2688 = 6 * 448, the E2M1 and E4M3 maxima), 1 when the amax is 0.
 * Query head h belongs to KV head h / (H_q / H_kv).
 */
BDFP4_API int bdfp4_calibrate(const void* k_cal, const void* q_cal, const void* v_cal, int Tc, int Tq, int H_q, int H_kv,
                    int d_k, int d_v, int flags, float* smooth, float* k_gscale, float* v_gscale, void* stream);

/*
 * Channel weights of the attention-aware key scale search, a variant of the
 * Outlier-Aware Key Quantization's scale search: the pages say the search
 * picks a better scale per group of keys but not by what measure ("FP4 KV
 * Cache Done Right", What is actually new; "BitDecoding-FP4 : décodage natif du
 * KV cache FP4", Analyse approfondie).  This measure weights each element's
 * squared error by what it costs the logits: for channel c of KV head h,
 * w[h][c] = the mean over the calibration queries of the group (Tq tokens x G
 * heads, G = H_q / H_kv) of x_c^2, x = the query transform (smoothing and, unless
 * BDFP4_FLAG_NO_HADAMARD, rotation, as the decode applies them) -- with
 * independent channels, the expected square of the logit error q'.(k' - k^)
 * the block adds.  Sums in fp64 in query order (token, then head), stored as
 * fp32 (the sum divided by Tq G).
 * q_cal [Tq][H_q][d_k] bf16, smooth [H_kv][d_k] (from bdfp4_calibrate), out w
 * [H_kv][d_k] fp32.  Pass w as bdfp4_kv_params.k_weight to select the weighted
 * search.  d_k in {128, 576}.
 */
BDFP4_API int bdfp4_key_weights(const void* q_cal, int Tq, int H_q, int H_kv, int d_k, int flags, const float* smooth,
                                float* w, void* stream);

/*
 * KV-append quantization into the paged cache (Outlier-Aware Key Quantization,
 * Article Summary; "Analyse approfondie" of the French page for what each
 * part does).  k [T][H_kv][d_k], v [T][H_kv][d_v] bf16; slot_mapping [T] int64
 * = page * 64 + slot, or -1 to skip the token.
 * Keys: x = H (k / s) * 2^-ceil(L/2) per power-of-two segment of length 2^L
 * of the head dim (576 = 512 + 64), computed as fixed fp32 butterflies; then
 * per block of beta channels a scale code is searched (NVFP4: E4M3 codes
 * c0+7 .. c0-2 around the plain code c0 = E4M3(amax / (6 g_k)); MXFP4: E8M0
 * codes c0+1, c0 around the OCP MX rule) minimising the block's squared error
 * (fp64, left to right; with kv->k_weight, element i's term is w_i d_i^2, the
 * channel weights of the attention-aware variant), ties to the larger code;
 * elements are E2M1(x / sigma),
 * sigma = fp32(E4M3(c) g_k) or 2^(c-127).
 * Values: the beta-slot blocks of the call's tokens are (re)quantized with the
 * plain rule; a block's tokens must form one run of consecutive tokens with
 * consecutive slots in this call, and slots of a touched block outside the
 * run become zero.  To append a token into a partly filled block, pass the
 * block's earlier tokens again in the same call.
 * Results are bit-identical to the stated fp32/fp64 operation sequence.
 */
BDFP4_API int bdfp4_quantize_kv(const void* k, const void* v, const int64_t* slot_mapping, int T, int H_kv, int d_k, int d_v,
                      bdfp4_fmt fmt, int flags, const bdfp4_kv_params* kv, void* k_pages, void* k_scales,
                      void* v_pages, void* v_scales, int64_t num_pages, int32_t* dev_status, void* stream);

/*
 * The two halves of bdfp4_quantize_kv, each on its own token list (same
 * arguments, layouts, rules and results as the corresponding half there).
 * A decode step appends the new token's key with bdfp4_quantize_k, and
 * re-quantizes the open value block (the new token and the earlier tokens of
 * its beta-slot block, kept in bf16 by the caller) with bdfp4_quantize_v: a
 * key is quantized per token, so stored keys never need touching again.
 * bdfp4_quantize_v reports nothing through a status word (bad slots are
 * skipped; bdfp4_quantize_k reports them).
 */
BDFP4_API int bdfp4_quantize_k(const void* k, const int64_t* slot_mapping, int T, int H_kv, int d_k, bdfp4_fmt fmt,
                    int flags, const bdfp4_kv_params* kv, void* k_pages, void* k_scales, int64_t num_pages,
                    int32_t* dev_status, void* stream);
BDFP4_API int bdfp4_quantize_v(const void* v, const int64_t* slot_mapping, int T, int H_kv, int d_v, bdfp4_fmt fmt,
                    const bdfp4_kv_params* kv, void* v_pages, void* v_scales, int64_t num_pages, void* stream);

/*
 * Dual-Residual Query Quantization on its own (Article Summary; the French
 * page: the second FP4 tensor encodes the residual of the first), exactly as
 * the decode prologue performs it.  q [B][H_q][d_k] bf16.  Query transform:
 * x = H (q * s) * 2^-floor(L/2).  NVFP4: g_q = fp32(amax(x) / 2688) per query
 * head (1 if 0); q1 = plain-rule FP4 of x; r = fp32(x - fp32(e1 * sigma1));
 * q2 = plain-rule FP4 of r with the same g_q.  MXFP4: E8M0 scales, no g_q.
 * Outputs (logical layout, one E2M1 code per byte): q1_codes, q2_codes
 * [B][H_q][d_k]; q1_scales, q2_scales [B][H_q][d_k / beta]; g_q [B][H_q].
 */
BDFP4_API int bdfp4_quantize_q(const void* q, int B, int H_q, int H_kv, int d_k, bdfp4_fmt fmt, int flags, const float* smooth,
                     uint8_t* q1_codes, uint8_t* q1_scales, uint8_t* q2_codes, uint8_t* q2_scales, float* g_q,
                     void* stream);

/*
 * Split plan for bdfp4_decode: tiles (128 tokens) per split.  Each split is
 * one CTA; at four CTAs per SM a grid runs in ceil(CTAs / (4 num_sms)) waves of
 * about c + 3 tile-times.  The plan is the c in [16, 64] (at most the longest
 * sequence's tiles) minimising that product, the longer c on ties.
 * host_seq_lens [B] is a HOST array.  Returns chunk_tiles >= 1, or a negative
 * status.  Sequence b then has ceil(ceil(N_b / 128) / chunk_tiles) splits.
 */
BDFP4_API int bdfp4_decode_plan(const int32_t* host_seq_lens, int B, int H_kv, int num_sms);

/*
 * The same plan for the kernel bdfp4_decode runs on this shape (H_q query heads,
 * head dims d_k / d_v): its CTAs per SM (4 for d = 128 with up to four query
 * heads per KV head, 3 up to sixteen, 1 for the MLA tensor-core kernel) and its
 * CTAs per split (one per KV head, times the 64-head slices of the MLA kernel).
 * bdfp4_decode_plan is this with four CTAs per SM and one CTA per KV head.
 * Returns chunk_tiles >= 1, or a negative status (BDFP4_ERR_SHAPE if H_q is not a
 * multiple of H_kv, BDFP4_ERR_UNSUPPORTED for head dims outside the compiled set).
 */
BDFP4_API int bdfp4_decode_plan_for(const int32_t* host_seq_lens, int B, int H_q, int H_kv, int d_k, int d_v,
                                    int num_sms);

/* The plan for bdfp4_decode_multi with T_q query tokens per sequence (T_q = 1
 * is bdfp4_decode_plan_for): the kernel that runs G T_q stacked rows per KV head
 * -- the d = 128 tensor-core decode at up to 16 rows, three (four up to four
 * rows) CTAs per SM; the CUDA-core decode otherwise. */
BDFP4_API int bdfp4_decode_multi_plan(const int32_t* host_seq_lens, int B, int T_q, int H_q, int H_kv, int d_k,
                                      int d_v, int num_sms);

/* Bytes of workspace bdfp4_decode needs for this shape and chunk_tiles: the
 * fp32 partial outputs and (m, l) pairs of the splits (when a sequence can
 * have more than one), then 656 bytes per query head for the query images the
 * tensor-core paths (d_k = 128; MLA d_k = 576 with G = 16, 32, 64 or 128)
 * compute once per (sequence, KV head, head slice) before the decode kernel
 * reads them.  Contents need no initialisation; calls that run at the
 * same time must not share a workspace. */
BDFP4_API size_t bdfp4_decode_workspace_size(int B, int H_q, int d_v, int max_pages_per_seq, int chunk_tiles);

/*
 * FP4 paged decode attention, one query token per sequence.
 * q [B][H_q][d_k] bf16; block_table [B][max_pages_per_seq] int32 page ids;
 * seq_lens [B] int32; out [B][H_q][d_v] bf16.
 * Per (sequence, query head): the query is transformed and dual-residual
 * quantized; logits s_t = sm_scale g_q g_k (q1 + q2) . k_t over the paged keys;
 * an online softmax runs over 128-token tiles from the sequence start, cut
 * into splits of chunk_tiles tiles; per tile p_t = exp(s_t - m_new), l sums the
 * unquantized p, and P is quantized in beta-token blocks (NVFP4: alpha = 2^11
 * underflow-aware pre-scale, divided out exactly; E4M3 block scale of
 * amax(alpha p) / 6, code 0 collapses the block; MXFP4: E8M0, alpha = 1;
 * BDFP4_FLAG_DYNAMIC_ALPHA: alpha per tile and head, see the flag);
 * O accumulates P^ V; splits merge by log-sum-exp.  An empty sequence gives
 * zeros.  chunk_tiles <= 0 picks a plan from device seq_lens' upper bound
 * (max_pages_per_seq * 64).  workspace: >= bdfp4_decode_workspace_size bytes
 * (required on the tensor-core paths and whenever a sequence can have several
 * splits).
 */
BDFP4_API int bdfp4_decode(const void* q, const void* k_pages, const void* k_scales, const void* v_pages,
                 const void* v_scales, const int32_t* block_table, const int32_t* seq_lens, int B, int H_q, int H_kv,
                 int d_k, int d_v, int max_pages_per_seq, int64_t num_pages, bdfp4_fmt fmt, int flags,
                 const bdfp4_kv_params* kv, float sm_scale, int chunk_tiles, void* workspace,
                 size_t workspace_bytes, void* out, int32_t* dev_status, void* stream);

/*
 * One decode step in one call: append each sequence's new token to the FP4
 * cache, then decode (the paper's generation loop -- the KV-append
 * quantization of the Article Summary's kernel followed by its decode
 * attention).  seq_lens[b] = N_b counts the new token, which goes to position
 * N_b - 1, i.e. slot (N_b - 1) % 64 of page block_table[b][(N_b - 1) / 64].
 *   k_new [B][H_kv][d_k], v_new [B][H_kv][d_v] bf16: the new keys and values.
 *   v_open [B][beta][H_kv][d_v] bf16, caller-owned and kept across steps: the
 *     open value block of each sequence, row i = slot (N_b - 1) - (N_b - 1) %
 *     beta + i.  The call writes v_new into row (N_b - 1) % beta and re-
 *     quantizes the block from rows 0 .. (N_b - 1) % beta (the rows before it
 *     must hold the block's earlier tokens: written by earlier steps, or by
 *     the caller after a prefill); the block's later slots become zero.
 * The cache bytes after the call equal those of bdfp4_quantize_k on the new
 * keys plus bdfp4_quantize_v on each open block's run of tokens; the output
 * is bdfp4_decode's over the updated cache.  Sequences with N_b = 0 append
 * nothing.  Other arguments, the workspace and the status bits are those of
 * bdfp4_decode (k_new and v_new 16-byte aligned).  On the d_k = 128 path the
 * append and the query images run in one prologue grid that the decode
 * overlaps; only each sequence's last tile waits for it.
 */
BDFP4_API int bdfp4_decode_step(const void* q, const void* k_new, const void* v_new, void* v_open, void* k_pages,
                                void* k_scales, void* v_pages, void* v_scales, const int32_t* block_table,
                                const int32_t* seq_lens, int B, int H_q, int H_kv, int d_k, int d_v,
                                int max_pages_per_seq, int64_t num_pages, bdfp4_fmt fmt, int flags,
                                const bdfp4_kv_params* kv, float sm_scale, int chunk_tiles, void* workspace,
                                size_t workspace_bytes, void* out, int32_t* dev_status, void* stream);

/*
 * Decode attention for several query tokens per sequence: speculative
 * verification or chunked decode, the T_q newest tokens of each sequence
 * (already appended to the cache) attending causally.  The pages describe one
 * query token per step; this extends their stacked-query MMA ("BitDecoding-FP4:
 * Native FP4 KV Cache Decoding via Algorithm-System Co-Design", Article
 * Summary: query operations stacked over the paged cache; "BitDecoding-FP4 :
 * décodage natif du KV cache FP4", Analyse approfondie) from the G heads of a
 * KV group to the G T_q (token, head) rows, which share each K/V tile read.
 * q [B][T_q][H_q][d_k] bf16, out [B][T_q][H_q][d_v] bf16.  Query token i of
 * sequence b (N_b = seq_lens[b] tokens, the last T_q of them the query tokens)
 * sees the first N_b - T_q + 1 + i tokens and gets exactly bdfp4_decode's
 * arithmetic on that prefix, with the same 128-token tiles and chunk_tiles
 * splits from the sequence start.  A sequence with 0 < N_b < T_q sets
 * BDFP4_DEV_BAD_SEQLEN (its rows that would see no token give zeros); N_b = 0
 * gives zeros.  workspace: >= bdfp4_decode_workspace_size(B * T_q, H_q, d_v,
 * max_pages_per_seq, chunk_tiles) bytes; chunk_tiles from
 * bdfp4_decode_multi_plan (<= 0 plans from max_pages_per_seq).  Flags,
 * layouts and other arguments as bdfp4_decode; T_q = 1 is bdfp4_decode.
 */
BDFP4_API int bdfp4_decode_multi(const void* q, const void* k_pages, const void* k_scales, const void* v_pages,
                                 const void* v_scales, const int32_t* block_table, const int32_t* seq_lens, int B,
                                 int T_q, int H_q, int H_kv, int d_k, int d_v, int max_pages_per_seq,
                                 int64_t num_pages, bdfp4_fmt fmt, int flags, const bdfp4_kv_params* kv,
                                 float sm_scale, int chunk_tiles, void* workspace, size_t workspace_bytes, void* out,
                                 int32_t* dev_status, void* stream);

/*
 * bdfp4_decode without a caller-provided workspace.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory themselves -- for example an operator plugged into a host
 * framework that hands it only its inputs and outputs (no workspace hook), or
 * a latency-critical serving loop that must not call into an allocator.
 * The split-KV partials go to a scratch array compiled into the library
 * (a file-scope __device__ array of BDFP4_NOALLOC_SCRATCH_BYTES bytes that
 * every GPU loading the library holds until the process exits); nothing is
 * allocated by this call.  Arguments are those of bdfp4_decode without
 * workspace / workspace_bytes.
 *  - If the split plan (chunk_tiles, or the automatic plan when chunk_tiles
 *    <= 0) needs more scratch than BDFP4_NOALLOC_SCRATCH_BYTES, the call
 *    returns BDFP4_ERR_WORKSPACE; pass a larger chunk_tiles to fit.
 *  - The first call on each device looks up the scratch array's device
 *    address (cudaGetSymbolAddress) with that device current; make that first
 *    call before any stream capture.  A failed lookup returns BDFP4_ERR_CUDA.
 *    The address is kept for the life of the process: it does not survive a
 *    cudaDeviceReset (or any other teardown of the device's primary context),
 *    after which this entry point must not be called again in that process.
 *  - All calls share the one array and it keeps the last call's contents (no
 *    part of it needs to start at zero: every partial is written before it is
 *    read).  Calls that overlap on the GPU -- on different streams, or from
 *    different host threads without ordering -- race on it.
 */
#define BDFP4_NOALLOC_SCRATCH_BYTES (16u << 20)
BDFP4_API int bdfp4_decode_noalloc(const void* q, const void* k_pages, const void* k_scales, const void* v_pages,
                                   const void* v_scales, const int32_t* block_table, const int32_t* seq_lens, int B,
                                   int H_q, int H_kv, int d_k, int d_v, int max_pages_per_seq, int64_t num_pages,
                                   bdfp4_fmt fmt, int flags, const bdfp4_kv_params* kv, float sm_scale,
                                   int chunk_tiles, void* out, int32_t* dev_status, void* stream);

/* Human-readable text of a host return code. */
BDFP4_API const char* bdfp4_status_string(int status);

/* Name and text of the last CUDA error this thread's calls into the library
 * met (the detail behind BDFP4_ERR_CUDA); the string stays valid until the
 * thread's next failing call. */
BDFP4_API const char* bdfp4_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BDFP4_H */
