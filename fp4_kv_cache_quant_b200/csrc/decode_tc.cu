// decode_tc.cu -- FP4 paged decode attention on the sm_100a tensor cores
// (BitDecoding-FP4, Article Summary: stacked query MMA on paged KV caches,
// transposed softmax with fused probability quantization, dual-residual
// query, underflow-aware probability scaling), for d_k = d_v = 128.
//
// One CTA per (sequence, KV head, split), four (up to four heads per KV head)
// or three per SM; ten warps (six for a single head):
//   producer    reads the block table and bulk-copies each 128-token tile (two
//               pages: K nibbles, K scales, V nibbles, V scales) into a K ring
//               and a V ring (mbarrier complete_tx);
//   MMA         one lane issues, the warp owns TMEM:
//                 S^T[token, q-row] = K_tile . [q1; q2]^T   (M = 128 tokens,
//                 N = 2G stacked query rows, block-scaled E2M1, fp32 in TMEM),
//                 O^T[chan, head]  += V^T . P^T             (M = 128 channels,
//                 N = G heads, K = the tile's tokens, one MMA per page),
//               O^T accumulating across the split's tiles;
//   softmax     two groups of four warps (one for a single head), each group
//               half of the heads: thread t owns token t of the tile (TMEM lane
//               t), so the softmax is transposed -- per-head maxima are warp
//               reductions, the FP4 quantization of P (beta-token blocks) takes
//               the maximum over the lanes of a block, and the P codes go
//               straight into the shared-memory operand of the PV MMA.  A
//               head's running maximum and per-tile terms are computed once per
//               warp, by the lanes that hold the head, and shuffled to the
//               others.  The same threads write the block-scale factors of P
//               and, when a running maximum rises, rescale their heads' O^T
//               columns in TMEM between the previous tile's PV and this one's.
// The dynamic variant (DYN, NVFP4) picks the probability pre-scale per tile and
// head and folds a change of it into that same rescale.
// Every wait is bounded; a timeout sets BDFP4_DEV_TIMEOUT and the CTA unwinds.

#include <type_traits>

#include "append_device.cuh"
#include "bdfp4_device.cuh"
#include "decode_common.cuh"
#include "host_common.h"
#include "prob_scale.cuh"
#include "quant_device.cuh"
#include "tc_ptx.cuh"


namespace bdfp4 {

template <int FMT, int G>
struct TcCfg {
    static constexpr int B = Fmt<FMT>::beta;
    static constexpr int DK = 128, DV = 128;
    static constexpr int NQ = (2 * G < 8) ? 8 : 2 * G;  // N of the QK MMA (q1 rows, q2 rows, padding)
    static constexpr int NP = (G < 8) ? 8 : G;          // N of the PV MMA
    static constexpr int KS = DK / 64;                   // MMA K steps of QK
    // CTAs per SM the register budget is shaped for: four for up to four heads
    // (4 x 10 warps at 48 registers), three for more (3 x 10 warps at 64)
    static constexpr int MIN_CTAS = G <= 4 ? 4 : 3;
    // two shared-memory rings: K stages are released when QK completes, V stages
    // when PV completes, so K (needed first) is prefetched further ahead; with four
    // CTAs per SM the rings are shallower (the SM holds as many tiles in flight)
    static constexpr int NSK = MIN_CTAS == 4 ? 3 : 4;
    static constexpr int NSV = MIN_CTAS == 4 ? 2 : 3;
    // tiles the V copies trail the K copies by: one (only PV needs V, and K is needed first)
    static constexpr int VLAG = 1;
    // softmax warpgroups: warps w and w + 4 read the same TMEM lanes (tokens), so
    // two groups split the query heads of every tile between them
    static constexpr int NSG = G >= 2 ? 2 : 1;
    static constexpr int HG = G / NSG;                   // heads per group
    static constexpr int NSW = 4 * NSG;                  // softmax warps
    static constexpr int PRODUCER = NSW, MMA_WARP = NSW + 1;
    static constexpr int THREADS = 32 * (NSW + 2);
    static constexpr int K_PAGE = kPageSlots * DK / 2;   // 4096
    static constexpr int NKG = (DK / B + 3) / 4;         // 4-block K scale groups per token (2 / 1)
    static constexpr int KPG = KS / NKG;                 // K steps per scale group (1 NVFP4, 2 MXFP4)
    static constexpr int KS_PAGE = 256 * NKG;            // K scale bytes per page (512 / 256)
    static constexpr int V_PAGE = DV * kPageSlots / 2;   // 4096
    static constexpr int VS_PAGE = DV * kPageSlots / B;
    // K stage of a 128-token tile: K of page 0 (MMA rows 0-63) and page 1 (rows
    // 64-127), then per scale group the 32 x 16-byte tcgen05.cp source: row i
    // holds the scale words of rows i, 32 + i, 64 + i, 96 + i
    static constexpr int OFF_K = 0;
    static constexpr int OFF_KS = 2 * K_PAGE;
    static constexpr int KSTAGE = OFF_KS + NKG * 512;
    // V stage: V [page][4 KB], then V scales [page][VS_PAGE]
    static constexpr int OFF_V = 0;
    static constexpr int OFF_VS = 2 * V_PAGE;
    static constexpr int VSTAGE = OFF_VS + 2 * VS_PAGE;
    static constexpr int Q_BYTES = (NQ / 8) * (DK / 32) * 128;
    static constexpr int P_PAGE = (NP / 8) * 256;
    static constexpr int P_BUF = 2 * P_PAGE;
    static constexpr int SPB = 64 / B;                   // scale blocks per 64 tokens / elements
    // the query image of a (sequence, KV head), copied into shared memory in one
    // piece: QK operand, its scale codes [NQ][8], the per-head logit scales [G]
    static constexpr int LSC_BYTES = (G * 4 + 15) / 16 * 16;
    static constexpr int QPACK = Q_BYTES + NQ * 8 + LSC_BYTES;
    static constexpr int QTHREADS = (G * RowGeom<FMT, 128>::rt + 31) / 32 * 32;   // threads of prep_query_kernel
    // shared memory map
    static constexpr int SM_KST = 0;
    static constexpr int SM_VST = SM_KST + NSK * KSTAGE;
    static constexpr int SM_Q = SM_VST + NSV * VSTAGE;
    static constexpr int SM_QSC = SM_Q + Q_BYTES;
    static constexpr int SM_LSC = SM_QSC + NQ * 8;
    static constexpr int SM_P = SM_Q + QPACK;
    static constexpr int SM_PSF = (SM_P + 2 * P_BUF + 127) / 128 * 128;  // [2 buf][2 page][32 rows][16 B] P scales
    // MXFP4: [2 buf][32 rows][16 B] V scales of a tile's two pages, interleaved by the MMA warp
    static constexpr int SM_VSF = SM_PSF + 2 * 2 * 512;
    // per S buffer: [G][4] warp maxima (floats)
    static constexpr int RED_BUF = 4 * G;
    static constexpr int SM_RED = SM_VSF + (FMT == BDFP4_MXFP4 ? 2 * 512 : 0);
    static constexpr int SM_BARS = (SM_RED + 2 * RED_BUF * 4 + 7) / 8 * 8;
    static constexpr int NBARS = 2 * NSK + 2 * NSV + 8;
    static constexpr int SM_MISC = SM_BARS + NBARS * 8;                  // tmem slot, abort flags
    static constexpr int SM_PFLAG = SM_MISC + 16;                        // [64] page flags of the split's tiles, any-bad
    static constexpr int SMEM = SM_PFLAG + 64 + 16;
    // TMEM column map
    static constexpr int T_S = 0;
    static constexpr int T_O = 2 * NQ;
    static constexpr int T_SFK = ((T_O + NP + 3) / 4) * 4;       // 2 x (4 per K scale group x NKG)
    // 2 x (4 per page x 2 pages); MXFP4 2 x 4: a column holds a channel's 2 scale bytes of
    // each page, page 0 in bytes 0-1 and page 1 in bytes 2-3 (scale-factor id 2)
    static constexpr int T_SFV = T_SFK + 2 * 4 * NKG;
    // every scale-factor operand starts on a 4-column boundary (one 32-bit
    // column per 32 rows of a 128-row chunk), B operands included
    static constexpr int T_SFQ = T_SFV + 2 * 8;                  // KS x 4 columns
    static constexpr int T_SFP = T_SFQ + 4 * KS;                 // 2 buffers x 2 pages x 4 columns
    static constexpr int T_USED = T_SFP + 16;
    static constexpr int T_ALLOC = T_USED <= 32 ? 32 : T_USED <= 64 ? 64 : T_USED <= 128 ? 128 : 256;
    // TMEM holds 512 columns per SM; request enough shared memory that one CTA
    // more than TMEM can serve never becomes resident (it would only wait in
    // tcgen05.alloc): with k = 512 / T_ALLOC CTAs per SM, (k + 1) * (smem + 1 KB)
    // must exceed the 228 KB of an SM
    static constexpr int MAX_CTAS = 512 / T_ALLOC;
    static constexpr int SMEM_MIN = 233472 / (MAX_CTAS + 1) - 1024 + 16;
    static constexpr int SMEM_LAUNCH = SMEM > SMEM_MIN ? SMEM : SMEM_MIN;
    // the query image of a (sequence, KV head) fits the workspace region reserved for it
    static_assert(QPACK <= kQueryImageBytes * G, "query image larger than its workspace share");
    static_assert(QPACK % 16 == 0, "query image copied in 16-byte units");
};


// Query image of one (sequence, KV head): smoothing + Hadamard transform and
// dual-residual FP4 of its G query heads, laid out as the decode CTA keeps them
// in shared memory (QK operand rows: group (r / HG) owns 2 HG consecutive rows,
// q1 of its heads then q2, so a softmax warp loads both logits of its heads with
// one TMEM load; element e -> chunk e/32, byte (e%32)/2; then the scale codes
// [NQ][8] and the logit scales sm_scale g_q g_k log2(e) per head).  Every split of
// the sequence copies it instead of recomputing it.
// One CTA (at least QTHREADS threads) builds the image of (sequence b, KV head hk).
// MT (several query tokens per sequence): the G stacked rows are the T_q
// tokens' query heads of the group, token-major (stacked_row).
template <int FMT, int G, bool MT = false>
__device__ __forceinline__ void query_image_cta(const DecodeArgs& a, int hk, int b) {
    using C = TcCfg<FMT, G>;
    using RG = RowGeom<FMT, 128>;
    constexpr int B = C::B, HG = C::HG;
    __shared__ __align__(16) uint8_t img[C::QPACK];
    __shared__ int row_amax[G];
    uint8_t* q_op = img;
    uint8_t* qsc = img + C::Q_BYTES;
    float* lsc = reinterpret_cast<float*>(img + C::Q_BYTES + C::NQ * 8);
    const int tid = threadIdx.x, h0 = hk * G;
    const bool hadamard = !(a.flags & BDFP4_FLAG_NO_HADAMARD);
    const bool dual = !(a.flags & BDFP4_FLAG_SINGLE_QUERY);
    for (int i = tid; i < C::QPACK / 16; i += blockDim.x) reinterpret_cast<uint4*>(img)[i] = make_uint4(0, 0, 0, 0);
    if (tid < G) row_amax[tid] = 0;
    __syncthreads();
    const int j = tid % RG::rt, r = tid / RG::rt;
    const bool active = r < G && j < RG::tpr;
    float x[B];
    if (active) {
        const int64_t qrow = MT ? stacked_row(a, b, hk, r) : (int64_t)b * a.H_q + h0 + r;
        load_bf16_block<B>(a.q + qrow * C::DK, j * B, x);
    } else {
#pragma unroll
        for (int i = 0; i < B; ++i) x[i] = 0.0f;
    }
    transform_block<FMT, 128, false>(x, a.smooth + (int64_t)hk * C::DK, j, hadamard);
    if (active) atomicMax(&row_amax[r], __float_as_int(block_amax<B>(x)));
    __syncthreads();
    if (active) {
        const float amax = __int_as_float(row_amax[r]);
        const float gq = FMT == BDFP4_NVFP4 ? (amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f) : 1.0f;
        uint32_t c1, c2, p1[B / 8], p2[B / 8];
        quantize_query_block<FMT, 128>(x, gq, dual, c1, p1, c2, p2);
        const int e0 = j * B;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int row = (r / HG) * 2 * HG + half * HG + r % HG;
            const uint32_t* pk = half ? p2 : p1;
            uint8_t* dst = q_op + (row / 8) * 512 + (e0 / 32) * 128 + (row % 8) * 16 + (e0 % 32) / 2;
            if constexpr (B == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            qsc[row * 8 + j] = (uint8_t)(half ? c2 : c1);
        }
        if (j == 0) {
            const float gk = FMT == BDFP4_NVFP4 ? a.k_gscale[hk] : 1.0f;
            lsc[r] = a.sm_scale * gq * gk * kLog2e;
        }
    }
    __syncthreads();
    uint4* out = reinterpret_cast<uint4*>(a.qpack + ((int64_t)b * a.H_kv + hk) * C::QPACK);
    for (int i = tid; i < C::QPACK / 16; i += blockDim.x) out[i] = reinterpret_cast<const uint4*>(img)[i];
}

template <int FMT, int G, bool MT = false>
__global__ void __launch_bounds__(TcCfg<FMT, G>::QTHREADS) prep_query_kernel(const DecodeArgs a) {
    // the decode grid may start now; it waits for this grid before copying the image
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    query_image_cta<FMT, G, MT>(a, blockIdx.x, blockIdx.y);
}

// Decode-step prologue: one grid whose CTAs take three roles side by side --
// the key append of every sequence's new token, the value append of its open
// block, and the query images -- so a step costs one launch ahead of the
// decode.  The decode grid starts as soon as every CTA here has started.
template <int FMT, int G>
__global__ void __launch_bounds__(256) prep_step_kernel(const DecodeArgs a, const StepArgs s) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t rows = (int64_t)a.B * a.H_kv;
    const NewestSlot slot{a.block_table, a.seq_lens, a.max_pages, a.num_pages, a.dev_status};
    const int nk = (int)k_append_ctas_wide<FMT, 128>(rows), nv = (int)v_append_ctas<128>(rows);
    const int blk = blockIdx.x;
    if (blk < nk) {
        append_k_cta_wide<FMT, 128>(blk, s.k_new, rows, a.H_kv, slot, a.smooth, a.k_gscale, a.k_weight, s.k_pages,
                                    s.k_scales, a.flags);
    } else if (blk < nk + nv) {
        append_v_open_cta<FMT, 128>(blk - nk, s.v_new, s.v_open, slot, a.B, a.H_kv, a.v_gscale, s.v_pages,
                                    s.v_scales);
    } else {
        const int qi = blk - nk - nv;
        query_image_cta<FMT, G>(a, qi % a.H_kv, qi / a.H_kv);
    }
}

// MT: several query tokens per sequence (a.T_q), their query heads stacked as
// the G rows (token-major); query token i sees the first N - T_q + 1 + i tokens.
// HOOK: the unwind test's instantiation (bdfp4_debug.h) -- its wait bound and
// its first-tile stall come from the arguments; every other instantiation bounds
// its waits at the compile-time kWaitLimitDefault.
template <int FMT, int G, bool DYN = false, bool MT = false, bool HOOK = false>
__global__ void __launch_bounds__(TcCfg<FMT, G>::THREADS, TcCfg<FMT, G>::MIN_CTAS) decode_tc_kernel(const DecodeArgs a) {
    using C = TcCfg<FMT, G>;
    const long long wlim = HOOK ? a.wait_limit : kWaitLimitDefault;
    const bool stall = HOOK && a.test_stall;
    // the split merge (a programmatic dependent) may be scheduled as CTAs of this grid retire
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr bool MX = FMT == BDFP4_MXFP4;
    constexpr int B = C::B;
    constexpr int HG = C::HG;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* q_op = smem + C::SM_Q;
    uint8_t* p_op = smem + C::SM_P;
    uint8_t* qsc = smem + C::SM_QSC;
    uint8_t* psf = smem + C::SM_PSF;
    float* red = reinterpret_cast<float*>(smem + C::SM_RED);
    float* lsc = reinterpret_cast<float*>(smem + C::SM_LSC);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SM_BARS);
    uint64_t* kfull = bars;                   // [NSK] K tile landed -> MMA
    uint64_t* kempty = kfull + C::NSK;        // [NSK] QK done -> producer
    uint64_t* vfull = kempty + C::NSK;        // [NSV] V tile landed -> MMA, softmax
    uint64_t* vempty = vfull + C::NSV;        // [NSV] PV done -> producer
    uint64_t* s_full = vempty + C::NSV;       // [2] QK done -> softmax
    uint64_t* p_ready = s_full + 2;           // [2] P + scale factors ready -> MMA
    uint64_t* o_full = p_ready + 2;           // [2] PV done -> softmax (rescale, epilogue)
    uint64_t* q_ready = o_full + 2;           // query operand and its scale factors -> MMA
    uint64_t* q_full = q_ready + 1;           // query image landed -> softmax
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SM_MISC + 4);   // any role gave up

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int h0 = hk * G;

    int N = a.seq_lens[b];
    if (N < 0 || N > a.max_pages * kPageSlots) {
        if (tid == 0 && split == 0) set_status(a.dev_status, BDFP4_DEV_BAD_SEQLEN);
        N = 0;
    }
    // MT: a sequence must hold its T_q query tokens (rows that would see no token give zeros)
    if (MT && N > 0 && N < a.T_q && tid == 0 && split == 0) set_status(a.dev_status, BDFP4_DEV_BAD_SEQLEN);
    // output / partial row of stacked row v
    auto row_of = [&](int v) -> int64_t {
        if constexpr (MT) return stacked_row(a, b, hk, v);
        else return (int64_t)b * a.H_q + h0 + v;
    };
    const int ntiles = (N + kTileTokens - 1) / kTileTokens;
    const int nspl = (ntiles + a.chunk_tiles - 1) / a.chunk_tiles;
    if (split > 0 && split >= nspl) return;
    if (N == 0) {
        for (int i = tid; i < G * C::DV; i += blockDim.x) a.out[row_of(i / C::DV) * C::DV + i % C::DV] = __float2bfloat16(0.0f);
        return;
    }
    const int tile0 = split * a.chunk_tiles;
    const int n = min(a.chunk_tiles, ntiles - tile0);   // tiles of this split (>= 1)

    if (tid == 0) {
        for (int s = 0; s < C::NSK; ++s) {
            tc::mbar_init(&kfull[s], 1 + 32);   // the byte count, then the producer lanes' cp.async
            tc::mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < C::NSV; ++s) {
            tc::mbar_init(&vfull[s], 1);
            tc::mbar_init(&vempty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&s_full[i], 1);
            tc::mbar_init(&p_ready[i], C::NSW);
            tc::mbar_init(&o_full[i], 1);
        }
        tc::mbar_init(q_ready, C::NSW);
        tc::mbar_init(q_full, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == C::MMA_WARP) {
        tc::tmem_alloc(tmem_slot, C::T_ALLOC);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == C::PRODUCER) {
        // ------------------------------------------------------------ producer
        // Step k issues the K half of tile k and the V half of tile k - VLAG, each
        // into its own ring, so K runs VLAG tiles ahead of V.  The warp reads the
        // page ids of 32 tiles at once (one tile per lane), so the dependent
        // block-table load is off the per-tile path; lane 0 then waits for free
        // stages, and one lane per bulk copy issues a step's copies together (a
        // single thread issuing them one after another is slower than the tiles
        // are consumed).
        bool ok = true;
        int pv0 = -1, pv1 = -1;   // pages of the previous tile (the V half of this step)
        int k_last = -1, v_last = -1;   // the last tiles whose K / V halves were announced
        for (int j0 = 0; ok && j0 <= n; j0 += 32) {
            int pg_l[2] = {-1, -1};
            if (j0 + lane < n) {
                const int tile = tile0 + j0 + lane;
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const int pi = tile * 2 + p;
                    if (pi * kPageSlots < N) {
                        const int v = a.block_table[(int64_t)b * a.max_pages + pi];
                        if (v >= 0 && v < a.num_pages) pg_l[p] = v;
                        else set_status(a.dev_status, BDFP4_DEV_BAD_PAGE);
                    }
                }
            }
            const int kmax = min(32, n + 1 - j0);
            for (int kk = 0; kk < kmax; ++kk) {
                const int k = j0 + kk;
                const int pg0 = __shfl_sync(0xffffffffu, pg_l[0], kk);
                const int pg1 = __shfl_sync(0xffffffffu, pg_l[1], kk);
                const int v = k - C::VLAG;   // the tile whose V half this step issues
                const bool do_k = k < n, do_v = v >= 0 && v < n;
                const int ks = k % C::NSK, vsi = (v + C::NSV) % C::NSV;
                const int pv0_ = C::VLAG ? pv0 : pg0, pv1_ = C::VLAG ? pv1 : pg1;
                // K half: lane 0 claims the stage and posts the byte count; lanes 0-1 bulk-copy
                // the two K pages and every lane copies, with cp.async, the 8 scale bytes of
                // slots lane and 32 + lane of each page and scale group into row lane of the
                // group's tcgen05.cp source, then arrives on the stage barrier once they land
                // the unwind test withholds tile 0's K half: the MMA warp's wait for it runs out
                if (do_k && !(stall && k == 0)) {
                    // the step prologue writes the new token into the sequence's last page:
                    // that tile's copies wait until the prologue grid has finished
                    if (a.append_wait && tile0 + k == ntiles - 1) asm volatile("griddepcontrol.wait;" ::: "memory");
                    if (lane == 0) {
                        if (k >= C::NSK && !tc::mbar_wait(&kempty[ks], ((k / C::NSK) - 1) & 1, abort_flag, wlim))
                            ok = false;
                        else
                            tc::mbar_arrive_expect_tx(&kfull[ks], (pg0 >= 0 ? C::K_PAGE : 0) + (pg1 >= 0 ? C::K_PAGE : 0));
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    uint8_t* stg = smem + C::SM_KST + ks * C::KSTAGE;
                    if (lane < 2) {
                        const int pg = lane ? pg1 : pg0;
                        if (pg >= 0)
                            tc::bulk_g2s(stg + C::OFF_K + lane * C::K_PAGE,
                                         a.k_pages + ((int64_t)pg * a.H_kv + hk) * C::K_PAGE, C::K_PAGE, &kfull[ks]);
                    }
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const int pg = p ? pg1 : pg0;
                        if (pg < 0) continue;
                        const uint8_t* ksrc = a.k_scales + ((int64_t)pg * a.H_kv + hk) * C::KS_PAGE + lane * 8;
#pragma unroll
                        for (int kg = 0; kg < C::NKG; ++kg)
                            tc::cp_async_8(stg + C::OFF_KS + kg * 512 + lane * 16 + p * 8, ksrc + kg * 256);
                    }
                    tc::cp_async_mbar_arrive_noinc(&kfull[ks]);
                    k_last = k;
                }
                // V half of tile v: lanes 0-1 copy the V pages, 2-3 their scales
                if (do_v) {
                    if (lane == 0) {
                        if (v >= C::NSV && !tc::mbar_wait(&vempty[vsi], ((v / C::NSV) - 1) & 1, abort_flag, wlim))
                            ok = false;
                        else
                            tc::mbar_arrive_expect_tx(&vfull[vsi], (pv0_ >= 0 ? C::V_PAGE + C::VS_PAGE : 0) +
                                                                       (pv1_ >= 0 ? C::V_PAGE + C::VS_PAGE : 0));
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    uint8_t* stg = smem + C::SM_VST + vsi * C::VSTAGE;
                    if (lane < 4) {
                        const int p = lane & 1, pg = p ? pv1_ : pv0_;
                        if (pg >= 0) {
                            const int64_t ph = (int64_t)pg * a.H_kv + hk;
                            if (lane < 2)
                                tc::bulk_g2s(stg + C::OFF_V + p * C::V_PAGE, a.v_pages + ph * C::V_PAGE, C::V_PAGE,
                                             &vfull[vsi]);
                            else
                                tc::bulk_g2s(stg + C::OFF_VS + p * C::VS_PAGE, a.v_scales + ph * C::VS_PAGE,
                                             C::VS_PAGE, &vfull[vsi]);
                        }
                    }
                    v_last = v;
                }
                pv0 = pg0;
                pv1 = pg1;
            }
        }
        if (!ok && lane == 0) *abort_flag = 1;
        // Unwinding: before the CTA can exit, every copy this warp started must have landed.
        // Each stage's last announced phase completes once its bytes (and the lanes' cp.async
        // arrivals) are in; announced tiles run consecutively from the first one announced.
        if (!ok || stall || *abort_flag) {
            if (lane == 0) {
                const int k_first = stall ? 1 : 0;
                for (int s = 0; s < C::NSK; ++s) {
                    if (k_last < s) continue;
                    const int t = k_last - (k_last - s) % C::NSK;
                    if (t >= k_first) tc::mbar_wait_drain(&kfull[s], (t / C::NSK) & 1, wlim);
                }
                for (int s = 0; s < C::NSV; ++s) {
                    if (v_last < s) continue;
                    const int t = v_last - (v_last - s) % C::NSV;
                    tc::mbar_wait_drain(&vfull[s], (t / C::NSV) & 1, wlim);
                }
            }
            __syncwarp();
        }
    } else if (warp == C::MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // Lane 0 issues every tcgen05 operation.  NVFP4: the other lanes leave (a lane that
        // spins alone while the rest of its warp waits for it costs issue slots).  MXFP4: all
        // lanes run every wait themselves, converged, because they also build each tile's V
        // scale-factor source: per channel group, the 2 bytes of page 0 and of page 1 side by
        // side, so one tcgen05.cp serves both pages' MMAs (scale-factor ids 0 and 2).
        if (MX || lane == 0) {
            const bool leader = lane == 0;
            // a decision every lane inside takes alike
            auto all = [&](bool v) -> bool {
                if constexpr (MX) return __all_sync(0xffffffffu, v);
                else return v;
            };
            auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
                return all(tc::mbar_wait(bar, parity, abort_flag, wlim));
            };
            constexpr uint32_t idesc_qk = tc::idesc_fp4(C::NQ, MX);
            constexpr uint32_t idesc_pv = tc::idesc_fp4(C::NP, MX);
            const uint32_t q_addr = tc::smem_u32(q_op);
            const uint32_t p_addr = tc::smem_u32(p_op);
            const uint32_t kst_addr = tc::smem_u32(smem + C::SM_KST);
            const uint32_t vst_addr = tc::smem_u32(smem + C::SM_VST);
            const uint32_t psf_addr = tc::smem_u32(psf);
            const uint32_t vsf_addr = tc::smem_u32(smem + C::SM_VSF);
            // the last commit: its phase completes once every tcgen05 operation issued before it has
            uint64_t* last_bar = nullptr;
            uint32_t last_par = 0;
            auto issue_qk = [&](int j) -> bool {
                const int s = j % C::NSK, buf = j & 1;
                if (!wait(&kfull[s], (j / C::NSK) & 1)) return false;
                tc::tc_fence_after();
                if (leader) {
                    // the scale rows came through cp.async (generic proxy); tcgen05.cp reads them
                    // through the async proxy
                    tc::fence_proxy_async_smem();
                    const uint32_t kt = kst_addr + s * C::KSTAGE + C::OFF_K;
                    // K scale factors: each 512-byte group chunk is the 32 x 16-byte copy source
#pragma unroll
                    for (int kg = 0; kg < C::NKG; ++kg)
                        tc::tmem_cp_32x128b_x4(tbase + C::T_SFK + (buf * C::NKG + kg) * 4,
                                               tc::smem_desc(kt - C::OFF_K + C::OFF_KS + kg * 512, 128, 128));
#pragma unroll
                    for (int ks = 0; ks < C::KS; ++ks) {
                        // MXFP4 packs two K steps per scale column: byte offset 2 (sf id) for the odd step
                        const uint32_t sfid = (uint32_t)(ks % C::KPG) * 2u;
                        tc::mma_fp4<MX>(tbase + C::T_S + buf * C::NQ, tc::smem_desc(kt + ks * 256, 128, 512),
                                        tc::smem_desc(q_addr + ks * 256, 128, 512), idesc_qk | (sfid << 29),
                                        (tbase + C::T_SFK + (buf * C::NKG + ks / C::KPG) * 4) | (sfid << 30),
                                        tbase + C::T_SFQ + ks * 4, ks > 0);
                    }
                    tc::mma_commit(&s_full[buf]);
                    tc::mma_commit(&kempty[s]);   // the K stage is free once QK has read it
                    last_bar = &kempty[s];
                    last_par = (uint32_t)(j / C::NSK) & 1u;
                }
                if constexpr (MX) __syncwarp();
                return true;
            };
            // the softmax warps quantize the query into shared memory and TMEM first (MXFP4: the
            // lanes then read the page flags those warps wrote before)
            bool ok = wait(q_ready, 0);
            if (ok) tc::tc_fence_after();
            const bool any_bad_page = MX && ok && *reinterpret_cast<volatile int*>(smem + C::SM_PFLAG + 64) != 0;
            ok = ok && issue_qk(0);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n && !(ok = issue_qk(j + 1))) break;
                const int s = j % C::NSV, buf = j & 1;
                if (!(ok = wait(&p_ready[buf], (j >> 1) & 1))) break;
                if (!(ok = wait(&vfull[s], (j / C::NSV) & 1))) break;
                tc::tc_fence_after();
                if constexpr (MX) {
                    // row `lane` of the source: TMEM lane `lane`, column c <- channel 32 c + lane;
                    // blocks past the sequence end and blocks of pages the block table gets wrong
                    // are zeroed (their bytes are never multiplied)
                    const int tile = tile0 + j;
                    const uint8_t* vs = smem + C::SM_VST + s * C::VSTAGE + C::OFF_VS;
                    const uint2 w0 = *reinterpret_cast<const uint2*>(vs + 8 * lane);
                    const uint2 w1 = *reinterpret_cast<const uint2*>(vs + C::VS_PAGE + 8 * lane);
                    uint32_t msk[2];
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        int nvb = (N - (tile * kTileTokens + p * kPageSlots) + B - 1) / B;
                        nvb = nvb < 0 ? 0 : (nvb > C::SPB ? C::SPB : nvb);
                        if (any_bad_page) {
                            const int pi = tile * 2 + p;
                            if (j < 64) {
                                if (!((smem + C::SM_PFLAG)[j] & (1u << p))) nvb = 0;
                            } else if (pi * kPageSlots < N) {
                                const int v = __ldg(a.block_table + (int64_t)b * a.max_pages + pi);
                                if (v < 0 || v >= a.num_pages) nvb = 0;
                            }
                        }
                        const uint32_t m16 = nvb >= 2 ? 0xffffu : ((1u << (8 * nvb)) - 1u);
                        msk[p] = m16 | (m16 << 16);
                    }
                    const uint32_t x0 = w0.x & msk[0], x1 = w0.y & msk[0], y0 = w1.x & msk[1], y1 = w1.y & msk[1];
                    *reinterpret_cast<uint4*>(smem + C::SM_VSF + buf * 512 + 16 * lane) =
                        make_uint4(__byte_perm(x0, y0, 0x5410), __byte_perm(x0, y0, 0x7632),
                                   __byte_perm(x1, y1, 0x5410), __byte_perm(x1, y1, 0x7632));
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                }
                if (leader) {
                    const uint32_t vt = vst_addr + s * C::VSTAGE + C::OFF_V;
                    // scale factors of P (written by the softmax warps) and of V: NVFP4 a page's scale
                    // block is already in the 32 x 16-byte copy layout, MXFP4 the interleaved rows
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        tc::tmem_cp_32x128b_x4(tbase + C::T_SFP + (buf * 2 + p) * 4,
                                               tc::smem_desc(psf_addr + (buf * 2 + p) * 512, 128, 128));
                        if constexpr (!MX)
                            tc::tmem_cp_32x128b_x4(tbase + C::T_SFV + buf * 8 + p * 4,
                                                   tc::smem_desc(vt - C::OFF_V + C::OFF_VS + p * C::VS_PAGE, 128, 128));
                    }
                    if constexpr (MX)
                        tc::tmem_cp_32x128b_x4(tbase + C::T_SFV + buf * 4, tc::smem_desc(vsf_addr + buf * 512, 128, 128));
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        // O^T accumulates across the split's tiles (the softmax warps rescale it in
                        // place when a running maximum rises)
                        const uint32_t sfid = MX ? (uint32_t)p * 2u : 0u;
                        const uint32_t sfa = MX ? (tbase + C::T_SFV + buf * 4) | (sfid << 30)
                                                : tbase + C::T_SFV + buf * 8 + p * 4;
                        tc::mma_fp4<MX>(tbase + C::T_O, tc::smem_desc(vt + p * C::V_PAGE, 128, 256),
                                        tc::smem_desc(p_addr + buf * C::P_BUF + p * C::P_PAGE, 128, 256),
                                        idesc_pv | (sfid << 29), sfa, tbase + C::T_SFP + (buf * 2 + p) * 4,
                                        (j > 0 || p > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&o_full[buf]);
                    tc::mma_commit(&vempty[s]);
                    last_bar = &vempty[s];
                    last_par = (uint32_t)(j / C::NSV) & 1u;
                }
                if constexpr (MX) __syncwarp();
            }
            if (!ok && leader) {
                *abort_flag = 1;
                // unwinding: the tensor memory is freed below, so the MMAs and copies into it
                // must have finished
                if (last_bar) tc::mbar_wait_drain(last_bar, last_par, wlim);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        // the body is instantiated once per head group, so the group's offsets are constants
        auto softmax_role = [&](auto grp_c) {
            constexpr int grp = decltype(grp_c)::value;   // head group
            const int qd = warp & 3;                   // TMEM lane quadrant = tokens 32 qd .. 32 qd + 31
            constexpr int gb = grp * HG;               // first head of the group
            constexpr int bar_id = 1 + grp;            // named barrier of the group (128 threads)
            const uint32_t tq = tbase + ((uint32_t)(32 * qd) << 16);
            const float alpha = (FMT == BDFP4_NVFP4 && !(a.flags & BDFP4_FLAG_NO_UNDERFLOW)) ? kAlphaNV : 1.0f;
            bool bad = false;
            bool grp_abort = false;   // the group's four warps gave up (alike in all of them)

            // Pages the block table gets wrong (the producer reports them and copies nothing) are
            // skipped like tokens past the end: their logits are masked and their V scales zeroed.
            // Before the first tile the softmax threads note, per tile of the split, whether both
            // of its pages are good (bit 0: first page, bit 1: second) and whether any is not;
            // splits longer than 64 tiles look tiles 64 on up in the block table as they go.
            uint8_t* const pflag = smem + C::SM_PFLAG;
            volatile int* const pflag_bad = reinterpret_cast<volatile int*>(smem + C::SM_PFLAG + 64);
            auto page_flags = [&](int jt) -> uint32_t {
                uint32_t r = 3u;
    #pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const int pi = (tile0 + jt) * 2 + p;
                    if (pi * kPageSlots < N) {   // pages past the end are masked anyway
                        const int v = __ldg(a.block_table + (int64_t)b * a.max_pages + pi);
                        if (v < 0 || v >= a.num_pages) r &= ~(1u << p);
                    }
                }
                return r;
        };
            if (tid == 0) *pflag_bad = n > 64 ? 1 : 0;
            tc::named_bar_sync(1 + C::NSG, 32 * C::NSW);
            if (tid < 64 && tid < n) {
                const uint32_t f = page_flags(tid);
                pflag[tid] = (uint8_t)f;
                if (f != 3u) *pflag_bad = 1;
            }
            // the query image (QK operand, scale codes, logit scales) of this (sequence, KV head)
            // arrives in one bulk copy from prep_query_kernel, which this grid may overlap:
            // griddepcontrol.wait holds the copy until that grid's writes are visible
            if (tid == 0) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                tc::mbar_arrive_expect_tx(q_full, C::QPACK);
                tc::bulk_g2s(q_op, a.qpack + ((int64_t)b * a.H_kv + hk) * C::QPACK, C::QPACK, q_full);
            }
            // the P scale-factor buffers: zero (rows of absent heads must stay zero)
            for (int i = tid; i < 2 * 2 * 512 / 16; i += 32 * C::NSW) reinterpret_cast<uint4*>(psf)[i] = make_uint4(0, 0, 0, 0);
            if (!tc::mbar_wait(q_full, 0, abort_flag, wlim)) bad = true;
            // query scale factors (SFB of QK): lane n <- row n, one 4-column chunk per K step
            if (grp == 0) {
    #pragma unroll
                for (int ks = 0; ks < C::KS; ++ks) {
                    uint32_t v = 0;
                    if (lane < C::NQ) {
                        if constexpr (B == 16) v = *reinterpret_cast<const uint32_t*>(qsc + lane * 8 + ks * 4);
                        else v = (uint32_t)qsc[lane * 8 + ks * 2] | ((uint32_t)qsc[lane * 8 + ks * 2 + 1] << 8);
                    }
                    tc::tmem_st4(tq + C::T_SFQ + ks * 4, v, 0u, 0u, 0u);
                }
                tc::tmem_wait_st();
            }
            tc::tc_fence_before();
            tc::fence_proxy_async_smem();
            tc::named_bar_sync(1 + C::NSG, 32 * C::NSW);   // psf zeroed and page flags set before any tile
            const bool any_bad_page = *pflag_bad != 0;
            if (lane == 0) tc::mbar_arrive(q_ready);
            // The running maximum of head gb + hl lives in the lanes hl, hl + HG, ... of each of the
            // group's warps (hl = lane % HG); they compute the head's per-tile terms once, and the
            // warp's lanes take them by shuffle.  DYN: e_l is log2 of the head's current pre-scale
            // (O^T and l are held in its units).
            const int hl = lane % HG;
            float m_l = -INFINITY;
            int e_l = 11;
            float l_part[HG];
    #pragma unroll
            for (int g = 0; g < HG; ++g) l_part[g] = 0.0f;
            // TMEM lane 32 qd + lane holds token 32 qd + lane of the tile: slot 32 (qd % 2) + lane
            // of page qd / 2, so a warp owns 32 consecutive slots of one page
            const int page_of_thread = qd >> 1;
            const int pos_in_page = 32 * (qd & 1) + lane;
            const int tok_in_tile = 32 * qd + lane;
            const int chan = 32 * qd + lane;   // O^T lane = value channel

            // log2 of alpha: alpha * 2^(x - m) is evaluated as 2^(x - (m - log2 alpha))
            const float la = alpha == kAlphaNV ? 11.0f : 0.0f;
            float lsr[HG];
    #pragma unroll
            for (int g = 0; g < HG; ++g) lsr[g] = lsc[gb + g];
            const bool lo_half = lane < 16;
            // P operand bytes: a lane pair (tokens 2i, 2i + 1 of a half warp) fills one byte of
            // each head row; with two heads per pair step the even lane writes head g, the odd
            // lane head g + 1.  Token pos of page p is K index pos: 16-byte chunk pos/32, byte (pos%32)/2
            const int hsel = HG >= 2 ? (lane & 1) : 0;
            const bool pstore = HG >= 2 || (lane & 1) == 0;
            // the lanes that write a block's scale byte: the first (two) of the half warp
            // (NVFP4, 16-token blocks) or of the warp (MXFP4, 32-token blocks)
            const bool sfstore = (lane & (B - 1)) < (HG >= 2 ? 2 : 1);
            const uint32_t psel = (lane & 1) ? 0x0004u : 0x0040u;   // byte 0 <- token 2i, byte 1 <- token 2i + 1
            uint8_t* const pbyte = p_op + page_of_thread * C::P_PAGE + (qd & 1) * 128 + (lane >> 1) + hsel * 16;
            uint8_t* const sfbyte = psf + page_of_thread * 512 + pos_in_page / B + hsel * 16;

            // The tile loop, in two copies: the page checks exist only in the copy a split with a
            // bad page runs, so the normal copy carries no extra live registers.
            auto tiles = [&](auto masked) {
                for (int j = 0; j < n; ++j) {
                    const int buf = j & 1, tile = tile0 + j;
                    bool pok0 = true, pok1 = true;
                    if constexpr (decltype(masked)::value) {
                        const uint32_t f = j < 64 ? pflag[j] : page_flags(j);
                        pok0 = (f & 1u) != 0;
                        pok1 = (f & 2u) != 0;
                    }
                    // logits of this thread's token for the group's heads (q1 then q2 columns)
                    if (!tc::mbar_wait(&s_full[buf], (j >> 1) & 1, abort_flag, wlim)) bad = true;
                    tc::tc_fence_after();
                    uint32_t sr[2 * HG];
                    tc::tmem_ld<2 * HG>(tq + C::T_S + buf * C::NQ + 2 * gb, sr);
                    tc::tmem_wait_ld();
                    const int token = tile * kTileTokens + tok_in_tile;
                    const bool valid = token < N && (page_of_thread ? pok1 : pok0);
                    // MT: the token is visible to query token i iff token <= N - T_q + i, i.e. to the
                    // stacked rows v = i G + g >= (token - (N - T_q)) G: rows g >= vis of this group
                    int vis = 0;
                    if constexpr (MT) vis = (token - (N - a.T_q)) * (a.H_q / a.H_kv) - gb;
                    // raw logits q1.k + q2.k (the positive factor lsc is applied later, so maxima
                    // commute with it) and their maxima over each half warp (16 consecutive slots)
                    float t[HG], hm_lo[HG], hm_hi[HG];
        #pragma unroll
                    for (int g = 0; g < HG; ++g) {
                        t[g] = (valid && (!MT || g >= vis)) ? __uint_as_float(sr[g]) + __uint_as_float(sr[HG + g]) : -INFINITY;
                        hm_lo[g] = tc::redux_max_f32(lo_half ? t[g] : -INFINITY, 0xffffffffu);
                        hm_hi[g] = tc::redux_max_f32(lo_half ? -INFINITY : t[g], 0xffffffffu);
                    }
                    float* rw = red + buf * C::RED_BUF;
                    if (lane == 0) {
        #pragma unroll
                        for (int g = 0; g < HG; ++g) {
                            rw[(gb + g) * 4 + qd] = fmaxf(hm_lo[g], hm_hi[g]);
                        }
                    }
                    // one decision for the group's four warps, taken by the barrier itself (a role
                    // that gave up leaves a wait here unfinished, and the wait sees its abort flag)
                    if (tc::named_bar_or(bar_id, 128, bad)) {
                        grp_abort = true;
                        break;
                    }
                    float y[HG], corr[HG];
                    [[maybe_unused]] float am[HG];   // block maxima of alpha p (NVFP4 up to two heads per group), MXFP4 elements
                    [[maybe_unused]] uint32_t mxc[HG];   // MXFP4 block scale codes
                    float corr_l, base_l, mz_l;
                    [[maybe_unused]] float eb_l = 0.0f;   // MXFP4: head hl's element exponent base m + (c - 127)
                    [[maybe_unused]] int c_l = 0;         // MXFP4: head hl's block scale code (the block is the warp)
                    // NVFP4, four or more heads per group: the block scale of head hl over half warp
                    // (lane / HG) % 2, its code and reciprocal (a 16-token block is a half warp)
                    constexpr bool NV_LANE = !MX && HG >= 4;
                    [[maybe_unused]] float rinv_l = 0.0f;
                    [[maybe_unused]] uint32_t code_l = 0u;
                    bool rose_l;
                    {
                        const float4 w4 = *reinterpret_cast<const float4*>(rw + (gb + hl) * 4);
                        const float mt = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
                        const float ls = lsc[gb + hl];
                        const float mn = fmaxf(m_l, mt * ls);
                        mz_l = mn == -INFINITY ? 0.0f : mn;
                        corr_l = tc::ex2_approx(m_l - mz_l);   // 0 on the split's first tile
                        rose_l = mn != m_l;
                        m_l = mn;
                        base_l = mz_l - la;
                        if constexpr (DYN) {
                            // this tile's pre-scale from its largest probability; the accumulators
                            // move to its units (an exact power of two, folded into corr)
                            const int e = dynamic_alpha_exp(tc::ex2_approx(mt * ls - mz_l));
                            corr_l *= pow2f(e - e_l);
                            rose_l |= e != e_l;
                            e_l = e;
                            base_l = mz_l - (float)e;
                        }
                        if constexpr (MX) {
                            // the OCP MX shared exponent of head hl's 32-token block (this warp), in
                            // the log domain: the block maximum is 2^d with d = x_b - m, so floor(log2) =
                            // floor(d) exactly (d = 0 for the tile's largest logit), and the element is
                            // 2^(x - m - e) for the scale 2^e
                            float bm = fmaxf(hm_lo[0], hm_hi[0]);
        #pragma unroll
                            for (int g = 1; g < HG; ++g) bm = hl == g ? fmaxf(hm_lo[g], hm_hi[g]) : bm;
                            const float dd = __fsub_rn(__fmul_rn(bm, ls), mz_l);
                            c_l = max(__float2int_rd(fmaxf(dd, -256.0f)) + 125, 0);
                            eb_l = mz_l + (float)(c_l - 127);
                        }
                        if constexpr (NV_LANE) {
                            const bool hh = ((lane / HG) & 1) != 0;
                            float bm = hh ? hm_hi[0] : hm_lo[0];
        #pragma unroll
                            for (int g = 1; g < HG; ++g) bm = hl == g ? (hh ? hm_hi[g] : hm_lo[g]) : bm;
                            const float ab = tc::ex2_approx(fmaf(bm, ls, -base_l));
                            code_l = tc::e4m3x2_encode(__fmul_rn(ab, 1.0f / 6.0f), 0.0f) & 0xffu;
                            // a zero scale zeroes the whole block inside the MMA, whatever the element codes
                            rinv_l = tc::rcp_approx(tc::e4m3x2_value(code_l).x);
                        }
                    }
                    // a running maximum of the group rose (alike in its four warps)
                    const bool rose = __any_sync(0xffffffffu, rose_l);
        #pragma unroll
                    for (int g = 0; g < HG; ++g) {
                        corr[g] = __shfl_sync(0xffffffffu, corr_l, g);
                        const float base = __shfl_sync(0xffffffffu, base_l, g);
                        // the same two instructions give a token's scaled probability and its block's
                        // maximum, so the block scale is the one its largest member picks
                        y[g] = tc::ex2_approx(fmaf(t[g], lsr[g], -base));   // 0 for masked tokens
                        l_part[g] = fmaf(l_part[g], corr[g], y[g]);         // l in units of alpha (cancels at the end)
                        if constexpr (!MX) {
                            // a 16-token block is this half warp
                            if constexpr (!NV_LANE) {
                                const float bm = lo_half ? hm_lo[g] : hm_hi[g];
                                am[g] = tc::ex2_approx(fmaf(bm, lsr[g], -base));
                            }
                        } else {
                            // a 32-token block is this warp: its exponent from the head's lanes
                            mxc[g] = (uint32_t)__shfl_sync(0xffffffffu, c_l, g);
                            am[g] = tc::ex2_approx(fmaf(t[g], lsr[g], -__shfl_sync(0xffffffffu, eb_l, g)));
                        }
                    }
                    // fused FP4 quantization of the probabilities, two heads per conversion
                    uint8_t* const pb = pbyte + buf * C::P_BUF;
                    uint8_t* const sfb = sfbyte + buf * 2 * 512;
        #pragma unroll
                    for (int g = 0; g < HG; g += 2) {
                        const int g1 = HG >= 2 ? g + 1 : g;
                        uint32_t codes;
                        float q0, q1;
                        if constexpr (NV_LANE) {
                            // the block scales of this half warp, from the lanes of heads g and g1
                            const int ho = lo_half ? 0 : HG;
                            q0 = y[g] * __shfl_sync(0xffffffffu, rinv_l, g + ho);
                            q1 = y[g1] * __shfl_sync(0xffffffffu, rinv_l, g1 + ho);
                            codes = __shfl_sync(0xffffffffu, code_l, g + hsel + ho) << (8 * hsel);
                        } else if constexpr (FMT == BDFP4_NVFP4) {
                            codes = tc::e4m3x2_encode(__fmul_rn(am[g], 1.0f / 6.0f), __fmul_rn(am[g1], 1.0f / 6.0f));
                            const float2 sg = tc::e4m3x2_value(codes);
                            // a zero scale zeroes the whole block inside the MMA, whatever the element codes
                            q0 = y[g] * tc::rcp_approx(sg.x);
                            q1 = y[g1] * tc::rcp_approx(sg.y);
                        } else {
                            codes = mxc[g] | (mxc[g1] << 8);
                            q0 = am[g];    // the element already divided by its block scale
                            q1 = am[g1];
                        }
                        const uint32_t mine = e2m1x2_encode(q0, q1);   // head g in bits 0..3, head g1 in 4..7
                        const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
                        const uint32_t w = __byte_perm(mine, other, psel) >> (4 * hsel);
                        const int hr = gb + g;
                        if (pstore) pb[(hr >> 3) * 256 + (hr & 7) * 16] = (uint8_t)((w & 0xfu) | ((w >> 4) & 0xf0u));
                        if (sfstore) sfb[hr * 16] = (uint8_t)(codes >> (8 * hsel));   // SFB rows hr, hr + 1
                    }
                    // O^T rescale of the group's heads once the previous tile's PV has completed,
                    // before this tile's PV is issued (the online-softmax update, in TMEM)
                    if (j > 0 && rose) {
                        if (!tc::mbar_wait(&o_full[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, wlim)) bad = true;
                        tc::tc_fence_after();
                        uint32_t ov[HG];
                        tc::tmem_ld<HG>(tq + C::T_O + gb, ov);
                        tc::tmem_wait_ld();
    #pragma unroll
                        for (int g = 0; g < HG; ++g) ov[g] = __float_as_uint(__uint_as_float(ov[g]) * corr[g]);
                        tc::tmem_st_n<HG>(tq + C::T_O + gb, ov);
                        tc::tmem_wait_st();
                        tc::tc_fence_before();
                    }
                    // NVFP4 V scale factors (group 0): blocks past the sequence end are zeroed, so the
                    // bytes a page holds there are never multiplied.  The V stage can not be
                    // refilled before this tile's PV, so waiting for it here is safe.  (MXFP4: the
                    // MMA warp builds the tile's V scale rows and masks them.)
                    if constexpr (B == 16) {
                        if (grp == 0) {
                            const int s = j % C::NSV;
                            const bool tail = (tile + 1) * kTileTokens > N;
                            uint8_t* vs = smem + C::SM_VST + s * C::VSTAGE + C::OFF_VS;
                            if (tail || !pok0 || !pok1) {
                                if (!tc::mbar_wait(&vfull[s], (j / C::NSV) & 1, abort_flag, wlim)) bad = true;
        #pragma unroll
                                for (int p = 0; p < 2; ++p) {
                                    const int t0 = tile * kTileTokens + p * kPageSlots;
                                    int nvb = (N - t0 + B - 1) / B;
                                    nvb = nvb < 0 ? 0 : (nvb > C::SPB ? C::SPB : nvb);
                                    if (!(p ? pok1 : pok0)) nvb = 0;
                                    for (int bb = nvb; bb < C::SPB; ++bb)
                                        vs[p * C::VS_PAGE + (chan & 31) * 16 + (chan >> 5) * 4 + bb] = 0;
                                }
                            }
                        }
                    }
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&p_ready[buf]);
                }
            };
            if (any_bad_page) tiles(std::true_type{});
            else tiles(std::false_type{});
            // the split's O^T once its last PV has completed
            uint32_t o_fin[HG];
    #pragma unroll
            for (int g = 0; g < HG; ++g) o_fin[g] = 0u;
            if (!grp_abort) {
                if (!tc::mbar_wait(&o_full[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, wlim)) bad = true;
                tc::tc_fence_after();
                tc::tmem_ld<HG>(tq + C::T_O + gb, o_fin);
                tc::tmem_wait_ld();
            }

            // ------------------------------------------------------------ epilogue (thread = channel)
            grp_abort = tc::named_bar_or(bar_id, 128, grp_abort || bad || *abort_flag);
            if (grp_abort) *abort_flag = 1;
            if (!grp_abort) {
                float* rl = red;   // [G][8] partial sums (the tile maxima are no longer read)
    #pragma unroll
                for (int g = 0; g < HG; ++g) {
                    float v = l_part[g];
    #pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    if (lane == 0) rl[(gb + g) * 8 + qd] = v;
                }
                tc::named_bar_sync(bar_id, 128);
                // O and l both carry the factor alpha (P^ is alpha p quantized), so it cancels
                const float oscale = FMT == BDFP4_NVFP4 ? a.v_gscale[hk] : 1.0f;
                const int ch = chan;
    #pragma unroll
                for (int g = 0; g < HG; ++g) {
                    const int hh = gb + g;
                    const float l = rl[hh * 8] + rl[hh * 8 + 1] + rl[hh * 8 + 2] + rl[hh * 8 + 3];
                    const int64_t row = row_of(hh);
                    if (nspl == 1) {
                        a.out[row * C::DV + ch] =
                            __float2bfloat16(l > 0.0f ? __uint_as_float(o_fin[g]) * oscale / l : 0.0f);
                    } else {
                        // DYN: splits end in different units; the partials leave in the units of p
                        const float un = DYN ? pow2f(-__shfl_sync(0xffffffffu, e_l, g)) : 1.0f;
                        const float m_g = __shfl_sync(0xffffffffu, m_l, g);
                        a.ws_o[(row * a.max_splits + split) * C::DV + ch] = __uint_as_float(o_fin[g]) * oscale * un;
                        if (chan == 0) {
                            a.ws_ml[(row * a.max_splits + split) * 2 + 0] = m_g;
                            a.ws_ml[(row * a.max_splits + split) * 2 + 1] = l * un;
                        }
                    }
                }
            }
        };
        if (C::NSG == 1 || warp < 4) softmax_role(std::integral_constant<int, 0>{});
        else softmax_role(std::integral_constant<int, (C::NSG > 1 ? 1 : 0)>{});
    }

    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) set_status(a.dev_status, BDFP4_DEV_TIMEOUT);
    if (warp == C::MMA_WARP) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tbase, C::T_ALLOC);
    }
}

template <int FMT, int G, bool DYN = false, bool MT = false, bool HOOK = false>
static int launch_tc(const DecodeArgs& a, cudaStream_t st, const StepArgs* step) {
    using C = TcCfg<FMT, G>;
    static bool attr_set = false;
    if (!attr_set) {
        const cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<FMT, G, DYN, MT, HOOK>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_LAUNCH);
        if (e != cudaSuccess) {
            record_cuda_error(e);
            return BDFP4_ERR_CUDA;
        }
        attr_set = true;
    }
    if constexpr (!MT) {
        if (step) {
            const int64_t rows = (int64_t)a.B * a.H_kv;
            const int64_t ctas = k_append_ctas_wide<FMT, 128>(rows) + v_append_ctas<128>(rows) + rows;
            prep_step_kernel<FMT, G><<<(unsigned)ctas, 256, 0, st>>>(a, *step);
        } else {
            prep_query_kernel<FMT, G><<<dim3(a.H_kv, a.B), C::QTHREADS, 0, st>>>(a);
        }
    } else {
        if (step) return BDFP4_ERR_UNSUPPORTED;   // a step appends one token per sequence
        prep_query_kernel<FMT, G, true><<<dim3(a.H_kv, a.B), C::QTHREADS, 0, st>>>(a);
    }
    const int rc = launch_status();
    if (rc != BDFP4_OK) return rc;
    // programmatic dependent launch: the decode CTAs start (TMEM, barriers, K/V
    // streaming) while the query images are computed
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.max_splits, a.H_kv, a.B);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_LAUNCH;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<FMT, G, DYN, MT, HOOK>, a);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return BDFP4_ERR_CUDA;
    }
    return launch_status();
}

template <bool MT>
static int dispatch_tc(const DecodeArgs& a, int fmt, int G, cudaStream_t st, const StepArgs* step) {
    if (fmt == BDFP4_NVFP4 && (a.flags & BDFP4_FLAG_DYNAMIC_ALPHA)) {
        switch (G) {
            case 1: if constexpr (!MT) return launch_tc<BDFP4_NVFP4, 1, true, false>(a, st, step); break;
            case 2: return launch_tc<BDFP4_NVFP4, 2, true, MT>(a, st, step);
            case 4: return launch_tc<BDFP4_NVFP4, 4, true, MT>(a, st, step);
            case 8: return launch_tc<BDFP4_NVFP4, 8, true, MT>(a, st, step);
            case 16: return launch_tc<BDFP4_NVFP4, 16, true, MT>(a, st, step);
        }
    } else if (fmt == BDFP4_NVFP4) {
        switch (G) {
            case 1: if constexpr (!MT) return launch_tc<BDFP4_NVFP4, 1, false, false>(a, st, step); break;
            case 2: return launch_tc<BDFP4_NVFP4, 2, false, MT>(a, st, step);
            case 4: return launch_tc<BDFP4_NVFP4, 4, false, MT>(a, st, step);
            case 8: return launch_tc<BDFP4_NVFP4, 8, false, MT>(a, st, step);
            case 16: return launch_tc<BDFP4_NVFP4, 16, false, MT>(a, st, step);
        }
    } else {
        switch (G) {
            case 1: if constexpr (!MT) return launch_tc<BDFP4_MXFP4, 1, false, false>(a, st, step); break;
            case 2: return launch_tc<BDFP4_MXFP4, 2, false, MT>(a, st, step);
            case 4: return launch_tc<BDFP4_MXFP4, 4, false, MT>(a, st, step);
            case 8: return launch_tc<BDFP4_MXFP4, 8, false, MT>(a, st, step);
            case 16: return launch_tc<BDFP4_MXFP4, 16, false, MT>(a, st, step);
        }
    }
    return BDFP4_ERR_UNSUPPORTED;
}

// G = rows stacked per (sequence, KV head): the query heads of the group, times
// the query tokens per sequence when a.T_q > 1 (which then takes the MT kernels)
int launch_decode_tc(const DecodeArgs& a, int fmt, int G, cudaStream_t st, const StepArgs* step) {
    if (a.test_stall || a.wait_limit != kWaitLimitDefault) {
        // the unwind test's instantiation: eight heads per KV head, one query token, no step
        if (G != 8 || a.T_q != 1 || step || (a.flags & BDFP4_FLAG_DYNAMIC_ALPHA)) return BDFP4_ERR_UNSUPPORTED;
        return fmt == BDFP4_NVFP4 ? launch_tc<BDFP4_NVFP4, 8, false, false, true>(a, st, step)
                                  : launch_tc<BDFP4_MXFP4, 8, false, false, true>(a, st, step);
    }
    return a.T_q > 1 ? dispatch_tc<true>(a, fmt, G, st, step) : dispatch_tc<false>(a, fmt, G, st, step);
}

}  // namespace bdfp4
