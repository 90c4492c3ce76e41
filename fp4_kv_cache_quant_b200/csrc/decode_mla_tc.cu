// decode_mla_tc.cu -- FP4 paged decode attention on the sm_100a tensor cores for
// latent-KV (MLA) shapes: d_k = 576 (512-d latent + 64-d rope), d_v = 512 (the
// latent), many query heads over one KV head (BitDecoding-FP4, Article Summary:
// stacked query MMA on paged KV caches, fused probability quantization,
// dual-residual query, underflow-aware probability scaling; the method is
// evaluated on GQA and MLA models).
//
// One CTA per (sequence, KV head, slice of GH <= 64 query heads, split), one
// CTA per SM.  The query operand stacks the slice's dual-residual halves as
// rows: row 2h holds q1 and row 2h + 1 holds q2 of head h.  TMEM (512 columns)
// holds
//   S [128 rows][128 tokens]           one QK MMA chain per tile (M = 128, N = 128),
//   O^T [512 channels = 4 x 128 lanes][GH heads], accumulated across the tiles,
//   and the scale factors of every MMA operand.
// A softmax lane owns one stacked row: its lane pair (q1, q2 of one head) adds
// the two halves over 16 tokens each, so a 16-token probability block (the
// NVFP4 block) is one lane's, and the 32-token MXFP4 block one lane pair's.
// O stays in TMEM: when a head's running maximum rises, every softmax warp
// rescales the head's O^T columns in its own lane quadrant and M tile, after
// the previous tile's PV completed and before this tile's PV is issued -- the
// online-softmax update, in place.
//   warps 0 .. 15   softmax: warp w reads S lane quadrant w % 4 (heads
//                   16 (w % 4) .. +15, when the slice has them) over tokens
//                   32 (w / 4) .. +31 of each tile, and rescales and writes out
//                   O^T M tile w / 4 of that lane quadrant
//   warp  16        producer: K and V pages by bulk copy, K scales by cp.async
//   warp  17        MMA issuer (one lane) and TMEM owner
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

constexpr long long kWaitLimitMla = 1LL << 32;   // clock cycles (about 2 s)

template <int FMT, int GH>
struct MlaCfg {
    static constexpr bool MX = FMT == BDFP4_MXFP4;
    static constexpr int B = Fmt<FMT>::beta;
    static constexpr int DK = 576, DV = 512;
    static constexpr int KS = DK / 64;                 // MMA K steps of QK
    static constexpr int NBLK = DK / B;                // scale blocks of a key or query row
    static constexpr int NKG = (NBLK + 3) / 4;         // 4-block key scale groups per token
    static constexpr int KPG = MX ? 2 : 1;             // K steps per key scale group
    static constexpr int MT = DV / 128;                // 128-channel M tiles of O^T
    static constexpr int ROWS = 2 * GH;                // stacked query rows (q1, q2 of each head)
    static constexpr int NQ = GH / 16;                 // S lane quadrants holding rows
    static constexpr int NSW = 16;                     // softmax warps
    static constexpr int PRODUCER = NSW, MMA_WARP = NSW + 1;
    static constexpr int THREADS = 32 * (NSW + 2);
    static constexpr int NSK = 2, NSV = 2;             // K and V ring stages
    static constexpr int K_PAGE = kPageSlots * DK / 2;
    static constexpr int KS_PAGE = 256 * NKG;
    static constexpr int V_PAGE = DV * kPageSlots / 2;
    static constexpr int VS_PAGE = DV * kPageSlots / B;
    static constexpr int VS_TILE = VS_PAGE / MT;       // V scale bytes of one M tile of a page
    static constexpr int SPB = kPageSlots / B;         // token blocks per page
    static constexpr int SBO = DK / 32 * 128;          // 8-row group stride of the K and query operands
    // K stage: the two pages (MMA rows 0-63, 64-127), then per scale group the
    // 32 x 16-byte tcgen05.cp source (row i: tokens i, 32 + i, 64 + i, 96 + i)
    static constexpr int OFF_KS = 2 * K_PAGE;
    static constexpr int KSTAGE = OFF_KS + NKG * 512;
    // V stage: the two pages, then their scale blocks
    static constexpr int OFF_VS = 2 * V_PAGE;
    static constexpr int VSTAGE = OFF_VS + 2 * VS_PAGE;
    // query image: the stacked operand [ROWS][DK] in K-major core blocks, its scale codes
    // [ROWS][NBLK], the logit scales [GH] (fp32).  Shared memory holds the operand at its
    // full 128 rows (rows past ROWS zero) and the codes and logit scales apart.
    static constexpr int Q_OP = 128 * DK / 2;
    static constexpr int QOP_IMG = ROWS * DK / 2;
    static constexpr int QSC = ROWS * NBLK;
    static constexpr int QMETA = QSC + GH * 4;
    static constexpr int QPACK = QOP_IMG + QMETA;
    static constexpr int P_PAGE = GH / 8 * 256;        // P^T operand of one page: GH rows x 64 tokens
    static constexpr int P_BUF = 2 * P_PAGE;
    // shared memory map
    static constexpr int SM_KST = 0;
    static constexpr int SM_VST = SM_KST + NSK * KSTAGE;
    static constexpr int SM_Q = SM_VST + NSV * VSTAGE;
    static constexpr int SM_QM = SM_Q + Q_OP;
    static constexpr int SM_P = (SM_QM + QMETA + 127) / 128 * 128;
    static constexpr int SM_PSF = SM_P + 2 * P_BUF;       // [2 buf][2 page][32 rows][16 B] P scales
    static constexpr int SM_RED = SM_PSF + 2 * 2 * 512;              // [2][GH][4 quarters] tile maxima
    static constexpr int SM_LRED = SM_RED + 2 * GH * 4 * 4;          // [GH][4 quarters] l partials
    static constexpr int SM_COR = SM_LRED + GH * 4 * 4;              // [2][GH] corrections
    static constexpr int SM_RISE = SM_COR + 2 * GH * 4;              // [2][4 quadrants] risen-head masks
    static constexpr int SM_HEAD = SM_RISE + 2 * 4 * 4;              // [GH] output scales
    static constexpr int SM_BARS = SM_HEAD + GH * 4;
    static constexpr int NBARS = 2 * NSK + 2 * NSV + 10;
    static constexpr int SM_MISC = SM_BARS + NBARS * 8;   // tmem slot, abort flags
    static constexpr int SM_PFLAG = SM_MISC + 32;   // [64] page flags of the split's tiles, any-bad
    static constexpr int SMEM = SM_PFLAG + 64 + 16;
    // TMEM column map
    static constexpr int T_S = 0;                      // 128 columns (tokens)
    static constexpr int T_O = 128;                    // M tile t at T_O + t GH
    static constexpr int T_SFK = (T_O + MT * GH + 3) / 4 * 4;   // NKG groups x 4
    static constexpr int T_SFQ = T_SFK + NKG * 4;               // KS steps x 4
    static constexpr int T_SFV = T_SFQ + KS * 4;                // NVFP4: MT tiles x 2 pages x 4; MXFP4: MT x 4
    static constexpr int T_SFP = T_SFV + MT * (MX ? 4 : 8);     // 2 buffers x 2 pages x 4
    static constexpr int T_USED = T_SFP + 16;
    static constexpr int T_ALLOC = 512;
    static_assert(GH % 16 == 0 && GH <= 64, "head slice");
    static_assert(T_USED <= T_ALLOC, "TMEM budget");
    static_assert(SMEM <= 232448 && SMEM > 232448 / 2, "one CTA per SM");
    static_assert(QOP_IMG % 16 == 0 && QMETA % 16 == 0, "query image copied in 16-byte units");
    // the image of a head slice fits the workspace region reserved for its heads
    static_assert(QPACK <= kQueryImageBytes * GH, "query image larger than its workspace share");
};

// ---------------------------------------------------------------- query image
// Row r of the CTA's query image (query head h0 + r): transform, dual-residual
// FP4, written straight into the image's operand, code and logit-scale slots.
// 256 threads handle 256 / rt rows of one image.
template <int FMT, int GH>
__device__ __forceinline__ void mla_query_rows(const DecodeArgs& a, int img, int h_first, int r_first) {
    using C = MlaCfg<FMT, GH>;
    using RG = RowGeom<FMT, 576>;
    constexpr int B = C::B;
    constexpr int RPC = 256 / RG::rt;   // rows per CTA
    __shared__ int row_amax[RPC];
    const int tid = threadIdx.x, j = tid % RG::rt, rl = tid / RG::rt;
    const int r = r_first + rl;
    const int G = a.H_q / a.H_kv;
    const int hq = h_first + rl;   // query head of this row (global index within the sequence)
    const int b = img / (a.H_kv * (G / GH));
    const bool active = rl < RPC && r < GH && j < RG::tpr;
    if (tid < RPC) row_amax[tid] = 0;
    __syncthreads();
    float x[B];
    if (active) {
        load_bf16_block<B>(a.q + ((int64_t)b * a.H_q + hq) * C::DK, j * B, x);
    } else {
#pragma unroll
        for (int i = 0; i < B; ++i) x[i] = 0.0f;
    }
    const int hk = hq / G;
    transform_block<FMT, 576, false>(x, a.smooth + (int64_t)(active ? hk : 0) * C::DK, j,
                                     !(a.flags & BDFP4_FLAG_NO_HADAMARD));
    if (active) atomicMax(&row_amax[rl], __float_as_int(block_amax<B>(x)));
    __syncthreads();
    if (!active) return;
    const float amax = __int_as_float(row_amax[rl]);
    const float gq = FMT == BDFP4_NVFP4 ? (amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f) : 1.0f;
    uint32_t c1, c2, p1[B / 8], p2[B / 8];
    quantize_query_block<FMT, 576>(x, gq, !(a.flags & BDFP4_FLAG_SINGLE_QUERY), c1, p1, c2, p2);
    uint8_t* im = a.qpack + (int64_t)img * C::QPACK;
    const int e0 = j * B;
#pragma unroll
    for (int o = 0; o < 2; ++o) {
        const uint32_t* pk = o ? p2 : p1;
        const int sr = 2 * r + o;   // stacked row: q1 of head r at 2r, q2 at 2r + 1
        uint8_t* dst = im + (sr >> 3) * C::SBO + (e0 >> 5) * 128 + (sr & 7) * 16 + (e0 & 31) / 2;
        if constexpr (B == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        im[C::QOP_IMG + sr * C::NBLK + j] = (uint8_t)(o ? c2 : c1);
    }
    if (j == 0) {
        const float gk = FMT == BDFP4_NVFP4 ? a.k_gscale[hk] : 1.0f;
        reinterpret_cast<float*>(im + C::QOP_IMG + C::QSC)[r] = a.sm_scale * gq * gk * kLog2e;
    }
}

// Prologue grid of the MLA decode: optionally the decode-step append (key CTAs,
// then value CTAs), then the query images, 256 / rt rows per CTA.
template <int FMT, int GH>
__global__ void __launch_bounds__(256) prep_mla_kernel(const DecodeArgs a, const StepArgs s, int with_step) {
    // the decode grid may start now; it waits for this grid before reading what it writes
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    using RG = RowGeom<FMT, 576>;
    constexpr int RPC = 256 / RG::rt;
    int blk = blockIdx.x;
    if (with_step) {
        const int64_t rows = (int64_t)a.B * a.H_kv;
        const NewestSlot slot{a.block_table, a.seq_lens, a.max_pages, a.num_pages, a.dev_status};
        const int nk = (int)k_append_ctas_wide<FMT, 576>(rows), nv = (int)v_append_ctas<512>(rows);
        if (blk < nk) {
            append_k_cta_wide<FMT, 576>(blk, s.k_new, rows, a.H_kv, slot, a.smooth, a.k_gscale, a.k_weight, s.k_pages, s.k_scales,
                                   a.flags);
            return;
        }
        if (blk < nk + nv) {
            append_v_open_cta<FMT, 512>(blk - nk, s.v_new, s.v_open, slot, a.B, a.H_kv, a.v_gscale, s.v_pages,
                                        s.v_scales);
            return;
        }
        blk -= nk + nv;
    }
    // query rows: image (sequence, KV head, slice) = blk / per_img, rows RPC at a time
    constexpr int per_img = (GH + RPC - 1) / RPC;
    const int img = blk / per_img, r0 = (blk % per_img) * RPC;
    const int G = a.H_q / a.H_kv;
    const int nh = G / GH;
    const int slice = img % (a.H_kv * nh);
    const int hk = slice / nh, hs = slice % nh;
    mla_query_rows<FMT, GH>(a, img, hk * G + hs * GH + r0, r0);
}


// ---------------------------------------------------------------- decode
// DYN (NVFP4): the probability pre-scale alpha = 2^E per tile and head; a head's
// O^T and l are held in units of its current tile's alpha, so a change of E joins
// the running-maximum correction as the exact factor 2^(E - E_prev).
template <int FMT, int GH, bool DYN = false>
__global__ void __launch_bounds__(MlaCfg<FMT, GH>::THREADS, 1) decode_mla_tc_kernel(const DecodeArgs a) {
    using C = MlaCfg<FMT, GH>;
    // the split merge (a programmatic dependent) may be scheduled as CTAs of this grid retire
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr bool MX = C::MX;
    constexpr int B = C::B, MT = C::MT;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* q_op = smem + C::SM_Q;
    const uint8_t* qsc = smem + C::SM_QM;
    const float* lsc = reinterpret_cast<const float*>(smem + C::SM_QM + C::QSC);
    uint8_t* p_op = smem + C::SM_P;
    uint8_t* psf = smem + C::SM_PSF;
    float* red = reinterpret_cast<float*>(smem + C::SM_RED);
    float* lred = reinterpret_cast<float*>(smem + C::SM_LRED);
    float* cor = reinterpret_cast<float*>(smem + C::SM_COR);
    uint32_t* rise = reinterpret_cast<uint32_t*>(smem + C::SM_RISE);
    float* hscale = reinterpret_cast<float*>(smem + C::SM_HEAD);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SM_BARS);
    uint64_t* kfull = bars;                   // [NSK] K tile landed -> MMA
    uint64_t* kempty = kfull + C::NSK;        // [NSK] QK done -> producer
    uint64_t* vfull = kempty + C::NSK;        // [NSV] V tile landed -> MMA, softmax
    uint64_t* vempty = vfull + C::NSV;        // [NSV] PV done -> producer
    uint64_t* s_full = vempty + C::NSV;       // QK done -> softmax
    uint64_t* s_free = s_full + 1;            // S read, the next tile's key scale factors stored -> MMA
    uint64_t* p_ready = s_free + 1;           // [2] P, its scales, V scales and O rescaled -> MMA
    uint64_t* o_done = p_ready + 2;           // [2] PV done -> softmax (rescale, epilogue), MMA
    uint64_t* q_ready = o_done + 2;           // query operand and its scale factors -> MMA
    uint64_t* q_full = q_ready + 1;           // query image landed -> softmax
    uint64_t* c_ready = q_full + 1;           // [2] the tile's corrections and risen heads posted -> softmax
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SM_MISC + 4);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, slice = blockIdx.y, b = blockIdx.z;
    const int G = a.H_q / a.H_kv, nh = G / GH;
    const int hk = slice / nh, hs = slice % nh;
    const int h0 = hk * G + hs * GH;   // first query head of the CTA
    const int img = b * a.H_kv * nh + slice;

    int N = a.seq_lens[b];
    if (N < 0 || N > a.max_pages * kPageSlots) {
        if (tid == 0 && split == 0 && slice == 0) set_status(a.dev_status, BDFP4_DEV_BAD_SEQLEN);
        N = 0;
    }
    const int ntiles = (N + kTileTokens - 1) / kTileTokens;
    const int nspl = (ntiles + a.chunk_tiles - 1) / a.chunk_tiles;
    if (split > 0 && split >= nspl) return;
    if (N == 0) {
        for (int i = tid; i < GH * C::DV; i += blockDim.x)
            a.out[((int64_t)b * a.H_q + h0 + i / C::DV) * C::DV + i % C::DV] = __float2bfloat16(0.0f);
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
        tc::mbar_init(s_full, 1);
        tc::mbar_init(s_free, 3 * C::NQ + 4);   // row-owning warps, and second-quarter warps without rows
        tc::mbar_init(&p_ready[0], C::NSW);
        tc::mbar_init(&p_ready[1], C::NSW);
        tc::mbar_init(&o_done[0], 1);
        tc::mbar_init(&o_done[1], 1);
        tc::mbar_init(q_ready, C::NSW);
        tc::mbar_init(q_full, 1);
        tc::mbar_init(&c_ready[0], C::NQ);
        tc::mbar_init(&c_ready[1], C::NQ);
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
        // Step k issues the K half of tile k and the V half of tile k - 1 (the
        // block-table reads of 32 tiles at a time, one per lane, as in the d = 128 kernel)
        bool ok = true;
        int pv0 = -1, pv1 = -1;
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
                const bool do_k = k < n, do_v = k >= 1;
                const int ks = k % C::NSK, v = k - 1, vsi = (k + C::NSV - 1) % C::NSV;
                if (do_k) {
                    // a decode-step prologue writes the new token into the sequence's last page
                    if (a.append_wait && tile0 + k == ntiles - 1) asm volatile("griddepcontrol.wait;" ::: "memory");
                    if (lane == 0) {
                        if (k >= C::NSK && !tc::mbar_wait(&kempty[ks], ((k / C::NSK) - 1) & 1, abort_flag, kWaitLimitMla))
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
                            tc::bulk_g2s(stg + lane * C::K_PAGE, a.k_pages + ((int64_t)pg * a.H_kv + hk) * C::K_PAGE,
                                         C::K_PAGE, &kfull[ks]);
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
                if (do_v) {
                    if (lane == 0) {
                        if (v >= C::NSV && !tc::mbar_wait(&vempty[vsi], ((v / C::NSV) - 1) & 1, abort_flag, kWaitLimitMla))
                            ok = false;
                        else
                            tc::mbar_arrive_expect_tx(&vfull[vsi], (pv0 >= 0 ? C::V_PAGE + C::VS_PAGE : 0) +
                                                                       (pv1 >= 0 ? C::V_PAGE + C::VS_PAGE : 0));
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    uint8_t* stg = smem + C::SM_VST + vsi * C::VSTAGE;
                    if (lane < 4) {
                        const int p = lane & 1, pg = p ? pv1 : pv0;
                        if (pg >= 0) {
                            const int64_t ph = (int64_t)pg * a.H_kv + hk;
                            if (lane < 2)
                                tc::bulk_g2s(stg + p * C::V_PAGE, a.v_pages + ph * C::V_PAGE, C::V_PAGE, &vfull[vsi]);
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
        // arrivals) are in; announced tiles run consecutively from the first.
        if (!ok || *abort_flag) {
            if (lane == 0) {
                for (int s = 0; s < C::NSK; ++s) {
                    if (k_last < s) continue;
                    const int t = k_last - (k_last - s) % C::NSK;
                    tc::mbar_wait_drain(&kfull[s], (t / C::NSK) & 1, kWaitLimitMla);
                }
                for (int s = 0; s < C::NSV; ++s) {
                    if (v_last < s) continue;
                    const int t = v_last - (v_last - s) % C::NSV;
                    tc::mbar_wait_drain(&vfull[s], (t / C::NSV) & 1, kWaitLimitMla);
                }
            }
            __syncwarp();
        }
    } else if (warp == C::MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = tc::idesc_fp4(128, MX);
            constexpr uint32_t idesc_pv = tc::idesc_fp4(GH, MX);
            const uint32_t q_addr = tc::smem_u32(q_op);
            const uint32_t p_addr = tc::smem_u32(p_op);
            const uint32_t kst_addr = tc::smem_u32(smem + C::SM_KST);
            const uint32_t vst_addr = tc::smem_u32(smem + C::SM_VST);
            const uint32_t psf_addr = tc::smem_u32(psf);
            uint64_t* last_bar = nullptr;   // the barrier of the last commit, and its phase
            uint32_t last_par = 0;
            // Descriptors and TMEM addresses are formed once; a K step, scale group or page moves
            // a shared-memory descriptor by its byte offset / 16 (the address field), so each
            // tcgen05 instruction costs the issuing lane an add or two.  The lane shares its
            // sub-partition's issue slots with four softmax warps.
            const uint64_t qdesc = tc::smem_desc(q_addr, 128, C::SBO);
            const uint32_t t_s = tbase + C::T_S, t_o = tbase + C::T_O, t_sfk = tbase + C::T_SFK;
            const uint32_t t_sfq = tbase + C::T_SFQ, t_sfv = tbase + C::T_SFV, t_sfp = tbase + C::T_SFP;
            auto issue_qk = [&](int j) -> bool {
                const int s = j % C::NSK;
                if (!tc::mbar_wait(&kfull[s], (j / C::NSK) & 1, abort_flag, kWaitLimitMla)) return false;
                tc::tc_fence_after();
                // the tile's key scale factors are in TMEM already: the softmax warps of the second
                // token quarter stored them before their arrival on s_free (or on q_ready)
                const uint32_t kt = kst_addr + s * C::KSTAGE;
                const uint64_t kdesc = tc::smem_desc(kt, 128, C::SBO);
                // S = Q_stacked K^T: rows are (head, residual half), columns the tile's tokens
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks) {
                    // MXFP4 packs two K steps per key scale column: byte offset 2 for the odd step
                    const uint32_t sfid = (uint32_t)(ks % C::KPG) * 2u;
                    tc::mma_fp4<MX>(t_s, qdesc + (uint64_t)(ks * 16), kdesc + (uint64_t)(ks * 16), idesc_qk | (sfid << 4),
                                    t_sfq + ks * 4, (t_sfk + (ks / C::KPG) * 4) | (sfid << 30), ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(s_full);
                tc::mma_commit(&kempty[s]);   // the K stage is free once QK has read it
                last_bar = &kempty[s];
                last_par = (uint32_t)(j / C::NSK) & 1u;
                return true;
            };
            bool ok = tc::mbar_wait(q_ready, 0, abort_flag, kWaitLimitMla);
            if (ok) tc::tc_fence_after();
            ok = ok && issue_qk(0);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n) {
                    // S has one buffer: QK of the next tile waits until every softmax warp read this one
                    if (!(ok = tc::mbar_wait(s_free, j & 1, abort_flag, kWaitLimitMla))) break;
                    tc::tc_fence_after();
                    if (!(ok = issue_qk(j + 1))) break;
                }
                const int s = j % C::NSV, pb = j & 1;
                if (!(ok = tc::mbar_wait(&p_ready[pb], (j >> 1) & 1, abort_flag, kWaitLimitMla))) break;
                if (!(ok = tc::mbar_wait(&vfull[s], (j / C::NSV) & 1, abort_flag, kWaitLimitMla))) break;
                tc::tc_fence_after();
                const uint32_t vt = vst_addr + s * C::VSTAGE;
                const uint64_t psd = tc::smem_desc(psf_addr + pb * 1024, 128, 128);
#pragma unroll
                for (int p = 0; p < 2; ++p) tc::tmem_cp_32x128b_x4(t_sfp + (pb * 2 + p) * 4, psd + (uint64_t)(p * 32));
                // the V scale factors were stored by the softmax warps of the first token quarter
                const uint64_t vd = tc::smem_desc(vt, 128, 256);
                const uint64_t pd = tc::smem_desc(p_addr + pb * C::P_BUF, 128, 256);
#pragma unroll
                for (int t = 0; t < MT; ++t) {
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const uint32_t sfid = MX ? (uint32_t)p * 2u : 0u;
                        const uint32_t sfa = MX ? (t_sfv + t * 4) | (sfid << 30) : t_sfv + t * 8 + p * 4;
                        tc::mma_fp4<MX>(t_o + t * GH, vd + (uint64_t)((p * C::V_PAGE + t * 4096) >> 4),
                                        pd + (uint64_t)((p * C::P_PAGE) >> 4), idesc_pv | (sfid << 29), sfa,
                                        t_sfp + (pb * 2 + p) * 4, (j > 0 || p > 0) ? 1u : 0u);
                    }
                }
                tc::mma_commit(&o_done[j & 1]);
                tc::mma_commit(&vempty[s]);
                last_bar = &vempty[s];
                last_par = (uint32_t)(j / C::NSV) & 1u;
            }
            if (!ok) {
                *abort_flag = 1;
                // unwinding: the tensor memory is freed below, so the MMAs and copies into it
                // must have finished
                if (last_bar) tc::mbar_wait_drain(last_bar, last_par, kWaitLimitMla);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int qd = warp & 3;                   // TMEM lane quadrant
        const int t4 = warp >> 2;                  // token quarter of S; M tile of O^T
        const bool rows_here = qd < C::NQ;         // the quadrant holds stacked query rows
        const int odd = lane & 1;                  // 0: the q1 row, 1: the q2 row of the lane pair
        const int h = 16 * qd + (lane >> 1);       // head (within the CTA) of the lane pair
        const uint32_t tq = tbase + ((uint32_t)(32 * qd) << 16);
        const float alpha = (FMT == BDFP4_NVFP4 && !(a.flags & BDFP4_FLAG_NO_UNDERFLOW)) ? kAlphaNV : 1.0f;
        bool bad = false;
        bool grp_abort = false;   // the quadrant's four warps gave up (alike in all of them)
        // a wait that gave up stops every role of the CTA
        auto fail_wait = [&]() {
            bad = true;
            *abort_flag = 1;
        };

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
        tc::named_bar_sync(5, 32 * C::NSW);
        if (tid < 64 && tid < n) {
            const uint32_t f = page_flags(tid);
            pflag[tid] = (uint8_t)f;
            if (f != 3u) *pflag_bad = 1;
        }
        // the query image arrives in two bulk copies from the prologue grid, which this grid
        // may overlap: griddepcontrol.wait holds the copies until its writes are visible
        if (tid == 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            const uint8_t* im = a.qpack + (int64_t)img * C::QPACK;
            tc::mbar_arrive_expect_tx(q_full, C::QPACK);
            tc::bulk_g2s(q_op, im, C::QOP_IMG, q_full);
            tc::bulk_g2s(smem + C::SM_QM, im + C::QOP_IMG, C::QMETA, q_full);
        }
        // the P scale-factor buffers: zero (rows past the heads must stay zero); operand rows
        // past the slice's stacked rows: zero
        for (int i = tid; i < 2 * 2 * 512 / 16; i += 32 * C::NSW) reinterpret_cast<uint4*>(psf)[i] = make_uint4(0, 0, 0, 0);
        for (int i = C::QOP_IMG / 16 + tid; i < C::Q_OP / 16; i += 32 * C::NSW)
            reinterpret_cast<uint4*>(q_op)[i] = make_uint4(0, 0, 0, 0);
        if (!tc::mbar_wait(q_full, 0, abort_flag, kWaitLimitMla)) fail_wait();
        // Key scale factors of tile jt (SFB of QK: token n at lane n % 32, column n / 32 of each
        // group's chunk, in every lane quadrant), from the K stage into this warp's lane quadrant.
        // The warps of the second token quarter store them once the tile's K stage landed and
        // the previous QK, the buffer's only reader, completed.
        auto write_sfk = [&](int jt) {
            const int s = jt % C::NSK;
            if (!tc::mbar_wait(&kfull[s], (jt / C::NSK) & 1, abort_flag, kWaitLimitMla)) fail_wait();
            const uint8_t* src = smem + C::SM_KST + s * C::KSTAGE + C::OFF_KS + 16 * lane;
#pragma unroll
            for (int kg = 0; kg < C::NKG; ++kg) {
                const uint4 w = *reinterpret_cast<const uint4*>(src + kg * 512);
                tc::tmem_st4(tq + C::T_SFK + kg * 4, w.x, w.y, w.z, w.w);
            }
            tc::tmem_wait_st();
        };
        if (t4 == 1) write_sfk(0);
        // query scale factors (SFA of QK): row r at lane r % 32, column r / 32 of each K step's
        // chunk, in every lane quadrant
        if (t4 == 0) {
#pragma unroll 1
            for (int ks = 0; ks < C::KS; ++ks) {
                uint32_t v[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int r = 32 * c + lane;
                    v[c] = 0u;
                    if (r < C::ROWS) {
                        const uint8_t* q = qsc + r * C::NBLK;
                        if constexpr (B == 16) v[c] = *reinterpret_cast<const uint32_t*>(q + ks * 4);
                        else v[c] = (uint32_t)q[ks * 2] | ((uint32_t)q[ks * 2 + 1] << 8);
                    }
                }
                tc::tmem_st4(tq + C::T_SFQ + ks * 4, v[0], v[1], v[2], v[3]);
            }
            tc::tmem_wait_st();
        }
        tc::tc_fence_before();
        tc::fence_proxy_async_smem();
        tc::named_bar_sync(5, 32 * C::NSW);   // psf and operand padding zeroed, page flags set before any tile
        const bool any_bad_page = *pflag_bad != 0;
        if (lane == 0) tc::mbar_arrive(q_ready);

        // per-lane state: the running maximum of head h (scaled log2 units), l over the lane's
        // tokens (in units of the current pre-scale), DYN: log2 of the head's current pre-scale
        float m_run = -INFINITY, l_run = 0.0f;
        int e_run = 11;
        const float ls = rows_here ? lsc[h] : 0.0f;   // logit scale of head h
        // log2 of alpha: alpha * 2^(x - m) is evaluated as 2^(x - (m - log2 alpha))
        const float la = alpha == kAlphaNV ? 11.0f : 0.0f;
        // the lane's 16 tokens: page t4 / 2 of the tile, slots 32 (t4 % 2) + 16 odd ..
        const int page_of_lane = t4 >> 1;
        const int tok_in_tile = 32 * t4 + 16 * odd;
        // P^T operand bytes of the lane (head h, its 16 tokens: 8 bytes of the row's 16-byte K
        // chunk t4 % 2) and its block-scale byte (NVFP4: block 2 (t4 % 2) + odd of the page;
        // MXFP4: block t4 % 2, the lane pair's)
        const int p_off = page_of_lane * C::P_PAGE + (h >> 3) * 256 + (t4 & 1) * 128 + (h & 7) * 16 + 8 * odd;
        const int sf_off = page_of_lane * 512 + (h & 31) * 16 + (h >> 5) * 4 + (MX ? (t4 & 1) : 2 * (t4 & 1) + odd);

        // The tile loop, in two copies: the page checks exist only in the copy a split with a
        // bad page runs, so the normal copy carries no extra live registers.
        auto tiles = [&](auto masked) {
            for (int j = 0; j < n; ++j) {
                const int tile = tile0 + j;
                bool pok0 = true, pok1 = true;
                if constexpr (decltype(masked)::value) {
                    const uint32_t f = j < 64 ? pflag[j] : page_flags(j);
                    pok0 = (f & 1u) != 0;
                    pok1 = (f & 2u) != 0;
                }
                const int jb = j & 1;
                if (rows_here) {
                    if (!tc::mbar_wait(s_full, j & 1, abort_flag, kWaitLimitMla)) fail_wait();
                    tc::tc_fence_after();
                    uint32_t sv[32];
                    tc::tmem_ld<32>(tq + C::T_S + 32 * t4, sv);
                    tc::tmem_wait_ld();
                    if (t4 == 1 && j + 1 < n) write_sfk(j + 1);
                    // S may be overwritten by the next QK once every row-owning warp has it in registers
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(s_free);
                    // (q1 + q2).k over the lane's 16 tokens: the pair's even lane keeps the first
                    // 16 of the quarter, the odd lane the last 16, each adding its partner's row
                    float x[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float lo = __uint_as_float(sv[i]), hi = __uint_as_float(sv[16 + i]);
                        const float give = odd ? lo : hi;
                        x[i] = (odd ? hi : lo) + __shfl_xor_sync(0xffffffffu, give, 1);
                    }
                    const int tok0 = tile * kTileTokens + tok_in_tile;
                    if (decltype(masked)::value || tok0 + 16 > N) {
                        int nv = N - tok0;
                        nv = nv < 0 ? 0 : (nv > 16 ? 16 : nv);
                        if (!(page_of_lane ? pok1 : pok0)) nv = 0;
#pragma unroll
                        for (int i = 0; i < 16; ++i) x[i] = i < nv ? x[i] : -INFINITY;
                    }
                    // block maximum (raw logits; the logit scale is positive), then the quarter's
                    // maximum of the head over the lane pair, posted for the quadrant's warps
                    float bm = x[0];
#pragma unroll
                    for (int i = 1; i < 16; ++i) bm = fmaxf(bm, x[i]);
                    const float pm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
                    float* rw = red + jb * GH * 4;
                    if (!odd) rw[h * 4 + t4] = pm;
                    // one decision for the quadrant's four warps, taken by the barrier itself (a
                    // role that gave up leaves a wait unfinished, and the wait sees its abort flag)
                    if (tc::named_bar_or(1 + qd, 128, bad)) {
                        grp_abort = true;
                        *abort_flag = 1;
                        break;
                    }
                    const float4 w4 = *reinterpret_cast<const float4*>(rw + h * 4);
                    const float mt = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
                    const float mn = fmaxf(m_run, mt * ls);
                    const float mz = mn == -INFINITY ? 0.0f : mn;
                    float corr = tc::ex2_approx(m_run - mz);   // 0 on the split's first tile
                    float base = mz - la;
                    bool rose = mn != m_run;
                    m_run = mn;
                    if constexpr (DYN) {
                        // this tile's pre-scale from its largest probability; O^T and l move to
                        // its units (an exact power of two, folded into corr)
                        const int e = dynamic_alpha_exp(tc::ex2_approx(fmaf(mt, ls, -mz)));
                        corr *= pow2f(e - e_run);
                        rose |= e != e_run;
                        e_run = e;
                        base = mz - (float)e;
                    }
                    // the quadrant's corrections and risen heads, for every softmax warp's O^T rescale
                    const uint32_t rb = __ballot_sync(0xffffffffu, rose) & 0x55555555u;
                    if (t4 == 0) {
                        if (!odd) cor[jb * GH + h] = rose ? corr : 1.0f;
                        if (lane == 0) rise[jb * 4 + qd] = rb;
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(&c_ready[jb]);
                    }
                    // probabilities and their FP4 quantization: NVFP4 one 16-token block per lane
                    // with the E4M3 scale of its largest alpha p; MXFP4 one 32-token block per lane
                    // pair, the OCP MX shared exponent taken in the log domain (the block maximum
                    // is 2^d with d = x_b ls - m <= 0, so floor(log2) = floor(d)) and the element
                    // 2^(x ls - m - (c - 127)), p its 2^(c - 127) multiple
                    float rinv, eb;
                    uint32_t code;
                    if constexpr (!MX) {
                        const float ab = tc::ex2_approx(fmaf(bm, ls, -base));
                        code = tc::e4m3x2_encode(__fmul_rn(ab, 1.0f / 6.0f), 0.0f) & 0xffu;
                        // a zero scale zeroes the whole block inside the MMA, whatever the element codes
                        rinv = tc::rcp_approx(tc::e4m3x2_value(code).x);
                        eb = base;
                    } else {
                        const float d = __fsub_rn(__fmul_rn(pm, ls), mz);
                        const int c = max(__float2int_rd(fmaxf(d, -256.0f)) + 125, 0);
                        code = (uint32_t)c;
                        eb = base + (float)(c - 127);   // base = m here (alpha = 1)
                        rinv = __uint_as_float(c > 0 ? (uint32_t)c << 23 : 0x00400000u);   // 2^(c - 127)
                    }
                    float lsum = 0.0f, pq[16];
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const float e0 = tc::ex2_approx(fmaf(x[i], ls, -eb));   // 0 for masked tokens
                        const float e1 = tc::ex2_approx(fmaf(x[i + 1], ls, -eb));
                        if constexpr (!MX) {
                            lsum += e0 + e1;   // alpha p
                            pq[i] = e0 * rinv;
                            pq[i + 1] = e1 * rinv;
                        } else {
                            lsum += (e0 + e1) * rinv;   // p
                            pq[i] = e0;
                            pq[i + 1] = e1;
                        }
                    }
                    l_run = fmaf(l_run, corr, lsum);
                    *reinterpret_cast<uint2*>(p_op + jb * C::P_BUF + p_off) = make_uint2(e2m1x8_encode(pq), e2m1x8_encode(pq + 8));
                    if (MX ? !odd : true) psf[jb * 1024 + sf_off] = (uint8_t)code;
                } else if (t4 == 1) {
                    // a lane quadrant without rows: only the next tile's key scale factors
                    if (!tc::mbar_wait(s_full, j & 1, abort_flag, kWaitLimitMla)) fail_wait();
                    tc::tc_fence_after();
                    if (j + 1 < n) write_sfk(j + 1);
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(s_free);
                }
                // V scale factors of the tile (SFA of PV: channel r of an M tile at lane r % 32,
                // column r / 32 of its chunk, in every lane quadrant), stored by the warps of the
                // first token quarter once the V stage landed and the previous PV, the buffer's
                // reader, completed.  Blocks past the sequence end or in a bad page are zeroed.
                // NVFP4: per M tile and page the stage holds the 32 x 16-byte rows as stored;
                // MXFP4: a row interleaves page 0's two blocks (bytes 0-1) with page 1's (2-3).
                if (t4 == 0) {
                    const int s = j % C::NSV;
                    if (!tc::mbar_wait(&vfull[s], (j / C::NSV) & 1, abort_flag, kWaitLimitMla)) fail_wait();
                    if (j > 0 && !tc::mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, kWaitLimitMla))
                        fail_wait();
                    tc::tc_fence_after();
                    const uint8_t* vs = smem + C::SM_VST + s * C::VSTAGE + C::OFF_VS;
                    uint32_t msk[2];
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const int t0 = tile * kTileTokens + p * kPageSlots;
                        int nvb = (N - t0 + B - 1) / B;
                        nvb = nvb < 0 ? 0 : (nvb > C::SPB ? C::SPB : nvb);
                        if (!(p ? pok1 : pok0)) nvb = 0;
                        if constexpr (!MX) {
                            msk[p] = nvb >= 4 ? 0xffffffffu : ((1u << (8 * nvb)) - 1u);
                        } else {
                            const uint32_t m16 = nvb >= 2 ? 0xffffu : ((1u << (8 * nvb)) - 1u);
                            msk[p] = m16 | (m16 << 16);
                        }
                    }
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        if constexpr (!MX) {
                            uint32_t w[8];
#pragma unroll
                            for (int p = 0; p < 2; ++p) {
                                const uint4 x = *reinterpret_cast<const uint4*>(vs + p * C::VS_PAGE + t * C::VS_TILE + 16 * lane);
                                w[4 * p + 0] = x.x & msk[p];
                                w[4 * p + 1] = x.y & msk[p];
                                w[4 * p + 2] = x.z & msk[p];
                                w[4 * p + 3] = x.w & msk[p];
                            }
                            tc::tmem_st8(tq + C::T_SFV + t * 8, w);
                        } else {
                            // lane i's 8 bytes of each page are channels 4 i .. 4 i + 3 of the tile's rows
                            const uint2 w0 = *reinterpret_cast<const uint2*>(vs + t * C::VS_TILE + 8 * lane);
                            const uint2 w1 = *reinterpret_cast<const uint2*>(vs + C::VS_PAGE + t * C::VS_TILE + 8 * lane);
                            const uint32_t x0 = w0.x & msk[0], x1 = w0.y & msk[0], y0 = w1.x & msk[1], y1 = w1.y & msk[1];
                            tc::tmem_st4(tq + C::T_SFV + t * 4, __byte_perm(x0, y0, 0x5410), __byte_perm(x0, y0, 0x7632),
                                         __byte_perm(x1, y1, 0x5410), __byte_perm(x1, y1, 0x7632));
                        }
                    }
                    tc::tmem_wait_st();
                }
                // O^T rescale of the heads whose maximum rose (any quadrant's), once the previous
                // tile's PV has completed: this warp's lane quadrant of M tile t4
                if (!tc::mbar_wait(&c_ready[jb], (j >> 1) & 1, abort_flag, kWaitLimitMla)) fail_wait();
                if (j > 0) {
                    uint32_t any = 0u;
#pragma unroll
                    for (int g = 0; g < C::NQ; ++g) any |= rise[jb * 4 + g];
                    if (any) {
                        if (!tc::mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, kWaitLimitMla)) fail_wait();
                        tc::tc_fence_after();
                        const uint32_t ob = tq + C::T_O + t4 * GH;
                        // per quadrant with a risen head: its 16 head columns in one round trip,
                        // the heads that did not rise multiplied by exactly 1
#pragma unroll 1
                        for (int g = 0; g < C::NQ; ++g) {
                            if (!rise[jb * 4 + g]) continue;
                            uint32_t ov[16];
                            tc::tmem_ld<16>(ob + 16 * g, ov);
                            const float4* cg = reinterpret_cast<const float4*>(cor + jb * GH + 16 * g);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const float4 c4 = cg[k];
                                ov[4 * k + 0] = __float_as_uint(__uint_as_float(ov[4 * k + 0]) * c4.x);
                                ov[4 * k + 1] = __float_as_uint(__uint_as_float(ov[4 * k + 1]) * c4.y);
                                ov[4 * k + 2] = __float_as_uint(__uint_as_float(ov[4 * k + 2]) * c4.z);
                                ov[4 * k + 3] = __float_as_uint(__uint_as_float(ov[4 * k + 3]) * c4.w);
                            }
                            tc::tmem_st16(ob + 16 * g, ov);
                        }
                        tc::tmem_wait_st();
                    }
                }
                tc::tc_fence_before();
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&p_ready[jb]);
                // a warp without rows takes part in no barrier of the loop: it stops here
                if (!rows_here && bad) break;
            }
        };
        if (any_bad_page) tiles(std::true_type{});
        else tiles(std::false_type{});
        if (!grp_abort && !bad) {
            if (!tc::mbar_wait(&o_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, kWaitLimitMla)) fail_wait();
            tc::tc_fence_after();
        }

        // ------------------------------------------------------------ epilogue (thread = channel)
        const bool fail = tc::named_bar_or(5, 32 * C::NSW, grp_abort || bad || *abort_flag);
        if (fail) {
            if (tid == 0) *abort_flag = 1;
        } else {
            if (rows_here) {
                const float l2 = l_run + __shfl_xor_sync(0xffffffffu, l_run, 1);
                if (!odd) lred[h * 4 + t4] = l2;
            }
            tc::named_bar_sync(5, 32 * C::NSW);
            // O and l both carry the factor alpha (P^ is alpha p quantized), so it cancels
            const float oscale = FMT == BDFP4_NVFP4 ? a.v_gscale[hk] : 1.0f;
            if (rows_here && t4 == 0 && !odd) {
                const float4 r4 = *reinterpret_cast<const float4*>(lred + h * 4);
                const float l = r4.x + r4.y + r4.z + r4.w;
                // DYN: splits end in different units; the partials leave in the units of p
                const float un = DYN ? pow2f(-e_run) : 1.0f;
                hscale[h] = nspl == 1 ? (l > 0.0f ? oscale / l : 0.0f) : oscale * un;
                if (nspl > 1) {
                    const int64_t row = (int64_t)b * a.H_q + h0 + h;
                    a.ws_ml[(row * a.max_splits + split) * 2 + 0] = m_run;
                    a.ws_ml[(row * a.max_splits + split) * 2 + 1] = l * un;
                }
            }
            tc::named_bar_sync(5, 32 * C::NSW);
            const int chan = t4 * 128 + 32 * qd + lane;
#pragma unroll 1
            for (int c0 = 0; c0 < GH; c0 += 16) {
                uint32_t ov[16];
                tc::tmem_ld<16>(tq + C::T_O + t4 * GH + c0, ov);
                tc::tmem_wait_ld();
#pragma unroll
                for (int g = 0; g < 16; ++g) {
                    const int64_t row = (int64_t)b * a.H_q + h0 + c0 + g;
                    const float o = __uint_as_float(ov[g]) * hscale[c0 + g];
                    if (nspl == 1) a.out[row * C::DV + chan] = __float2bfloat16(o);
                    else a.ws_o[(row * a.max_splits + split) * C::DV + chan] = o;
                }
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) set_status(a.dev_status, BDFP4_DEV_TIMEOUT);
    if (warp == C::MMA_WARP) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tbase, C::T_ALLOC);
    }
}

template <int FMT, int GH, bool DYN = false>
static int launch_mla(const DecodeArgs& a, cudaStream_t st, const StepArgs* step) {
    using C = MlaCfg<FMT, GH>;
    using RG = RowGeom<FMT, 576>;
    static bool attr_set = false;
    if (!attr_set) {
        const cudaError_t e = cudaFuncSetAttribute(decode_mla_tc_kernel<FMT, GH, DYN>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) {
            record_cuda_error(e);
            return BDFP4_ERR_CUDA;
        }
        attr_set = true;
    }
    const int G = a.H_q / a.H_kv, nh = G / GH;
    const int64_t images = (int64_t)a.B * a.H_kv * nh;
    constexpr int RPC = 256 / RG::rt, per_img = (GH + RPC - 1) / RPC;
    int64_t ctas = images * per_img;
    StepArgs s{};
    if (step) {
        const int64_t rows = (int64_t)a.B * a.H_kv;
        ctas += k_append_ctas_wide<FMT, 576>(rows) + v_append_ctas<512>(rows);
        s = *step;
    }
    prep_mla_kernel<FMT, GH><<<(unsigned)ctas, 256, 0, st>>>(a, s, step ? 1 : 0);
    const int rc = launch_status();
    if (rc != BDFP4_OK) return rc;
    // programmatic dependent launch: the decode CTAs start (TMEM, barriers, K/V
    // streaming) while the prologue runs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.max_splits, a.H_kv * nh, a.B);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_mla_tc_kernel<FMT, GH, DYN>, a);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return BDFP4_ERR_CUDA;
    }
    return launch_status();
}

bool mla_tc_supported(int d_k, int d_v, int G) {
    return d_k == 576 && d_v == 512 && (G == 16 || G == 32 || G == 64 || G == 128);
}

int mla_query_image_bytes(int fmt, int G) {
    const int gh = G < 64 ? G : 64;
    return fmt == BDFP4_NVFP4 ? (gh == 16 ? MlaCfg<BDFP4_NVFP4, 16>::QPACK
                                          : gh == 32 ? MlaCfg<BDFP4_NVFP4, 32>::QPACK : MlaCfg<BDFP4_NVFP4, 64>::QPACK)
                              : (gh == 16 ? MlaCfg<BDFP4_MXFP4, 16>::QPACK
                                          : gh == 32 ? MlaCfg<BDFP4_MXFP4, 32>::QPACK : MlaCfg<BDFP4_MXFP4, 64>::QPACK);
}

int launch_decode_mla_tc(const DecodeArgs& a, int fmt, int G, cudaStream_t st, const StepArgs* step) {
    const int gh = G < 64 ? G : 64;
    if (fmt == BDFP4_NVFP4 && (a.flags & BDFP4_FLAG_DYNAMIC_ALPHA)) {
        switch (gh) {
            case 16: return launch_mla<BDFP4_NVFP4, 16, true>(a, st, step);
            case 32: return launch_mla<BDFP4_NVFP4, 32, true>(a, st, step);
            case 64: return launch_mla<BDFP4_NVFP4, 64, true>(a, st, step);
        }
    } else if (fmt == BDFP4_NVFP4) {
        switch (gh) {
            case 16: return launch_mla<BDFP4_NVFP4, 16>(a, st, step);
            case 32: return launch_mla<BDFP4_NVFP4, 32>(a, st, step);
            case 64: return launch_mla<BDFP4_NVFP4, 64>(a, st, step);
        }
    } else {
        switch (gh) {
            case 16: return launch_mla<BDFP4_MXFP4, 16>(a, st, step);
            case 32: return launch_mla<BDFP4_MXFP4, 32>(a, st, step);
            case 64: return launch_mla<BDFP4_MXFP4, 64>(a, st, step);
        }
    }
    return BDFP4_ERR_UNSUPPORTED;
}

}  // namespace bdfp4
