// decode_mla_tc.cu -- FP4 paged decode attention on the sm_100a tensor cores for
// latent-KV (MLA) shapes: d_k = 576 (512-d latent + 64-d rope), d_v = 512 (the
// latent), many query heads over one KV head (BitDecoding-FP4, Article Summary:
// stacked query MMA on paged KV caches, transposed softmax with fused probability
// quantization, dual-residual query, underflow-aware probability scaling; the
// method is evaluated on GQA and MLA models).
//
// One CTA per (sequence, KV head, slice of GH <= 64 query heads, split), one
// CTA per SM.  TMEM (512 columns) holds
//   S^T [128 tokens][GH heads]         q1.k and q2.k accumulate into the same cells,
//   O^T [512 channels = 4 x 128 lanes][GH heads], accumulated across the tiles,
//   and the scale factors of every MMA operand.
// O stays in TMEM: when a head's running maximum rises, the softmax warps that
// own the head rescale its O columns after the previous tile's PV completed and
// before this tile's PV is issued -- the online-softmax update, in place.
//   warps 0 .. 4 NSG - 1   softmax: group g owns heads 16 g .. 16 g + 15, its warp q
//                          the tokens (TMEM lanes) 32 q .. 32 q + 31
//   warp  4 NSG            producer: K and V pages by bulk copy, K scales by cp.async
//   warp  4 NSG + 1        MMA issuer (one lane) and TMEM owner
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
    static constexpr int HG = 16;                      // heads per softmax group
    static constexpr int NSG = GH / HG;                // softmax groups
    static constexpr int NSW = 4 * NSG;                // softmax warps
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
    // 32 x 16-byte tcgen05.cp source (row i: rows i, 32 + i, 64 + i, 96 + i)
    static constexpr int OFF_KS = 2 * K_PAGE;
    static constexpr int KSTAGE = OFF_KS + NKG * 512;
    // V stage: the two pages, then their scale blocks
    static constexpr int OFF_VS = 2 * V_PAGE;
    static constexpr int VSTAGE = OFF_VS + 2 * VS_PAGE;
    // query image: q1 and q2 operands [GH rows][DK] in K-major core blocks, their
    // scale codes [2][GH][NBLK], the logit scales [GH] (fp32)
    static constexpr int Q_OP = GH * DK / 2;
    static constexpr int QSC = GH * NBLK;
    static constexpr int QPACK = 2 * Q_OP + 2 * QSC + GH * 4;
    static constexpr int P_PAGE = GH / 8 * 256;        // P^T operand of one page: GH rows x 64 tokens
    static constexpr int P_BUF = 2 * P_PAGE;
    static constexpr int RED_BUF = GH * 8;             // floats: [GH][4 quadrants][2 half warps]
    // shared memory map
    static constexpr int SM_KST = 0;
    static constexpr int SM_VST = SM_KST + NSK * KSTAGE;
    static constexpr int SM_Q = SM_VST + NSV * VSTAGE;
    static constexpr int SM_P = (SM_Q + QPACK + 127) / 128 * 128;
    static constexpr int SM_PSF = SM_P + 2 * P_BUF;    // [2 buf][2 page][32 rows][16 B] P scales
    static constexpr int SM_RED = SM_PSF + 2 * 2 * 512;
    // per softmax warp and head of its group: the tile's softmax terms for the warp's two
    // token blocks {logit scale, exponent base, correction, 1 / block scale} x 2, the two
    // block-scale codes, and an output scale
    static constexpr int WST_WARP = HG * 32 + HG * 4 + HG * 4;
    static constexpr int SM_WST = SM_RED + 2 * RED_BUF * 4;
    static constexpr int SM_BARS = SM_WST + NSW * WST_WARP;
    static constexpr int NBARS = 2 * NSK + 2 * NSV + 8;
    static constexpr int SM_MISC = SM_BARS + NBARS * 8;   // tmem slot, abort flags
    static constexpr int SM_PFLAG = SM_MISC + 32;   // [64] page flags of the split's tiles, any-bad
    static constexpr int SMEM = SM_PFLAG + 64 + 16;
    // TMEM column map
    static constexpr int T_S = 0;
    static constexpr int T_O = GH;                     // M tile t at T_O + t GH
    static constexpr int T_SFK = (T_O + MT * GH + 3) / 4 * 4;   // 2 buffers x NKG groups x 4
    static constexpr int T_SFQ = T_SFK + 2 * NKG * 4;           // 2 operands x KS steps x 4
    static constexpr int NSFV = MX ? 2 : 1;                     // V scale-factor buffers
    static constexpr int T_SFV = T_SFQ + 2 * KS * 4;            // NSFV x MT tiles x 2 pages x 4
    static constexpr int T_SFP = T_SFV + NSFV * MT * 8;         // 2 buffers x 2 pages x 4
    static constexpr int T_USED = T_SFP + 16;
    static constexpr int T_ALLOC = 512;
    static_assert(GH % HG == 0 && GH <= 64, "head slice");
    static_assert(T_USED <= T_ALLOC, "TMEM budget");
    static_assert(SMEM <= 232448 && SMEM > 232448 / 2, "one CTA per SM");
    static_assert(QPACK % 16 == 0, "query image copied in 16-byte units");
    // the image of a head slice fits the workspace region reserved for its heads
    static_assert(QPACK <= kQueryImageBytes * GH, "query image larger than its workspace share");
    static_assert(NSG + 2 <= 16, "named barriers");
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
        uint8_t* dst = im + o * C::Q_OP + (r >> 3) * C::SBO + (e0 >> 5) * 128 + (r & 7) * 16 + (e0 & 31) / 2;
        if constexpr (B == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        im[2 * C::Q_OP + o * C::QSC + r * C::NBLK + j] = (uint8_t)(o ? c2 : c1);
    }
    if (j == 0) {
        const float gk = FMT == BDFP4_NVFP4 ? a.k_gscale[hk] : 1.0f;
        reinterpret_cast<float*>(im + 2 * C::Q_OP + 2 * C::QSC)[r] = a.sm_scale * gq * gk * kLog2e;
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
    constexpr int B = C::B, HG = C::HG, MT = C::MT;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* q_op = smem + C::SM_Q;
    const uint8_t* qsc = q_op + 2 * C::Q_OP;
    const float* lsc = reinterpret_cast<const float*>(q_op + 2 * C::Q_OP + 2 * C::QSC);
    uint8_t* p_op = smem + C::SM_P;
    uint8_t* psf = smem + C::SM_PSF;
    float* red = reinterpret_cast<float*>(smem + C::SM_RED);
    uint8_t* wst = smem + C::SM_WST;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SM_BARS);
    uint64_t* kfull = bars;                   // [NSK] K tile landed -> MMA
    uint64_t* kempty = kfull + C::NSK;        // [NSK] QK done -> producer
    uint64_t* vfull = kempty + C::NSK;        // [NSV] V tile landed -> MMA, softmax
    uint64_t* vempty = vfull + C::NSV;        // [NSV] PV done -> producer
    uint64_t* s_full = vempty + C::NSV;       // QK done -> softmax
    uint64_t* s_free = s_full + 1;            // S read by every softmax warp -> MMA
    uint64_t* p_ready = s_free + 1;           // [2] P, its scales and O rescaled -> MMA
    uint64_t* o_done = p_ready + 2;           // [2] PV done -> softmax (rescale, epilogue), MMA
    uint64_t* q_ready = o_done + 2;           // query operand and its scale factors -> MMA
    uint64_t* q_full = q_ready + 1;           // query image landed -> softmax
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
        tc::mbar_init(s_free, C::NSW);
        tc::mbar_init(&p_ready[0], C::NSW);
        tc::mbar_init(&p_ready[1], C::NSW);
        tc::mbar_init(&o_done[0], 1);
        tc::mbar_init(&o_done[1], 1);
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
        // Step k issues the K half of tile k and the V half of tile k - 1 (the
        // block-table reads of 32 tiles at a time, one per lane, as in the d = 128 kernel)
        bool ok = true;
        int pv0 = -1, pv1 = -1;
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
                }
                pv0 = pg0;
                pv1 = pg1;
            }
        }
        if (!ok && lane == 0) *abort_flag = 1;
    } else if (warp == C::MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_fp4(GH, MX);
            const uint32_t q_addr = tc::smem_u32(q_op);
            const uint32_t p_addr = tc::smem_u32(p_op);
            const uint32_t kst_addr = tc::smem_u32(smem + C::SM_KST);
            const uint32_t vst_addr = tc::smem_u32(smem + C::SM_VST);
            const uint32_t psf_addr = tc::smem_u32(psf);
            auto issue_qk = [&](int j) -> bool {
                const int s = j % C::NSK, buf = j & 1;
                if (!tc::mbar_wait(&kfull[s], (j / C::NSK) & 1, abort_flag, kWaitLimitMla)) return false;
                tc::tc_fence_after();
                // the scale rows came through cp.async (generic proxy); tcgen05.cp reads them
                // through the async proxy
                tc::fence_proxy_async_smem();
                const uint32_t kt = kst_addr + s * C::KSTAGE;
#pragma unroll
                for (int kg = 0; kg < C::NKG; ++kg)
                    tc::tmem_cp_32x128b_x4(tbase + C::T_SFK + (buf * C::NKG + kg) * 4,
                                           tc::smem_desc(kt + C::OFF_KS + kg * 512, 128, 128));
                // S^T = K (q1 + q2)^T: the q2 products accumulate onto the q1 ones (loops kept
                // rolled: one lane issues them, and unrolled descriptors cost registers
                // every warp of the CTA is sized for)
#pragma unroll 1
                for (int o = 0; o < 2; ++o) {
#pragma unroll 1
                    for (int ks = 0; ks < C::KS; ++ks) {
                        // MXFP4 packs two K steps per key scale column: byte offset 2 for the odd step
                        const uint32_t sfid = (uint32_t)(ks % C::KPG) * 2u;
                        tc::mma_fp4<MX>(tbase + C::T_S, tc::smem_desc(kt + ks * 256, 128, C::SBO),
                                        tc::smem_desc(q_addr + o * C::Q_OP + ks * 256, 128, C::SBO),
                                        idesc | (sfid << 29),
                                        (tbase + C::T_SFK + (buf * C::NKG + ks / C::KPG) * 4) | (sfid << 30),
                                        tbase + C::T_SFQ + (o * C::KS + ks) * 4, (o > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                tc::mma_commit(s_full);
                tc::mma_commit(&kempty[s]);   // the K stage is free once QK has read it
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
                // NVFP4 V scale factors have one TMEM buffer: the previous PV must have read it
                if (!MX && j > 0 && !(ok = tc::mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag,
                                                         kWaitLimitMla)))
                    break;
                tc::tc_fence_after();
                const uint32_t vt = vst_addr + s * C::VSTAGE;
#pragma unroll
                for (int p = 0; p < 2; ++p)
                    tc::tmem_cp_32x128b_x4(tbase + C::T_SFP + (pb * 2 + p) * 4,
                                           tc::smem_desc(psf_addr + (pb * 2 + p) * 512, 128, 128));
                if constexpr (!MX) {
                    // each M tile's scale block of a page is already the 32 x 16-byte copy source
#pragma unroll
                    for (int t = 0; t < MT; ++t)
#pragma unroll
                        for (int p = 0; p < 2; ++p)
                            tc::tmem_cp_32x128b_x4(tbase + C::T_SFV + t * 8 + p * 4,
                                                   tc::smem_desc(vt + C::OFF_VS + p * C::VS_PAGE + t * C::VS_TILE,
                                                                 128, 128));
                }
                const int vb = MX ? pb : 0;
#pragma unroll 1
                for (int t = 0; t < MT; ++t) {
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        tc::mma_fp4<MX>(tbase + C::T_O + t * GH, tc::smem_desc(vt + p * C::V_PAGE + t * 4096, 128, 256),
                                        tc::smem_desc(p_addr + pb * C::P_BUF + p * C::P_PAGE, 128, 256), idesc,
                                        tbase + C::T_SFV + (vb * MT + t) * 8 + p * 4,
                                        tbase + C::T_SFP + (pb * 2 + p) * 4, (j > 0 || p > 0) ? 1u : 0u);
                    }
                }
                tc::mma_commit(&o_done[j & 1]);
                tc::mma_commit(&vempty[s]);
            }
            if (!ok) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int grp = warp >> 2;                 // head group
        const int qd = warp & 3;                   // TMEM lane quadrant = tokens 32 qd .. 32 qd + 31
        const int gb = grp * HG;                   // first head of the group (within the CTA)
        const int bar_id = 1 + grp;                // named barrier of the group (128 threads)
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
        // the query image arrives in one bulk copy from the prologue grid, which this
        // grid may overlap: griddepcontrol.wait holds the copy until its writes are visible
        if (tid == 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            tc::mbar_arrive_expect_tx(q_full, C::QPACK);
            tc::bulk_g2s(q_op, a.qpack + (int64_t)img * C::QPACK, C::QPACK, q_full);
        }
        // the P scale-factor buffers: zero (columns past the heads must stay zero)
        for (int i = tid; i < 2 * 2 * 512 / 16; i += 32 * C::NSW) reinterpret_cast<uint4*>(psf)[i] = make_uint4(0, 0, 0, 0);
        if (!tc::mbar_wait(q_full, 0, abort_flag, kWaitLimitMla)) bad = true;
        // query scale factors (SFB of QK): row n at lane n % 32, column n / 32 of each K step's chunk
        if (grp == 0) {
#pragma unroll
            for (int o = 0; o < 2; ++o) {
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks) {
                    uint32_t v[2] = {0u, 0u};
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int r = 32 * c + lane;
                        if (r < GH) {
                            const uint8_t* q = qsc + o * C::QSC + r * C::NBLK;
                            if constexpr (B == 16) v[c] = *reinterpret_cast<const uint32_t*>(q + ks * 4);
                            else v[c] = (uint32_t)q[ks * 2] | ((uint32_t)q[ks * 2 + 1] << 8);
                        }
                    }
                    tc::tmem_st4(tq + C::T_SFQ + (o * C::KS + ks) * 4, v[0], v[1], 0u, 0u);
                }
            }
            tc::tmem_wait_st();
        }
        tc::tc_fence_before();
        tc::fence_proxy_async_smem();
        tc::named_bar_sync(1 + C::NSG, 32 * C::NSW);   // psf zeroed and page flags set before any tile
        const bool any_bad_page = *pflag_bad != 0;
        if (lane == 0) tc::mbar_arrive(q_ready);

        // Running maxima (scaled log2 units) are kept one head per lane: lane g of every warp
        // of the group tracks head gb + g and posts, per tile, the terms every lane of the
        // warp needs for that head to the warp's own shared-memory slots.
        float4* const wterm = reinterpret_cast<float4*>(wst + warp * C::WST_WARP);   // [HG][2 blocks]
        uint32_t* const wcode = reinterpret_cast<uint32_t*>(wst + warp * C::WST_WARP + HG * 32);   // [HG]
        float* const wout = reinterpret_cast<float*>(wst + warp * C::WST_WARP + HG * 36);          // [HG]
        float m_lane = -INFINITY;                   // running maximum of head gb + lane
        int e_lane = 11;                            // DYN: log2 of head gb + lane's current pre-scale
        const float ls_lane = lane < HG ? lsc[gb + lane] : 0.0f;
        float l_part[HG];
#pragma unroll
        for (int g = 0; g < HG; ++g) l_part[g] = 0.0f;
        // TMEM lane 32 qd + lane holds token 32 qd + lane of the tile: slot 32 (qd % 2) + lane
        // of page qd / 2
        const int page_of_thread = qd >> 1;
        const int pos_in_page = 32 * (qd & 1) + lane;
        const int tok_in_tile = 32 * qd + lane;
        // log2 of alpha: alpha * 2^(x - m) is evaluated as 2^(x - (m - log2 alpha))
        const float la = alpha == kAlphaNV ? 11.0f : 0.0f;
        const bool lo_half = lane < 16;
        // P^T operand bytes: a lane pair (tokens 2i, 2i + 1) fills one byte of each head
        // row; per pair of heads the even lane writes the first, the odd lane the second
        const int hsel = lane & 1;
        const uint32_t psel = (lane & 1) ? 0x0004u : 0x0040u;   // byte 0 <- token 2i, byte 1 <- token 2i + 1
        const bool sfstore = (lane & (B - 1)) < 2;             // first two lanes of a token block
        uint8_t* const pbyte = p_op + page_of_thread * C::P_PAGE + (qd & 1) * 128 + (lane >> 1);
        uint8_t* const sfbase = psf + page_of_thread * 512 + pos_in_page / B;

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
                if (!tc::mbar_wait(s_full, j & 1, abort_flag, kWaitLimitMla)) bad = true;
                tc::tc_fence_after();
                uint32_t sr[HG];
                tc::tmem_ld<HG>(tq + C::T_S + gb, sr);
                tc::tmem_wait_ld();
                // S may be overwritten by the next QK once every softmax warp has it in registers
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(s_free);
                const int token = tile * kTileTokens + tok_in_tile;
                const bool valid = token < N && (page_of_thread ? pok1 : pok0);
                // raw logits (q1 + q2).k; maxima over each half warp (16 consecutive slots)
                float* rw = red + (j & 1) * C::RED_BUF;
    #pragma unroll
                for (int g = 0; g < HG; ++g) {
                    const float x = valid ? __uint_as_float(sr[g]) : -INFINITY;
                    const float lo = tc::redux_max_f32(lo_half ? x : -INFINITY, 0xffffffffu);
                    const float hi = tc::redux_max_f32(lo_half ? -INFINITY : x, 0xffffffffu);
                    if (lane == 0) *reinterpret_cast<float2*>(rw + ((gb + g) * 4 + qd) * 2) = make_float2(lo, hi);
                }
                // one decision for the group's four warps, taken by the barrier itself (a role
                // that gave up leaves a wait here unfinished, and the wait sees its abort flag)
                if (tc::named_bar_or(bar_id, 128, bad)) {
                    grp_abort = true;
                    break;
                }
                // new running maxima, one head per lane, and the scales of the warp's two token
                // blocks: the block maximum of alpha p is 2^(x_b ls - base) for the block's largest
                // logit x_b, so the scale is the one the block's largest member picks
                bool rose = false;
                if (lane < HG) {
                    const float* w = rw + (gb + lane) * 8;
                    const float4 w0 = *reinterpret_cast<const float4*>(w);
                    const float4 w1 = *reinterpret_cast<const float4*>(w + 4);
                    const float mt = fmaxf(fmaxf(fmaxf(w0.x, w0.y), fmaxf(w0.z, w0.w)),
                                           fmaxf(fmaxf(w1.x, w1.y), fmaxf(w1.z, w1.w)));
                    const float mn = fmaxf(m_lane, mt * ls_lane);
                    const float mz = mn == -INFINITY ? 0.0f : mn;
                    float corr = tc::ex2_approx(m_lane - mz);   // 0 on the split's first tile
                    float base = mz - la;
                    rose = mn != m_lane;
                    m_lane = mn;
                    if constexpr (DYN) {
                        // this tile's pre-scale from its largest probability; O^T and l move to
                        // its units (an exact power of two, folded into corr)
                        const int e = dynamic_alpha_exp(tc::ex2_approx(fmaf(mt, ls_lane, -mz)));
                        corr *= pow2f(e - e_lane);
                        rose |= e != e_lane;
                        e_lane = e;
                        base = mz - (float)e;
                    }
                    const float bm_lo = w[qd * 2], bm_hi = w[qd * 2 + 1];
                    // per block: NVFP4 {ls, base, corr, 1 / scale}, the element is alpha p / scale;
                    // MXFP4 {ls, base + e, corr, 2^e} for the scale 2^e, the element is 2^(x ls - base - e)
                    // (the exponent's argument stays small, as the OCP rule's element) and p its 2^e multiple
                    float r_lo, r_hi, b_lo = base, b_hi = base;
                    uint32_t codes;
                    if constexpr (!MX) {
                        const float a_lo = tc::ex2_approx(fmaf(bm_lo, ls_lane, -base));
                        const float a_hi = tc::ex2_approx(fmaf(bm_hi, ls_lane, -base));
                        codes = tc::e4m3x2_encode(__fmul_rn(a_lo, 1.0f / 6.0f), __fmul_rn(a_hi, 1.0f / 6.0f));
                        const float2 sg = tc::e4m3x2_value(codes);
                        // a zero scale zeroes the whole block inside the MMA, whatever the element codes
                        r_lo = tc::rcp_approx(sg.x);
                        r_hi = tc::rcp_approx(sg.y);
                    } else {
                        // one 32-token block per warp; the OCP MX shared exponent in the log domain:
                        // the block maximum is 2^d with d = x_b ls - m <= 0, so floor(log2) = floor(d)
                        // and the element is p 2^(127 - c) for the E8M0 code c
                        const float d = __fsub_rn(__fmul_rn(fmaxf(bm_lo, bm_hi), ls_lane), mz);
                        const int c = max(__float2int_rd(fmaxf(d, -256.0f)) + 125, 0);
                        codes = (uint32_t)c | ((uint32_t)c << 8);
                        b_lo = b_hi = mz + (float)(c - 127);
                        r_lo = r_hi = __uint_as_float(c > 0 ? (uint32_t)c << 23 : 0x00400000u);   // 2^(c - 127)
                    }
                    wterm[lane * 2 + 0] = make_float4(ls_lane, b_lo, corr, r_lo);
                    wterm[lane * 2 + 1] = make_float4(ls_lane, b_hi, corr, r_hi);
                    wcode[lane] = codes;
                }
                const uint32_t rmask = j > 0 ? __ballot_sync(0xffffffffu, rose) : 0u;
                __syncwarp();
                // O^T rescale of the heads whose maximum rose, once the previous tile's PV has
                // completed; the group's warps decide alike, having read the same maxima
                if (rmask) {
                    if (!tc::mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, kWaitLimitMla)) bad = true;
                    tc::tc_fence_after();
                    uint32_t rem = rmask;
                    while (rem) {
                        // up to four heads per round trip: their columns in the four M tiles
                        int hs_[4];
                        uint32_t ov[4][MT];
    #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            hs_[k] = rem ? __ffs(rem) - 1 : -1;
                            if (rem) rem &= rem - 1;
                            if (hs_[k] >= 0) {
    #pragma unroll
                                for (int t = 0; t < MT; ++t) tc::tmem_ld<1>(tq + C::T_O + t * GH + gb + hs_[k], &ov[k][t]);
                            }
                        }
                        tc::tmem_wait_ld();
    #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            if (hs_[k] < 0) continue;
                            const float c = wterm[hs_[k] * 2].z;
    #pragma unroll
                            for (int t = 0; t < MT; ++t)
                                tc::tmem_st1(tq + C::T_O + t * GH + gb + hs_[k], __float_as_uint(__uint_as_float(ov[k][t]) * c));
                        }
                    }
                    tc::tmem_wait_st();
                }
                // probabilities and their FP4 quantization, two heads per conversion
                uint8_t* const pb = pbyte + (j & 1) * C::P_BUF;
                uint8_t* const sfb = sfbase + (j & 1) * 2 * 512;
                const int half = lo_half ? 0 : 1;
    #pragma unroll
                for (int g = 0; g < HG; g += 2) {
                    float q[2];
    #pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const float4 v = wterm[(g + u) * 2 + half];
                        const float x = valid ? __uint_as_float(sr[g + u]) : -INFINITY;
                        const float e = tc::ex2_approx(fmaf(x, v.x, -v.y));   // 0 for masked tokens
                        const float y = MX ? e * v.w : e;                     // alpha p
                        l_part[g + u] = fmaf(l_part[g + u], v.z, y);          // l in units of alpha
                        q[u] = MX ? e : e * v.w;
                    }
                    const uint32_t mine = e2m1x2_encode(q[0], q[1]);   // head g in bits 0..3, head g + 1 in 4..7
                    const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
                    const uint32_t wv = __byte_perm(mine, other, psel) >> (4 * hsel);
                    const int hr = gb + g + hsel;
                    pb[(hr >> 3) * 256 + (hr & 7) * 16] = (uint8_t)((wv & 0xfu) | ((wv >> 4) & 0xf0u));
                    if (sfstore) sfb[(hr & 31) * 16 + (hr >> 5) * 4] = (uint8_t)(wcode[g + hsel] >> (8 * half));
                }
                // V scale factors (group 0): blocks past the sequence end are zeroed (NVFP4, in the
                // stage before its TMEM copy) or masked (MXFP4, stored into TMEM by these warps)
                if (grp == 0) {
                    const int s = j % C::NSV;
                    const bool tail = (tile + 1) * kTileTokens > N;
                    uint8_t* vs = smem + C::SM_VST + s * C::VSTAGE + C::OFF_VS;
                    if constexpr (!MX) {
                        if (tail || !pok0 || !pok1) {
                            if (!tc::mbar_wait(&vfull[s], (j / C::NSV) & 1, abort_flag, kWaitLimitMla)) bad = true;
    #pragma unroll
                            for (int p = 0; p < 2; ++p) {
                                const int t0 = tile * kTileTokens + p * kPageSlots;
                                int nvb = (N - t0 + B - 1) / B;
                                nvb = nvb < 0 ? 0 : (nvb > C::SPB ? C::SPB : nvb);
                                if (!(p ? pok1 : pok0)) nvb = 0;
                                for (int bb = nvb; bb < C::SPB; ++bb)
    #pragma unroll
                                    for (int t = 0; t < MT; ++t)
                                        vs[p * C::VS_PAGE + t * C::VS_TILE + lane * 16 + qd * 4 + bb] = 0;
                            }
                        }
                    } else {
                        if (!tc::mbar_wait(&vfull[s], (j / C::NSV) & 1, abort_flag, kWaitLimitMla)) bad = true;
                        uint32_t mask[2];
    #pragma unroll
                        for (int p = 0; p < 2; ++p) {
                            const int t0 = tile * kTileTokens + p * kPageSlots;
                            int nvb = (N - t0 + B - 1) / B;
                            nvb = nvb < 0 ? 0 : (nvb > C::SPB ? C::SPB : nvb);
                            if (!(p ? pok1 : pok0)) nvb = 0;
                            mask[p] = nvb >= 2 ? 0xffffu : ((1u << (8 * nvb)) - 1u);
                        }
    #pragma unroll
                        for (int t = 0; t < MT; ++t) {
                            uint32_t v[8];
    #pragma unroll
                            for (int p = 0; p < 2; ++p) {
                                const uint2 w = *reinterpret_cast<const uint2*>(vs + p * C::VS_PAGE + t * C::VS_TILE + 8 * lane);
                                v[p * 4 + 0] = w.x & mask[p];
                                v[p * 4 + 1] = (w.x >> 16) & mask[p];
                                v[p * 4 + 2] = w.y & mask[p];
                                v[p * 4 + 3] = (w.y >> 16) & mask[p];
                            }
                            tc::tmem_st8(tq + C::T_SFV + ((j & 1) * MT + t) * 8, v);
                        }
                        tc::tmem_wait_st();
                    }
                }
                tc::tc_fence_before();
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&p_ready[j & 1]);
            }
        };
        if (any_bad_page) tiles(std::true_type{});
        else tiles(std::false_type{});
        if (!grp_abort) {
            if (!tc::mbar_wait(&o_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, kWaitLimitMla)) bad = true;
            tc::tc_fence_after();
        }

        // ------------------------------------------------------------ epilogue (thread = channel)
        grp_abort = tc::named_bar_or(bar_id, 128, grp_abort || bad || *abort_flag);
        if (grp_abort) *abort_flag = 1;
        if (!grp_abort) {
            float* rl = red;   // [GH][4] partial sums (the tile maxima are no longer read)
#pragma unroll
            for (int g = 0; g < HG; ++g) {
                float v = l_part[g];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) rl[(gb + g) * 4 + qd] = v;
            }
            tc::named_bar_sync(bar_id, 128);
            // O and l both carry the factor alpha (P^ is alpha p quantized), so it cancels
            const float oscale = FMT == BDFP4_NVFP4 ? a.v_gscale[hk] : 1.0f;
            // lane g: the output scale and (m, l) of head gb + g, through the warp's slots
            if (lane < HG) {
                const float4 r4 = *reinterpret_cast<const float4*>(rl + (gb + lane) * 4);
                const float l = r4.x + r4.y + r4.z + r4.w;
                // DYN: splits end in different units; the partials leave in the units of p
                const float un = DYN ? pow2f(-e_lane) : 1.0f;
                wout[lane] = nspl == 1 ? (l > 0.0f ? oscale / l : 0.0f) : oscale * un;
                if (nspl > 1 && qd == 0) {
                    const int64_t row = (int64_t)b * a.H_q + h0 + gb + lane;
                    a.ws_ml[(row * a.max_splits + split) * 2 + 0] = m_lane;
                    a.ws_ml[(row * a.max_splits + split) * 2 + 1] = l * un;
                }
            }
            __syncwarp();
#pragma unroll 1
            for (int t = 0; t < MT; ++t) {
                uint32_t ov[HG];
                tc::tmem_ld<HG>(tq + C::T_O + t * GH + gb, ov);
                tc::tmem_wait_ld();
                const int chan = t * 128 + 32 * qd + lane;
#pragma unroll
                for (int g = 0; g < HG; ++g) {
                    const int64_t row = (int64_t)b * a.H_q + h0 + gb + g;
                    const float o = __uint_as_float(ov[g]) * wout[g];
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
