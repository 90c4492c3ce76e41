// decode_bf16.cu -- the BF16-KV comparator of the FP4 decode: the same paged
// tiles, bulk copies, tcgen05 MMA with TMEM accumulators, transposed online
// softmax and split merge as decode_tc.cu, on bf16 K/V pages with bf16
// queries and probabilities and no quantization (the BF16 cache the pages
// measure against: "BitDecoding-FP4 tests native 4-bit attention for long
// contexts", Key Takeaways).
//
// One CTA per (sequence, KV head, split); warps 0 .. NSW-1 run the softmax
// (two groups split the query heads), warp NSW is the producer (bulk copies of
// 128-token tiles into a 3-stage ring of 64 KB stages), warp NSW+1 issues the
// MMAs: S^T = K_tile q^T (M = 128 tokens, N = 16 padded query rows, K = 128)
// and O^T = V^T P^T (M = 128 channels, N = 16, K = 64 per page).

#include <algorithm>

#include "../../include/bdfp4_bf16.h"
#include "bdfp4_device.cuh"
#include "decode_common.cuh"
#include "host_common.h"
#include "merge.cuh"
#include "tc_ptx.cuh"

namespace bdfp4 {

template <int G>
struct Bf16Cfg {
    static constexpr int D = 128;
    static constexpr int NQ = 16;                        // N of QK: query rows, padded
    static constexpr int NP = 16;                        // N of PV
    static constexpr int KS = D / 16;                    // MMA K steps of QK (16 bf16 each)
    static constexpr int NS = 3;                         // pipeline stages
    static constexpr int NSG = G >= 2 ? 2 : 1;           // softmax warpgroups (split the heads)
    static constexpr int HG = G / NSG;                   // heads per group
    static constexpr int NSW = 4 * NSG;                  // softmax warps
    static constexpr int PRODUCER = NSW, MMA_WARP = NSW + 1;
    static constexpr int THREADS = 32 * (NSW + 2);
    static constexpr int PAGE = kPageSlots * D * 2;      // 16 KB of K or V per (page, head)
    // a stage holds one 128-token tile: K of pages 0, 1 (MMA rows 0-63, 64-127), V of pages 0, 1
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = 2 * PAGE;
    static constexpr int STAGE = 4 * PAGE;
    static constexpr int Q_BYTES = NQ * D * 2;           // [row/8][elem/8][row%8][8 elements]
    static constexpr int P_PAGE = NP * kPageSlots * 2;   // [row/8][slot/8][row%8][8 slots] per page
    static constexpr int P_BUF = 2 * P_PAGE;
    // shared memory map
    static constexpr int SM_STAGES = 0;
    static constexpr int SM_Q = SM_STAGES + NS * STAGE;
    static constexpr int SM_P = SM_Q + Q_BYTES;
    static constexpr int SM_RED = SM_P + 2 * P_BUF;                      // [2][G][4] warp maxima (floats)
    static constexpr int SM_PAGES = SM_RED + 2 * G * 4 * 4;              // [NS][2] page ids
    static constexpr int SM_BARS = (SM_PAGES + NS * 2 * 4 + 7) / 8 * 8;
    static constexpr int NBARS = 2 * NS + 7;
    static constexpr int SM_MISC = SM_BARS + NBARS * 8;                  // tmem slot, abort flags
    static constexpr int SMEM = SM_MISC + 16;
    static_assert(SMEM <= 232448 - 1024, "shared memory");
    // TMEM columns: S^T double buffer, O^T double buffer
    static constexpr int T_S = 0;
    static constexpr int T_O = 2 * NQ;
    static constexpr int T_ALLOC = 64;
};

constexpr long long kBf16WaitLimit = 1LL << 32;   // clock cycles (about 2 s)

// ------------------------------------------------------------------ append
// One thread per (token, head, 8-element chunk): the keys' 16-byte chunk goes
// whole into the K page; the values' 8 channels go to 8 channel rows of the
// token-contiguous V^T page.
template <int D>
__global__ void __launch_bounds__(256) bf16_append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                          const int64_t* __restrict__ slot_mapping, int T, int H_kv,
                                                          uint8_t* k_pages, uint8_t* v_pages, int64_t num_pages,
                                                          int32_t* dev_status) {
    constexpr int CH = D / 8;
    constexpr int PAGE = kPageSlots * D * 2;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)T * H_kv * CH) return;
    const int c = (int)(idx % CH);
    const int64_t row = idx / CH;
    const int t = (int)(row / H_kv), h = (int)(row % H_kv);
    const int64_t sm = __ldg(slot_mapping + t);
    if (sm < 0) return;
    if (sm >= num_pages * kPageSlots) {
        if (c == 0) set_status(dev_status, BDFP4_DEV_BAD_SLOT);
        return;
    }
    const int64_t page = sm / kPageSlots;
    const int slot = (int)(sm % kPageSlots);
    const int64_t base = (page * H_kv + h) * (int64_t)PAGE;
    const uint4 kw = __ldg(k + idx);
    *reinterpret_cast<uint4*>(k_pages + base + (slot >> 3) * (D * 16) + c * 128 + (slot & 7) * 16) = kw;
    const uint4 vw = __ldg(v + idx);
    const uint32_t w[4] = {vw.x, vw.y, vw.z, vw.w};
    uint8_t* vp = v_pages + base + c * 1024 + (slot >> 3) * 128 + (slot & 7) * 2;
#pragma unroll
    for (int e = 0; e < 8; ++e)
        *reinterpret_cast<uint16_t*>(vp + e * 16) = (uint16_t)(e & 1 ? w[e >> 1] >> 16 : w[e >> 1] & 0xffffu);
}

struct Bf16Args {
    const __nv_bfloat16* q;
    const uint8_t* k_pages;
    const uint8_t* v_pages;
    const int32_t* block_table;
    const int32_t* seq_lens;
    float* ws_o;
    float* ws_ml;
    __nv_bfloat16* out;
    int32_t* dev_status;
    int B, H_q, H_kv, max_pages, chunk_tiles, max_splits;
    int64_t num_pages;
    float sm_scale;
};


// ------------------------------------------------------------------ decode
template <int G>
__global__ void __launch_bounds__(Bf16Cfg<G>::THREADS, 1) decode_bf16_kernel(const Bf16Args a) {
    using C = Bf16Cfg<G>;
    // the split merge (a programmatic dependent) may be scheduled as CTAs of this grid retire
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int HG = C::HG;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* q_op = smem + C::SM_Q;
    uint8_t* p_op = smem + C::SM_P;
    float* red = reinterpret_cast<float*>(smem + C::SM_RED);
    int* page_ids = reinterpret_cast<int*>(smem + C::SM_PAGES);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SM_BARS);
    uint64_t* full = bars;                    // [NS] producer -> consumers
    uint64_t* empty = bars + C::NS;           // [NS] PV done -> producer
    uint64_t* s_full = bars + 2 * C::NS;      // [2] QK done -> softmax
    uint64_t* p_ready = s_full + 2;           // [2] P written (and dead V columns zeroed) -> MMA
    uint64_t* o_full = p_ready + 2;           // [2] PV done -> softmax
    uint64_t* q_ready = o_full + 2;           // query operand written -> MMA
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SM_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SM_MISC + 4);   // any role gave up
    volatile int* sm_abort = reinterpret_cast<volatile int*>(smem + C::SM_MISC + 8);     // [NSG] group decisions

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int h0 = hk * G;

    int N = a.seq_lens[b];
    if (N < 0 || N > a.max_pages * kPageSlots) {
        if (tid == 0 && split == 0) set_status(a.dev_status, BDFP4_DEV_BAD_SEQLEN);
        N = 0;
    }
    const int ntiles = (N + kTileTokens - 1) / kTileTokens;
    const int nspl = (ntiles + a.chunk_tiles - 1) / a.chunk_tiles;
    if (split > 0 && split >= nspl) return;
    if (N == 0) {
        for (int i = tid; i < G * C::D; i += blockDim.x)
            a.out[((int64_t)b * a.H_q + h0 + i / C::D) * C::D + i % C::D] = __float2bfloat16(0.0f);
        return;
    }
    const int tile0 = split * a.chunk_tiles;
    const int n = min(a.chunk_tiles, ntiles - tile0);   // tiles of this split (>= 1)

    if (tid == 0) {
        for (int s = 0; s < C::NS; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&s_full[i], 1);
            tc::mbar_init(&p_ready[i], C::NSW);
            tc::mbar_init(&o_full[i], 1);
        }
        tc::mbar_init(q_ready, C::NSW);
        *abort_flag = 0;
        sm_abort[0] = 0;
        sm_abort[1] = 0;
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
        // Lanes read the page ids of 32 tiles at once; lane 0 then waits for a
        // free stage and issues four 16 KB bulk copies per tile.
        bool ok = true;
        for (int j0 = 0; ok && j0 < n; j0 += 32) {
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
            const int kmax = min(32, n - j0);
            for (int k = 0; k < kmax; ++k) {
                const int j = j0 + k;
                const int pg0 = __shfl_sync(0xffffffffu, pg_l[0], k);
                const int pg1 = __shfl_sync(0xffffffffu, pg_l[1], k);
                if (lane == 0) {
                    const int s = j % C::NS;
                    if (j >= C::NS && !tc::mbar_wait(&empty[s], ((j / C::NS) - 1) & 1, abort_flag, kBf16WaitLimit)) {
                        ok = false;
                    } else {
                        const int pg[2] = {pg0, pg1};
                        uint32_t bytes = 0;
#pragma unroll
                        for (int p = 0; p < 2; ++p) {
                            page_ids[s * 2 + p] = pg[p];
                            if (pg[p] >= 0) bytes += 2 * C::PAGE;
                        }
                        tc::mbar_arrive_expect_tx(&full[s], bytes);
                        uint8_t* st = smem + C::SM_STAGES + s * C::STAGE;
#pragma unroll
                        for (int p = 0; p < 2; ++p) {
                            if (pg[p] < 0) continue;
                            const int64_t ph = (int64_t)pg[p] * a.H_kv + hk;
                            tc::bulk_g2s(st + C::OFF_K + p * C::PAGE, a.k_pages + ph * C::PAGE, C::PAGE, &full[s]);
                            tc::bulk_g2s(st + C::OFF_V + p * C::PAGE, a.v_pages + ph * C::PAGE, C::PAGE, &full[s]);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        if (!ok && lane == 0) *abort_flag = 1;
    } else if (warp == C::MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = tc::idesc_bf16(C::NQ);
            constexpr uint32_t idesc_pv = tc::idesc_bf16(C::NP);
            const uint32_t q_addr = tc::smem_u32(q_op);
            const uint32_t p_addr = tc::smem_u32(p_op);
            const uint32_t st_addr = tc::smem_u32(smem + C::SM_STAGES);
            auto issue_qk = [&](int j) -> bool {
                const int s = j % C::NS, buf = j & 1;
                if (!tc::mbar_wait(&full[s], (j / C::NS) & 1, abort_flag, kBf16WaitLimit)) return false;
                tc::tc_fence_after();
                const uint32_t kt = st_addr + s * C::STAGE + C::OFF_K;
                // K tile rows: 8-row groups 2 KB apart (SBO), 8-element chunks 128 B apart (LBO)
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks)
                    tc::mma_bf16(tbase + C::T_S + buf * C::NQ, tc::smem_desc(kt + ks * 256, 128, C::D * 16),
                                 tc::smem_desc(q_addr + ks * 256, 128, C::D * 16), idesc_qk, ks > 0);
                tc::mma_commit(&s_full[buf]);
                return true;
            };
            bool ok = tc::mbar_wait(q_ready, 0, abort_flag, kBf16WaitLimit);
            if (ok) tc::tc_fence_after();
            ok = ok && issue_qk(0);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n && !(ok = issue_qk(j + 1))) break;
                const int s = j % C::NS, buf = j & 1;
                if (!(ok = tc::mbar_wait(&p_ready[buf], (j >> 1) & 1, abort_flag, kBf16WaitLimit))) break;
                tc::tc_fence_after();
                const uint32_t vt = st_addr + s * C::STAGE + C::OFF_V;
                // V^T page: 8-channel groups 1 KB apart, 8-slot chunks 128 B apart; P^T likewise
#pragma unroll
                for (int p = 0; p < 2; ++p) {
#pragma unroll
                    for (int ks = 0; ks < kPageSlots / 16; ++ks)
                        tc::mma_bf16(tbase + C::T_O + buf * C::NP, tc::smem_desc(vt + p * C::PAGE + ks * 256, 128, 1024),
                                     tc::smem_desc(p_addr + buf * C::P_BUF + p * C::P_PAGE + ks * 256, 128, 1024),
                                     idesc_pv, (p | ks) > 0);
                }
                tc::mma_commit(&o_full[buf]);
                tc::mma_commit(&empty[s]);
            }
            if (!ok) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int grp = warp >> 2;                 // head group
        const int qd = warp & 3;                   // TMEM lane quadrant = tokens 32 qd .. 32 qd + 31
        const int gb = grp * HG;                   // first head of the group
        const int bar_id = 1 + grp;                // named barrier of the group (128 threads)
        const uint32_t tq = tbase + ((uint32_t)(32 * qd) << 16);
        const float lsc = a.sm_scale * kLog2e;     // logits in log2 units
        bool bad = false;

        // query prologue: the G query rows (bf16, unchanged) into the QK operand, zero padding
        for (int i = tid; i < C::NQ * (C::D / 8); i += 32 * C::NSW) {
            const int row = i / (C::D / 8), c = i % (C::D / 8);
            uint4 w = make_uint4(0, 0, 0, 0);
            if (row < G) w = __ldg(reinterpret_cast<const uint4*>(a.q + ((int64_t)b * a.H_q + h0 + row) * C::D) + c);
            *reinterpret_cast<uint4*>(q_op + (row >> 3) * (C::D * 16) + c * 128 + (row & 7) * 16) = w;
        }
        // P rows of absent heads stay zero
        for (int i = tid; i < 2 * C::P_BUF / 16; i += 32 * C::NSW) reinterpret_cast<uint4*>(p_op)[i] = make_uint4(0, 0, 0, 0);
        tc::fence_proxy_async_smem();
        tc::named_bar_sync(1 + C::NSG, 32 * C::NSW);
        if (lane == 0) tc::mbar_arrive(q_ready);

        float m_run[HG], l_part[HG], o_acc[HG], corr_prev[HG];
#pragma unroll
        for (int g = 0; g < HG; ++g) {
            m_run[g] = -INFINITY;
            l_part[g] = 0.0f;
            o_acc[g] = 0.0f;
            corr_prev[g] = 0.0f;
        }
        // TMEM lane 32 qd + lane holds token 32 qd + lane of the tile: page qd / 2, slot 32 (qd % 2) + lane
        const int page_of_thread = qd >> 1;
        const int slot = 32 * (qd & 1) + lane;
        const int tok_in_tile = 32 * qd + lane;
        const int chan = 32 * qd + lane;   // O^T lane = value channel
        auto fold_o = [&](int j) -> bool {
            if (!tc::mbar_wait(&o_full[j & 1], (j >> 1) & 1, abort_flag, kBf16WaitLimit)) return false;
            tc::tc_fence_after();
            uint32_t ov[HG];
            tc::tmem_ld<HG>(tq + C::T_O + (j & 1) * C::NP + gb, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < HG; ++g) o_acc[g] = o_acc[g] * corr_prev[g] + __uint_as_float(ov[g]);
            return true;
        };
        uint8_t* const pslot = p_op + page_of_thread * C::P_PAGE + (slot >> 3) * 128 + (slot & 7) * 2;

        for (int j = 0; j < n; ++j) {
            const int s = j % C::NS, buf = j & 1, tile = tile0 + j;
            if (!tc::mbar_wait(&full[s], (j / C::NS) & 1, abort_flag, kBf16WaitLimit)) bad = true;
            if (!tc::mbar_wait(&s_full[buf], (j >> 1) & 1, abort_flag, kBf16WaitLimit)) bad = true;
            tc::tc_fence_after();
            uint32_t sr[HG];
            tc::tmem_ld<HG>(tq + C::T_S + buf * C::NQ + gb, sr);
            tc::tmem_wait_ld();
            const int token = tile * kTileTokens + tok_in_tile;
            const bool valid = token < N && page_ids[s * 2 + page_of_thread] >= 0;
            float t[HG];
            float* rw = red + buf * G * 4;   // [G][4] warp maxima
#pragma unroll
            for (int g = 0; g < HG; ++g) {
                t[g] = valid ? __uint_as_float(sr[g]) : -INFINITY;
                const float wm = tc::redux_max_f32(t[g], 0xffffffffu);
                if (lane == 0) rw[(gb + g) * 4 + qd] = wm;
            }
            // a token past the end (or on a page that was not loaded) gets a zero value
            // column, so whatever bits sit there meet a zero probability as 0, not NaN
            if (grp == 0 && !valid) {
                uint8_t* vcol = smem + C::SM_STAGES + s * C::STAGE + C::OFF_V + page_of_thread * C::PAGE +
                                (slot >> 3) * 128 + (slot & 7) * 2;
#pragma unroll 8
                for (int c = 0; c < C::D; ++c) *reinterpret_cast<uint16_t*>(vcol + (c >> 3) * 1024 + (c & 7) * 16) = 0;
            }
            if (bad || *abort_flag) sm_abort[grp] = 1;
            tc::named_bar_sync(bar_id, 128);
            if (sm_abort[grp]) break;
            float corr[HG];
            uint8_t* const pb = pslot + buf * C::P_BUF;
#pragma unroll
            for (int g = 0; g < HG; ++g) {
                const float4 w4 = *reinterpret_cast<const float4*>(rw + (gb + g) * 4);
                const float mt = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
                const float mn = fmaxf(m_run[g], mt * lsc);
                const float mz = mn == -INFINITY ? 0.0f : mn;
                corr[g] = tc::ex2_approx(m_run[g] - mz);   // 0 on the split's first tile
                m_run[g] = mn;
                const float p = tc::ex2_approx(fmaf(t[g], lsc, -mz));   // 0 for masked tokens
                l_part[g] = fmaf(l_part[g], corr[g], p);
                const int hr = gb + g;
                *reinterpret_cast<__nv_bfloat16*>(pb + (hr >> 3) * 1024 + (hr & 7) * 16) = __float2bfloat16_rn(p);
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&p_ready[buf]);
            if (j >= 1) bad |= !fold_o(j - 1);
#pragma unroll
            for (int g = 0; g < HG; ++g) corr_prev[g] = corr[g];
        }
        if (!sm_abort[grp] && !fold_o(n - 1)) bad = true;
        if (bad || *abort_flag) sm_abort[grp] = 1;

        // ------------------------------------------------------------ epilogue (thread = channel)
        tc::named_bar_sync(bar_id, 128);
        if (sm_abort[grp]) *abort_flag = 1;
        if (!sm_abort[grp]) {
            float* rl = red;   // [G][8] partial sums (the tile maxima are no longer read)
#pragma unroll
            for (int g = 0; g < HG; ++g) {
                float v = l_part[g];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) rl[(gb + g) * 8 + qd] = v;
            }
            tc::named_bar_sync(bar_id, 128);
#pragma unroll
            for (int g = 0; g < HG; ++g) {
                const int hh = gb + g;
                const float l = rl[hh * 8] + rl[hh * 8 + 1] + rl[hh * 8 + 2] + rl[hh * 8 + 3];
                const int64_t row = (int64_t)b * a.H_q + h0 + hh;
                if (nspl == 1) {
                    a.out[row * C::D + chan] = __float2bfloat16(l > 0.0f ? o_acc[g] / l : 0.0f);
                } else {
                    a.ws_o[(row * a.max_splits + split) * C::D + chan] = o_acc[g];
                    if (chan == 0) {
                        a.ws_ml[(row * a.max_splits + split) * 2 + 0] = m_run[g];
                        a.ws_ml[(row * a.max_splits + split) * 2 + 1] = l;
                    }
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

template <int G>
static int launch_bf16(const Bf16Args& a, cudaStream_t st) {
    using C = Bf16Cfg<G>;
    static bool attr_set = false;
    if (!attr_set) {
        const cudaError_t e =
            cudaFuncSetAttribute(decode_bf16_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) {
            record_cuda_error(e);
            return BDFP4_ERR_CUDA;
        }
        attr_set = true;
    }
    dim3 grid(a.max_splits, a.H_kv, a.B);
    decode_bf16_kernel<G><<<grid, C::THREADS, C::SMEM, st>>>(a);
    const int rc = launch_status();
    if (rc != BDFP4_OK || a.max_splits <= 1) return rc;
    const cudaError_t e = launch_merge<C::D>(a.ws_o, a.ws_ml, a.seq_lens, a.B, a.H_q, a.max_pages, a.chunk_tiles,
                                             a.max_splits, a.out, st);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return BDFP4_ERR_CUDA;
    }
    return launch_status();
}

}  // namespace bdfp4

using namespace bdfp4;

extern "C" int bdfp4_bf16_append(const void* k, const void* v, const int64_t* slot_mapping, int T, int H_kv, int d,
                                 void* k_pages, void* v_pages, int64_t num_pages, int32_t* dev_status, void* stream) {
    if (T < 0 || H_kv <= 0 || num_pages < 0) return BDFP4_ERR_ARG;
    if (d != 128) return BDFP4_ERR_UNSUPPORTED;
    if (T == 0) return BDFP4_OK;
    if (!k || !v || !slot_mapping || !k_pages || !v_pages) return BDFP4_ERR_ARG;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_pages, 128) || !aligned(v_pages, 128)) return BDFP4_ERR_ALIGN;
    const int64_t threads = (int64_t)T * H_kv * (128 / 8);
    bf16_append_kernel<128><<<(unsigned)((threads + 255) / 256), 256, 0, (cudaStream_t)stream>>>(
        (const uint4*)k, (const uint4*)v, slot_mapping, T, H_kv, (uint8_t*)k_pages, (uint8_t*)v_pages, num_pages,
        dev_status);
    return launch_status();
}

extern "C" int bdfp4_bf16_decode(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                                 const int32_t* seq_lens, int B, int H_q, int H_kv, int d, int max_pages_per_seq,
                                 int64_t num_pages, float sm_scale, int chunk_tiles, void* workspace,
                                 size_t workspace_bytes, void* out, int32_t* dev_status, void* stream) {
    if (B < 0 || H_q <= 0 || H_kv <= 0 || max_pages_per_seq <= 0 || num_pages < 0) return BDFP4_ERR_ARG;
    if (H_q % H_kv) return BDFP4_ERR_SHAPE;
    const int G = H_q / H_kv;
    if (d != 128 || G > 16 || (G & (G - 1)) != 0) return BDFP4_ERR_UNSUPPORTED;
    if (B == 0) return BDFP4_OK;
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !out) return BDFP4_ERR_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_pages, 128) || !aligned(v_pages, 128))
        return BDFP4_ERR_ALIGN;
    if (chunk_tiles <= 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BDFP4_ERR_CUDA;
        const int ntiles = (max_pages_per_seq * kPageSlots + kTileTokens - 1) / kTileTokens;
        chunk_tiles = plan_chunk_tiles(B, [&](int) { return ntiles; }, H_kv, sms, 1);   // one CTA per SM
    }
    Bf16Args a{};
    const int ntiles_max = (max_pages_per_seq * kPageSlots + kTileTokens - 1) / kTileTokens;
    a.max_splits = std::max(1, (ntiles_max + chunk_tiles - 1) / chunk_tiles);
    if (a.max_splits > 1) {
        const size_t need = bdfp4_decode_workspace_size(B, H_q, d, max_pages_per_seq, chunk_tiles);
        if (!workspace || workspace_bytes < need) return BDFP4_ERR_WORKSPACE;
        if (!aligned(workspace, 128)) return BDFP4_ERR_ALIGN;
        const size_t o_bytes = (size_t)B * H_q * a.max_splits * d * sizeof(float);
        a.ws_o = (float*)workspace;
        a.ws_ml = (float*)((char*)workspace + ((o_bytes + 255) / 256) * 256);
    }
    a.q = (const __nv_bfloat16*)q;
    a.k_pages = (const uint8_t*)k_pages;
    a.v_pages = (const uint8_t*)v_pages;
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.out = (__nv_bfloat16*)out;
    a.dev_status = dev_status;
    a.B = B;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.max_pages = max_pages_per_seq;
    a.num_pages = num_pages;
    a.chunk_tiles = chunk_tiles;
    a.sm_scale = sm_scale;
    cudaStream_t st = (cudaStream_t)stream;
    switch (G) {
        case 1: return launch_bf16<1>(a, st);
        case 2: return launch_bf16<2>(a, st);
        case 4: return launch_bf16<4>(a, st);
        case 8: return launch_bf16<8>(a, st);
        case 16: return launch_bf16<16>(a, st);
    }
    return BDFP4_ERR_UNSUPPORTED;
}
