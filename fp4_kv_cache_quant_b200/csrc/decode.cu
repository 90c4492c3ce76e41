// decode.cu -- FP4 paged decode attention with split-KV and a log-sum-exp
// merge (BitDecoding-FP4, Article Summary: dual-residual query, transposed
// softmax with fused, underflow-aware probability quantization, paged KV).
//
// One CTA of 128 threads per (sequence, KV head, head chunk, split).  The
// softmax is transposed: thread t owns token t of the current 128-token tile
// (two pages) for every query head of the group, so row maxima and sums are
// warp-shuffle reductions, and the FP4 quantization of the probabilities
// (beta-token blocks) is a 4- or 5-step shuffle max inside the owning lanes.
// For P.V the threads switch to owning value channels, reading each page's
// channel-major FP4 block with 16-byte loads.

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "../../include/bdfp4_debug.h"
#include "bdfp4_device.cuh"
#include "host_common.h"
#include "quant_device.cuh"
#include "decode_common.cuh"
#include "merge.cuh"
#include "prob_scale.cuh"

namespace bdfp4 {

template <int FMT, int DK, int DV, int HG>
__global__ void __launch_bounds__(kThreads) decode_fp4_kernel(const DecodeArgs a) {
    // the split merge (a programmatic dependent) may be scheduled as CTAs of this grid retire
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int B = Fmt<FMT>::beta;
    constexpr int NCH = DV / kThreads;   // value channels per thread
    using RG = RowGeom<FMT, DK>;

    __shared__ __align__(16) float dq[HG][DK];            // dequantized q1 + q2 (scale values, no g)
    __shared__ __align__(16) float ph[HG][kTileTokens];   // quantized probabilities (times alpha)
    __shared__ float2 lut[256];                            // E2M1 byte -> (low, high) values
    __shared__ float red[4][HG];
    __shared__ float lsc[HG];                              // sm_scale g_q g_k log2(e)
    __shared__ int row_amax[kThreads];
    __shared__ int pages[2];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x;
    // the rows of a (sequence, KV head): the group's G query heads, for each of the T_q
    // query tokens (token-major, stacked_row); this CTA takes HG of them from v0
    const int G = a.H_q / a.H_kv, T = a.T_q;
    const int chunks = G * T / HG;
    const int hk = blockIdx.y / chunks;
    const int v0 = (blockIdx.y % chunks) * HG;
    const int b = blockIdx.z;
    auto row_of = [&](int r) -> int64_t { return stacked_row(a, b, hk, v0 + r); };

    int N = a.seq_lens[b];
    if (N < 0 || N > a.max_pages * kPageSlots) {
        if (tid == 0 && split == 0) set_status(a.dev_status, BDFP4_DEV_BAD_SEQLEN);
        N = 0;
    }
    // several query tokens: the sequence must hold them (rows that see no token give zeros)
    if (T > 1 && N > 0 && N < T && tid == 0 && split == 0 && blockIdx.y == 0)
        set_status(a.dev_status, BDFP4_DEV_BAD_SEQLEN);
    const int ntiles = (N + kTileTokens - 1) / kTileTokens;
    const int nspl = (ntiles + a.chunk_tiles - 1) / a.chunk_tiles;
    if (split > 0 && split >= nspl) return;
    if (N == 0) {  // empty sequence: zeros
        for (int i = tid; i < HG * DV; i += kThreads) a.out[row_of(i / DV) * DV + i % DV] = __float2bfloat16(0.0f);
        return;
    }

    // ---------------------------------------------------------------- prologue
    for (uint32_t by = tid; by < 256u; by += kThreads) lut[by] = make_float2(e2m1_value(by & 15u), e2m1_value(by >> 4));
    const bool hadamard = !(a.flags & BDFP4_FLAG_NO_HADAMARD);
    const bool dual = !(a.flags & BDFP4_FLAG_SINGLE_QUERY);
    constexpr int rows_per_pass = kThreads / RG::rt;
    for (int r0 = 0; r0 < HG; r0 += rows_per_pass) {
        const int j = tid % RG::rt, rl = tid / RG::rt, r = r0 + rl;
        const bool active = r < HG && j < RG::tpr;
        row_amax[tid] = 0;
        float x[B];
        if (active) {
            load_bf16_block<B>(a.q + row_of(r) * DK, j * B, x);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i) x[i] = 0.0f;
        }
        transform_block<FMT, DK, false>(x, a.smooth + (int64_t)hk * DK, j, hadamard);
        __syncthreads();
        if (active) atomicMax(&row_amax[rl], __float_as_int(block_amax<B>(x)));
        __syncthreads();
        if (active) {
            const float amax = __int_as_float(row_amax[rl]);
            const float gq = FMT == BDFP4_NVFP4 ? (amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f) : 1.0f;
            uint32_t c1, c2, p1[B / 8], p2[B / 8];
            quantize_query_block<FMT, DK>(x, gq, dual, c1, p1, c2, p2);
            const float s1 = scale_value<FMT>(c1), s2 = scale_value<FMT>(c2);
#pragma unroll
            for (int i = 0; i < B; ++i) {
                const uint32_t e1 = (p1[i / 8] >> (4 * (i % 8))) & 15u, e2 = (p2[i / 8] >> (4 * (i % 8))) & 15u;
                dq[r][j * B + i] = e2m1_value(e1) * s1 + e2m1_value(e2) * s2;
            }
            if (j == 0) {
                const float gk = FMT == BDFP4_NVFP4 ? a.k_gscale[hk] : 1.0f;
                lsc[r] = a.sm_scale * gq * gk * kLog2e;
            }
        }
        __syncthreads();
    }

    const float alpha = (FMT == BDFP4_NVFP4 && !(a.flags & BDFP4_FLAG_NO_UNDERFLOW)) ? kAlphaNV : 1.0f;
    // dynamic variant: each tile's alpha is divided out of its probabilities
    const bool dyn = FMT == BDFP4_NVFP4 && (a.flags & BDFP4_FLAG_DYNAMIC_ALPHA);
    const float vg = FMT == BDFP4_NVFP4 ? a.v_gscale[hk] : 1.0f;
    const int64_t kv_stride_k = (int64_t)kPageSlots * DK / 2, kv_stride_ks = k_scale_page_bytes(DK, B);
    const int64_t kv_stride_v = (int64_t)DV * kPageSlots / 2, kv_stride_vs = (int64_t)DV * kPageSlots / B;

    float m_run[HG], l_part[HG], o[HG][NCH];
#pragma unroll
    for (int g = 0; g < HG; ++g) {
        m_run[g] = -INFINITY;
        l_part[g] = 0.0f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) o[g][c] = 0.0f;
    }

    const int tile0 = split * a.chunk_tiles;
    const int tile1 = min(tile0 + a.chunk_tiles, ntiles);
    for (int tile = tile0; tile < tile1; ++tile) {
        // ------------------------------------------------ logits (thread = token)
        const int token = tile * kTileTokens + tid;
        bool valid = token < N;
        float s[HG];
#pragma unroll
        for (int g = 0; g < HG; ++g) s[g] = -INFINITY;
        if (tid < 2) {
            int pg = -1;
            const int pi = tile * 2 + tid;
            if (pi * kPageSlots < N) {
                pg = a.block_table[(int64_t)b * a.max_pages + pi];
                if (pg < 0 || pg >= a.num_pages) {
                    set_status(a.dev_status, BDFP4_DEV_BAD_PAGE);
                    pg = -1;
                }
            }
            pages[tid] = pg;
        }
        __syncthreads();
        const int page = pages[tid >> 6];
        valid = valid && page >= 0;
        if (valid) {
            const int slot = tid & 63;
            const uint8_t* kp = a.k_pages + ((int64_t)page * a.H_kv + hk) * kv_stride_k;
            const uint8_t* ks = a.k_scales + ((int64_t)page * a.H_kv + hk) * kv_stride_ks;
            float acc[HG];
#pragma unroll
            for (int g = 0; g < HG; ++g) acc[g] = 0.0f;
#pragma unroll 2
            for (int kc = 0; kc < DK / 32; ++kc) {
                const uint4 w = __ldg(reinterpret_cast<const uint4*>(kp + k_nib_offset(DK, slot, kc * 32)));
                const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int half = 0; half < 32 / B; ++half) {
                    const int blk = (kc * 32) / B + half;
                    const float sc = scale_value<FMT>(__ldg(ks + k_scale_offset<B>(DK, slot, blk)));
#pragma unroll
                    for (int wi = 0; wi < B / 8; ++wi) {
                        const uint32_t word = words[half * (B / 8) + wi];
#pragma unroll
                        for (int by = 0; by < 4; ++by) {
                            const float2 v2 = lut[(word >> (8 * by)) & 0xffu];
                            const int e = kc * 32 + half * B + wi * 8 + by * 2;
                            const float k0 = v2.x * sc, k1 = v2.y * sc;
#pragma unroll
                            for (int g = 0; g < HG; ++g) {
                                const float2 qq = *reinterpret_cast<const float2*>(&dq[g][e]);
                                acc[g] = fmaf(qq.x, k0, acc[g]);
                                acc[g] = fmaf(qq.y, k1, acc[g]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < HG; ++g) s[g] = acc[g] * lsc[g];
            // query token i of the stacked row sees the first N - T + 1 + i tokens
            if (T > 1) {
#pragma unroll
                for (int g = 0; g < HG; ++g)
                    if (token >= N - T + 1 + (v0 + g) / G) s[g] = -INFINITY;
            }
        }
        // ------------------------------------------------ transposed online softmax
        float p[HG], corr[HG];
#pragma unroll
        for (int g = 0; g < HG; ++g) {
            float mx = s[g];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            if (lane == 0) red[warp][g] = mx;
        }
        __syncthreads();
#pragma unroll
        for (int g = 0; g < HG; ++g) {
            const float mt = fmaxf(fmaxf(red[0][g], red[1][g]), fmaxf(red[2][g], red[3][g]));
            const float mn = fmaxf(m_run[g], mt);
            // a split whose tiles so far hold only masked tokens (bad pages) keeps m = -inf:
            // take 0 as the reference there, so corr and p are 0 rather than NaN
            const float mz = mn == -INFINITY ? 0.0f : mn;
            corr[g] = exp2f(m_run[g] - mz);   // 0 on the split's first tile
            m_run[g] = mn;
            p[g] = valid && s[g] != -INFINITY ? exp2f(s[g] - mz) : 0.0f;
            l_part[g] = l_part[g] * corr[g] + p[g];
            float ag = alpha, ig = 1.0f;
            if (dyn) {
                const int E = dynamic_alpha_exp(exp2f(mt - mz));   // the tile's largest p
                ag = pow2f(E);
                ig = pow2f(-E);
            }
            // fused probability quantization over beta-token blocks of lanes
            const float y = p[g] * ag;
            float am = y;
#pragma unroll
            for (int off = B / 2; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
            float sigma;
            if constexpr (FMT == BDFP4_NVFP4) {
                sigma = am > 0.0f ? e4m3_value(e4m3_encode(__fdiv_rn(am, 6.0f))) : 0.0f;
            } else {
                sigma = e8m0_value(mx_scale_code(am));
            }
            const uint32_t e = sigma > 0.0f ? e2m1_encode(__fdiv_rn(y, sigma)) : 0u;
            ph[g][tid] = e2m1_value(e) * sigma * ig;
        }
        __syncthreads();
        // ------------------------------------------------ P.V (thread = value channel)
#pragma unroll
        for (int g = 0; g < HG; ++g)
#pragma unroll
            for (int c = 0; c < NCH; ++c) o[g][c] *= corr[g];
        const int n_valid = min(kTileTokens, N - tile * kTileTokens);
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
            const int pg = pages[pp];
            const int nv = min(kPageSlots, n_valid - pp * kPageSlots);
            if (pg < 0 || nv <= 0) continue;
            const uint8_t* vp = a.v_pages + ((int64_t)pg * a.H_kv + hk) * kv_stride_v;
            const uint8_t* vs = a.v_scales + ((int64_t)pg * a.H_kv + hk) * kv_stride_vs;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int ch = tid + c * kThreads;
#pragma unroll
                for (int kc = 0; kc < 2; ++kc) {
                    const uint4 w = __ldg(reinterpret_cast<const uint4*>(vp + v_nib_offset(ch, kc * 32)));
                    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
                        for (int by = 0; by < 4; ++by) {
                            const int sl = kc * 32 + wi * 8 + by * 2;   // slot of the low nibble
                            if (sl >= nv) continue;                      // masked slots: select, never multiply
                            const float sc = scale_value<FMT>(__ldg(vs + v_scale_offset<B>(ch, sl / B)));
                            const float2 v2 = lut[(words[wi] >> (8 * by)) & 0xffu];
                            const float v0 = v2.x * sc;
                            const float v1 = (sl + 1 < nv) ? v2.y * sc : 0.0f;
                            const int tt = pp * kPageSlots + sl;
#pragma unroll
                            for (int g = 0; g < HG; ++g) {
                                const float2 pq = *reinterpret_cast<const float2*>(&ph[g][tt]);
                                o[g][c] = fmaf(pq.x, v0, o[g][c]);
                                o[g][c] = fmaf(pq.y, v1, o[g][c]);
                            }
                        }
                    }
                }
            }
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- epilogue
    // l = sum over the tile threads of their partial sums (warp shuffle + smem)
    __shared__ float lsum[4][HG];
#pragma unroll
    for (int g = 0; g < HG; ++g) {
        float v = l_part[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) lsum[warp][g] = v;
    }
    __syncthreads();
    const float oscale = dyn ? vg : vg / alpha;
    const bool single = nspl == 1;
#pragma unroll
    for (int g = 0; g < HG; ++g) {
        const float l = lsum[0][g] + lsum[1][g] + lsum[2][g] + lsum[3][g];
        const int64_t row = row_of(g);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int ch = tid + c * kThreads;
            if (single) {
                a.out[row * DV + ch] = __float2bfloat16(l > 0.0f ? o[g][c] * oscale / l : 0.0f);
            } else {
                a.ws_o[(row * a.max_splits + split) * DV + ch] = o[g][c] * oscale;
            }
        }
        if (!single && tid == 0) {
            a.ws_ml[(row * a.max_splits + split) * 2 + 0] = m_run[g];
            a.ws_ml[(row * a.max_splits + split) * 2 + 1] = l;
        }
    }
}

}  // namespace bdfp4

using namespace bdfp4;


static int max_splits_for(int max_pages, int chunk_tiles) {
    const int ntiles = (max_pages * kPageSlots + kTileTokens - 1) / kTileTokens;
    return std::max(1, (ntiles + chunk_tiles - 1) / chunk_tiles);
}

// Workspace regions: split partials (fp32 O, then (m, l)) when a sequence can
// have more than one split, then the query images of the tensor-core path
// (at most kQueryImageBytes per query head: 592 at d_k = 128, 652 for MLA).

struct WorkspaceMap {
    size_t o_bytes, ml_bytes, q_off, total;
};

static WorkspaceMap workspace_map(int B, int H_q, int d_v, int max_splits) {
    WorkspaceMap m{};
    const size_t ms = max_splits > 1 ? (size_t)max_splits : 0;
    m.o_bytes = (size_t)B * H_q * ms * d_v * sizeof(float);
    m.ml_bytes = (size_t)B * H_q * ms * 2 * sizeof(float);
    m.q_off = ((m.o_bytes + 255) / 256) * 256 + ((m.ml_bytes + 255) / 256) * 256;
    m.total = m.q_off + (size_t)B * H_q * (size_t)kQueryImageBytes;
    return m;
}

extern "C" size_t bdfp4_decode_workspace_size(int B, int H_q, int d_v, int max_pages_per_seq, int chunk_tiles) {
    if (B <= 0 || H_q <= 0 || d_v <= 0 || max_pages_per_seq <= 0 || chunk_tiles <= 0) return 0;
    return workspace_map(B, H_q, d_v, max_splits_for(max_pages_per_seq, chunk_tiles)).total;
}

static int host_tiles(const int32_t* host_seq_lens, int b) {
    return ((host_seq_lens[b] > 0 ? host_seq_lens[b] : 0) + kTileTokens - 1) / kTileTokens;
}

extern "C" int bdfp4_decode_plan(const int32_t* host_seq_lens, int B, int H_kv, int num_sms) {
    if (!host_seq_lens || B <= 0 || H_kv <= 0 || num_sms <= 0) return BDFP4_ERR_ARG;
    return plan_chunk_tiles(B, [&](int b) { return host_tiles(host_seq_lens, b); }, H_kv, num_sms, 4);
}

extern "C" int bdfp4_decode_plan_for(const int32_t* host_seq_lens, int B, int H_q, int H_kv, int d_k, int d_v,
                                     int num_sms) {
    return bdfp4_decode_multi_plan(host_seq_lens, B, 1, H_q, H_kv, d_k, d_v, num_sms);
}

extern "C" int bdfp4_decode_multi_plan(const int32_t* host_seq_lens, int B, int T_q, int H_q, int H_kv, int d_k,
                                       int d_v, int num_sms) {
    if (!host_seq_lens || B <= 0 || T_q <= 0 || H_q <= 0 || H_kv <= 0 || num_sms <= 0) return BDFP4_ERR_ARG;
    if (H_q % H_kv) return BDFP4_ERR_SHAPE;
    if (!supported_dims(d_k, d_v)) return BDFP4_ERR_UNSUPPORTED;
    const DecodeShape ks = decode_shape(d_k, d_v, H_q / H_kv, T_q);
    return plan_chunk_tiles(B, [&](int b) { return host_tiles(host_seq_lens, b); }, H_kv * ks.items_per_kv_head,
                            num_sms, ks.ctas_per_sm);
}

// The split merge after a decode grid (nothing when no sequence can split).  Its
// rows are the [B][T_q][H_q] output rows; a sequence's T_q H_q rows share its length.
template <int DV>
static int merge_splits(const DecodeArgs& a, cudaStream_t st) {
    const int rc = launch_status();
    if (rc != BDFP4_OK || a.max_splits <= 1) return rc;
    const cudaError_t e = launch_merge<DV>(a.ws_o, a.ws_ml, a.seq_lens, a.B, a.H_q * a.T_q, a.max_pages,
                                           a.chunk_tiles, a.max_splits, a.out, st);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return BDFP4_ERR_CUDA;
    }
    return launch_status();
}

template <int FMT, int DK, int DV>
static int launch_decode(const DecodeArgs& a, int G, cudaStream_t st, const StepArgs* step) {
    const DecodePath path = decode_path(DK, DV, G, a.T_q);
    if (path == DecodePath::kTensorCore128) {
        // tensor-core path (decode_tc.cu) on the G T_q stacked rows; a step's append runs in
        // its prologue grid
        const int rc = launch_decode_tc(a, FMT, G * a.T_q, st, step);
        if (rc != BDFP4_OK) return rc;
        return merge_splits<DV>(a, st);
    }
    if (path == DecodePath::kTensorCoreMla) {
        // tensor-core path for MLA shapes (decode_mla_tc.cu); a step's append runs in its prologue grid
        const int rc = launch_decode_mla_tc(a, FMT, G, st, step);
        if (rc != BDFP4_OK) return rc;
        return merge_splits<DV>(a, st);
    }
    if (step) {
        const int rc = launch_step_append(a, *step, FMT, DK, st);
        if (rc != BDFP4_OK) return rc;
    }
    const int rows = G * a.T_q, hg = cuda_core_rows(rows);
    dim3 grid(a.max_splits, a.H_kv * (rows / hg), a.B);
    switch (hg) {
        case 1: decode_fp4_kernel<FMT, DK, DV, 1><<<grid, kThreads, 0, st>>>(a); break;
        case 2: decode_fp4_kernel<FMT, DK, DV, 2><<<grid, kThreads, 0, st>>>(a); break;
        case 4: decode_fp4_kernel<FMT, DK, DV, 4><<<grid, kThreads, 0, st>>>(a); break;
        case 8: decode_fp4_kernel<FMT, DK, DV, 8><<<grid, kThreads, 0, st>>>(a); break;
        case 16: decode_fp4_kernel<FMT, DK, DV, 16><<<grid, kThreads, 0, st>>>(a); break;
        default: return BDFP4_ERR_UNSUPPORTED;
    }
    return merge_splits<DV>(a, st);
}

static int run_decode(const void* q, const void* k_pages, const void* k_scales, const void* v_pages,
                      const void* v_scales, const int32_t* block_table, const int32_t* seq_lens, int B, int T_q,
                      int H_q, int H_kv, int d_k, int d_v, int max_pages_per_seq, int64_t num_pages, bdfp4_fmt fmt,
                      int flags, const bdfp4_kv_params* kv, float sm_scale, int chunk_tiles, void* workspace,
                      size_t workspace_bytes, void* out, int32_t* dev_status, void* stream, StepArgs* step,
                      long long wait_limit = kWaitLimitDefault, int test_stall = 0) {
    if (B < 0 || T_q <= 0 || H_q <= 0 || H_kv <= 0 || max_pages_per_seq <= 0 || num_pages < 0) return BDFP4_ERR_ARG;
    if (fmt != BDFP4_NVFP4 && fmt != BDFP4_MXFP4) return BDFP4_ERR_ARG;
    if (H_q % H_kv) return BDFP4_ERR_SHAPE;
    if (!supported_dims(d_k, d_v)) return BDFP4_ERR_UNSUPPORTED;
    const int G = H_q / H_kv;
    if (G > 16 ? (G % 16 != 0 || G > 128) : (G & (G - 1)) != 0) return BDFP4_ERR_UNSUPPORTED;
    if ((int64_t)G * T_q > 4096) return BDFP4_ERR_UNSUPPORTED;
    if (B == 0) return BDFP4_OK;
    if (!q || !k_pages || !k_scales || !v_pages || !v_scales || !block_table || !seq_lens || !out || !kv ||
        !kv->smooth)
        return BDFP4_ERR_ARG;
    if (fmt == BDFP4_NVFP4 && (!kv->k_gscale || !kv->v_gscale)) return BDFP4_ERR_ARG;
    if ((flags & BDFP4_FLAG_DYNAMIC_ALPHA) && (flags & BDFP4_FLAG_NO_UNDERFLOW)) return BDFP4_ERR_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_pages, 128) || !aligned(k_scales, 128) ||
        !aligned(v_pages, 128) || !aligned(v_scales, 128))
        return BDFP4_ERR_ALIGN;
    if (chunk_tiles <= 0) {
        // no host sequence lengths: plan for the longest possible sequence
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BDFP4_ERR_CUDA;
        const int ntiles = (max_pages_per_seq * kPageSlots + kTileTokens - 1) / kTileTokens;
        const DecodeShape ks = decode_shape(d_k, d_v, G, T_q);
        chunk_tiles = plan_chunk_tiles(B, [&](int) { return ntiles; }, H_kv * ks.items_per_kv_head, sms,
                                       ks.ctas_per_sm);
    }
    DecodeArgs a{};
    a.max_splits = max_splits_for(max_pages_per_seq, chunk_tiles);
    const bool tensor_core_path = decode_path(d_k, d_v, G, T_q) != DecodePath::kCudaCore;
    if (a.max_splits > 1 || tensor_core_path) {
        const WorkspaceMap m = workspace_map(B * T_q, H_q, d_v, a.max_splits);
        if (!workspace || workspace_bytes < m.total) return BDFP4_ERR_WORKSPACE;
        if (!aligned(workspace, 128)) return BDFP4_ERR_ALIGN;
        a.ws_o = (float*)workspace;
        a.ws_ml = (float*)((char*)workspace + ((m.o_bytes + 255) / 256) * 256);
        a.qpack = (uint8_t*)workspace + m.q_off;
    }
    a.q = (const __nv_bfloat16*)q;
    a.k_pages = (const uint8_t*)k_pages;
    a.k_scales = (const uint8_t*)k_scales;
    a.v_pages = (const uint8_t*)v_pages;
    a.v_scales = (const uint8_t*)v_scales;
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.smooth = kv->smooth;
    a.k_gscale = kv->k_gscale;
    a.v_gscale = kv->v_gscale;
    a.k_weight = kv->k_weight;
    a.out = (__nv_bfloat16*)out;
    a.dev_status = dev_status;
    a.B = B;
    a.T_q = T_q;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.max_pages = max_pages_per_seq;
    a.num_pages = num_pages;
    a.flags = flags;
    a.chunk_tiles = chunk_tiles;
    a.sm_scale = sm_scale;
    a.append_wait = step != nullptr;
    a.wait_limit = wait_limit;
    a.test_stall = test_stall;
    if (step) {
        step->k_pages = (uint8_t*)k_pages;
        step->k_scales = (uint8_t*)k_scales;
        step->v_pages = (uint8_t*)v_pages;
        step->v_scales = (uint8_t*)v_scales;
    }
    cudaStream_t st = (cudaStream_t)stream;
    if (fmt == BDFP4_NVFP4)
        return d_k == 128 ? launch_decode<BDFP4_NVFP4, 128, 128>(a, G, st, step)
                          : launch_decode<BDFP4_NVFP4, 576, 512>(a, G, st, step);
    return d_k == 128 ? launch_decode<BDFP4_MXFP4, 128, 128>(a, G, st, step)
                      : launch_decode<BDFP4_MXFP4, 576, 512>(a, G, st, step);
}

extern "C" int bdfp4_decode(const void* q, const void* k_pages, const void* k_scales, const void* v_pages,
                            const void* v_scales, const int32_t* block_table, const int32_t* seq_lens, int B, int H_q,
                            int H_kv, int d_k, int d_v, int max_pages_per_seq, int64_t num_pages, bdfp4_fmt fmt,
                            int flags, const bdfp4_kv_params* kv, float sm_scale, int chunk_tiles, void* workspace,
                            size_t workspace_bytes, void* out, int32_t* dev_status, void* stream) {
    return run_decode(q, k_pages, k_scales, v_pages, v_scales, block_table, seq_lens, B, 1, H_q, H_kv, d_k, d_v,
                      max_pages_per_seq, num_pages, fmt, flags, kv, sm_scale, chunk_tiles, workspace,
                      workspace_bytes, out, dev_status, stream, nullptr);
}

extern "C" int bdfp4_decode_step(const void* q, const void* k_new, const void* v_new, void* v_open, void* k_pages,
                                 void* k_scales, void* v_pages, void* v_scales, const int32_t* block_table,
                                 const int32_t* seq_lens, int B, int H_q, int H_kv, int d_k, int d_v,
                                 int max_pages_per_seq, int64_t num_pages, bdfp4_fmt fmt, int flags,
                                 const bdfp4_kv_params* kv, float sm_scale, int chunk_tiles, void* workspace,
                                 size_t workspace_bytes, void* out, int32_t* dev_status, void* stream) {
    if (B > 0 && (!k_new || !v_new || !v_open)) return BDFP4_ERR_ARG;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(v_open, 16)) return BDFP4_ERR_ALIGN;
    StepArgs s{};
    s.k_new = (const __nv_bfloat16*)k_new;
    s.v_new = (const __nv_bfloat16*)v_new;
    s.v_open = (__nv_bfloat16*)v_open;
    return run_decode(q, k_pages, k_scales, v_pages, v_scales, block_table, seq_lens, B, 1, H_q, H_kv, d_k, d_v,
                      max_pages_per_seq, num_pages, fmt, flags, kv, sm_scale, chunk_tiles, workspace,
                      workspace_bytes, out, dev_status, stream, &s);
}

extern "C" int bdfp4_decode_multi(const void* q, const void* k_pages, const void* k_scales, const void* v_pages,
                                  const void* v_scales, const int32_t* block_table, const int32_t* seq_lens, int B,
                                  int T_q, int H_q, int H_kv, int d_k, int d_v, int max_pages_per_seq,
                                  int64_t num_pages, bdfp4_fmt fmt, int flags, const bdfp4_kv_params* kv,
                                  float sm_scale, int chunk_tiles, void* workspace, size_t workspace_bytes, void* out,
                                  int32_t* dev_status, void* stream) {
    return run_decode(q, k_pages, k_scales, v_pages, v_scales, block_table, seq_lens, B, T_q, H_q, H_kv, d_k, d_v,
                      max_pages_per_seq, num_pages, fmt, flags, kv, sm_scale, chunk_tiles, workspace,
                      workspace_bytes, out, dev_status, stream, nullptr);
}

// ---------------------------------------------------------------- unwind test (bdfp4_debug.h)
extern "C" int bdfp4_debug_decode_wait_test(const void* q, const void* k_pages, const void* k_scales,
                                            const void* v_pages, const void* v_scales, const int32_t* block_table,
                                            const int32_t* seq_lens, int B, int H_q, int H_kv, int d_k, int d_v,
                                            int max_pages_per_seq, int64_t num_pages, bdfp4_fmt fmt, int flags,
                                            const bdfp4_kv_params* kv, float sm_scale, int chunk_tiles,
                                            void* workspace, size_t workspace_bytes, void* out,
                                            int32_t* dev_status, long long wait_limit_cycles, int stall,
                                            void* stream) {
    // only the d = 128 tensor-core decode's eight-head instantiation takes the switch
    if (d_k != 128 || d_v != 128 || H_kv <= 0 || H_q % H_kv || H_q / H_kv != 8 ||
        (flags & BDFP4_FLAG_DYNAMIC_ALPHA))
        return BDFP4_ERR_UNSUPPORTED;
    if (wait_limit_cycles <= 0) return BDFP4_ERR_ARG;
    return run_decode(q, k_pages, k_scales, v_pages, v_scales, block_table, seq_lens, B, 1, H_q, H_kv, d_k, d_v,
                      max_pages_per_seq, num_pages, fmt, flags, kv, sm_scale, chunk_tiles, workspace,
                      workspace_bytes, out, dev_status, stream, nullptr, wait_limit_cycles, stall ? 1 : 0);
}

// ---------------------------------------------------------------- no-allocation variant
// Scratch for the split partials of bdfp4_decode_noalloc: a file-scope device
// array (held by every GPU that loads the library).  Host code must not pass
// the symbol itself to a kernel -- on the host it is only a stand-in -- so its
// device address is looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[BDFP4_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on failure).
void* noalloc_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}
}  // namespace

extern "C" int bdfp4_decode_noalloc(const void* q, const void* k_pages, const void* k_scales, const void* v_pages,
                                    const void* v_scales, const int32_t* block_table, const int32_t* seq_lens, int B,
                                    int H_q, int H_kv, int d_k, int d_v, int max_pages_per_seq, int64_t num_pages,
                                    bdfp4_fmt fmt, int flags, const bdfp4_kv_params* kv, float sm_scale,
                                    int chunk_tiles, void* out, int32_t* dev_status, void* stream) {
    if (B <= 0 || H_q <= 0 || d_v <= 0 || max_pages_per_seq <= 0)
        return bdfp4_decode(q, k_pages, k_scales, v_pages, v_scales, block_table, seq_lens, B, H_q, H_kv, d_k, d_v,
                            max_pages_per_seq, num_pages, fmt, flags, kv, sm_scale, chunk_tiles, nullptr, 0, out,
                            dev_status, stream);
    if (chunk_tiles <= 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BDFP4_ERR_CUDA;
        const int ntiles = (max_pages_per_seq * kPageSlots + kTileTokens - 1) / kTileTokens;
        const DecodeShape ks = decode_shape(d_k, d_v, H_kv > 0 && H_q % H_kv == 0 ? H_q / H_kv : 1);
        chunk_tiles = plan_chunk_tiles(B, [&](int) { return ntiles; }, (H_kv > 0 ? H_kv : 1) * ks.items_per_kv_head,
                                       sms, ks.ctas_per_sm);
    }
    if (bdfp4_decode_workspace_size(B, H_q, d_v, max_pages_per_seq, chunk_tiles) > BDFP4_NOALLOC_SCRATCH_BYTES)
        return BDFP4_ERR_WORKSPACE;
    void* scratch = noalloc_scratch_address();
    if (!scratch) return BDFP4_ERR_CUDA;
    return bdfp4_decode(q, k_pages, k_scales, v_pages, v_scales, block_table, seq_lens, B, H_q, H_kv, d_k, d_v,
                        max_pages_per_seq, num_pages, fmt, flags, kv, sm_scale, chunk_tiles, scratch,
                        BDFP4_NOALLOC_SCRATCH_BYTES, out, dev_status, stream);
}

namespace bdfp4 {
static thread_local char g_last_error[256] = "no CUDA error recorded";
void record_cuda_error(cudaError_t e) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
}
}  // namespace bdfp4

extern "C" const char* bdfp4_last_error(void) { return bdfp4::g_last_error; }

extern "C" const char* bdfp4_status_string(int status) {
    switch (status) {
        case BDFP4_OK: return "ok";
        case BDFP4_ERR_ARG: return "invalid argument (null pointer, negative size or bad enum)";
        case BDFP4_ERR_SHAPE: return "inconsistent shapes";
        case BDFP4_ERR_ALIGN: return "pointer not aligned (cache arrays and workspace 128 B, bf16 16 B)";
        case BDFP4_ERR_UNSUPPORTED: return "shape outside the compiled set";
        case BDFP4_ERR_CUDA: return "CUDA launch failed";
        case BDFP4_ERR_WORKSPACE: return "workspace too small for the split plan";
        default: return "unknown status";
    }
}
