// quantize.cu -- calibration, KV-append quantization and query quantization
// for the FP4 paged cache (BitDecoding-FP4, Article Summary: Outlier-Aware Key
// Quantization = static smoothing + Hadamard rotation + scale search under
// token-wise scaling; Dual-Residual Query Quantization = q ~ q1 + q2).
//
// Thread mapping: one thread per scale block of a row (beta = 16 or 32
// consecutive channels), so the Hadamard butterflies of stages below beta run
// in registers and the wider stages are lane shuffles inside the row's thread
// group.  The key scale search then gives every candidate code of a block its
// own thread (each fp64 error summed left to right) and one thread picks the
// winner in window order.

#include "bdfp4_device.cuh"
#include "host_common.h"
#include "quant_device.cuh"
#include "append_device.cuh"
#include "decode_common.cuh"

namespace bdfp4 {

// ---------------------------------------------------------------- KV append
template <int FMT, int DK>
__global__ void __launch_bounds__(256, FMT == BDFP4_NVFP4 ? 4 : 2) quantize_k_kernel(const __nv_bfloat16* __restrict__ k,
                                                         const int64_t* __restrict__ slot_mapping, int T, int H_kv,
                                                         const float* __restrict__ smooth,
                                                         const float* __restrict__ k_gscale,
                                                         const float* __restrict__ k_weight, uint8_t* k_pages,
                                                         uint8_t* k_scales, int64_t num_pages, int flags,
                                                         int32_t* dev_status) {
    append_k_cta<FMT, DK>(blockIdx.x, k, (int64_t)T * H_kv, H_kv, MappedSlot{slot_mapping, num_pages, dev_status},
                          smooth, k_gscale, k_weight, k_pages, k_scales, flags);
}

// One thread per (range of beta tokens, head, group of VC channels: 8 for
// NVFP4, 4 for MXFP4): for each token of its range that leads a run within a
// beta-slot block (see bdfp4_quantize_kv in bdfp4.h; usually the range's first
// token) it quantizes the block of its VC channels, loading the run's tokens
// with one 16- or 8-byte load each.  A warp covers whole (range, head) rows, so
// its threads find the same leaders; a thread per token would leave 15 of 16
// CTAs with nothing to do but start and exit.
template <int FMT>
struct VAppend {
    static constexpr int B = Fmt<FMT>::beta;
    static constexpr int VC = FMT == BDFP4_NVFP4 ? 8 : 4;   // channels per thread
    static constexpr int W = VC / 2;                        // 32-bit words of a token's channels
};

template <int FMT, int DV>
__global__ void __launch_bounds__(256) quantize_v_kernel(const __nv_bfloat16* __restrict__ v,
                                                         const int64_t* __restrict__ slot_mapping, int T, int H_kv,
                                                         const float* __restrict__ v_gscale, uint8_t* v_pages,
                                                         uint8_t* v_scales, int64_t num_pages) {
    using VA = VAppend<FMT>;
    constexpr int B = VA::B, VC = VA::VC, W = VA::W;
    constexpr int GPR = DV / VC;   // channel groups of a row
    const int64_t gid = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const int64_t row = gid / GPR;
    const int c0 = (int)(gid % GPR) * VC;
    const int64_t nranges = ((int64_t)T + B - 1) / B;
    if (row >= nranges * H_kv) return;
    const int t0 = (int)(row / H_kv) * B, h = (int)(row % H_kv);
    const int t1 = t0 + B < T ? t0 + B : T;
    int64_t sm_prev = t0 > 0 ? __ldg(slot_mapping + t0 - 1) : -2;
    for (int t = t0; t < t1; ++t) {
    const int64_t sm = __ldg(slot_mapping + t);
    const int64_t smp = sm_prev;
    sm_prev = sm;
    if (sm < 0 || sm >= num_pages * kPageSlots) continue;  // bad slots are reported by the K kernel
    const int slot = (int)(sm % kPageSlots);
    const bool leader = (slot % B == 0) || t == 0 || smp != sm - 1;
    if (!leader) continue;
    int64_t sm_next[B - 1];
#pragma unroll
    for (int i = 1; i < B; ++i) sm_next[i - 1] = t + i < T ? __ldg(slot_mapping + t + i) : -2;
    // run: the following tokens on consecutive slots of the same block
    int n = 1;
    bool run = true;
#pragma unroll
    for (int i = 1; i < B; ++i) {
        run = run && sm_next[i - 1] == sm + i && (slot + i) / B == slot / B;
        n += run ? 1 : 0;
    }
    const int first = slot - slot % B;
    const int off = slot - first;   // block slot of token t
    // raw[i]: the channels of block slot i (token t + i - off when it lies in the run)
    uint32_t raw[B][W];
#pragma unroll
    for (int i = 0; i < B; ++i) {
        const int jt = i - off;
        const bool in = jt >= 0 && jt < n;
        const __nv_bfloat16* src = v + ((int64_t)(t + (in ? jt : 0)) * H_kv + h) * DV + c0;
        if constexpr (W == 4) {
            uint4 u = in ? __ldg(reinterpret_cast<const uint4*>(src)) : make_uint4(0u, 0u, 0u, 0u);
            raw[i][0] = u.x; raw[i][1] = u.y; raw[i][2] = u.z; raw[i][3] = u.w;
        } else {
            uint2 u = in ? __ldg(reinterpret_cast<const uint2*>(src)) : make_uint2(0u, 0u);
            raw[i][0] = u.x; raw[i][1] = u.y;
        }
    }
    const float g = FMT == BDFP4_NVFP4 ? __ldg(v_gscale + h) : 1.0f;
    const int64_t page = sm / kPageSlots;
    uint8_t* vp = v_pages + (page * H_kv + h) * (int64_t)(DV * kPageSlots / 2);
    uint8_t* vs = v_scales + (page * H_kv + h) * (int64_t)(DV * kPageSlots / B);
#pragma unroll
    for (int cc = 0; cc < VC; ++cc) {
        float x[B];
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const uint32_t w = raw[i][cc >> 1];
            x[i] = __uint_as_float((cc & 1) ? (w & 0xffff0000u) : (w << 16));
        }
        const uint32_t code = plain_scale_code<FMT>(block_amax<B>(x), g);
        uint32_t packed[B / 8];
        if constexpr (FMT == BDFP4_MXFP4) {
            // sigma = 2^(code - 127): dividing by it is multiplying by 2^(127 - code), exactly
            const float inv = __uint_as_float(code == 254u ? 0x00400000u : (254u - code) << 23);
            quantize_block<B, false, true>(x, block_sigma<FMT>(code, g), packed, nullptr, inv);
        } else {
            quantize_block<B>(x, block_sigma<FMT>(code, g), packed);
        }
        uint8_t* dst = vp + v_nib_offset(c0 + cc, first);
        if constexpr (B == 16) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
        } else {
            *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
        vs[v_scale_offset<B>(c0 + cc, first / B)] = (uint8_t)code;
    }
    }
}

// Decode-step append: key CTAs first, then value CTAs, one (sequence, KV
// head) row per new token.
template <int FMT, int DK, int DV>
__global__ void __launch_bounds__(256) step_append_kernel(const DecodeArgs a, const StepArgs s) {
    const int64_t rows = (int64_t)a.B * a.H_kv;
    const NewestSlot slot{a.block_table, a.seq_lens, a.max_pages, a.num_pages, a.dev_status};
    const int nk = (int)k_append_ctas_wide<FMT, DK>(rows);
    if ((int)blockIdx.x < nk)
        append_k_cta_wide<FMT, DK>(blockIdx.x, s.k_new, rows, a.H_kv, slot, a.smooth, a.k_gscale, a.k_weight, s.k_pages, s.k_scales,
                              a.flags);
    else
        append_v_open_cta<FMT, DV>(blockIdx.x - nk, s.v_new, s.v_open, slot, a.B, a.H_kv, a.v_gscale, s.v_pages,
                                   s.v_scales);
}

template <int FMT, int DK, int DV>
static int launch_step_append_t(const DecodeArgs& a, const StepArgs& s, cudaStream_t st) {
    const int64_t rows = (int64_t)a.B * a.H_kv;
    const int64_t ctas = k_append_ctas_wide<FMT, DK>(rows) + v_append_ctas<DV>(rows);
    step_append_kernel<FMT, DK, DV><<<(unsigned)ctas, 256, 0, st>>>(a, s);
    return launch_status();
}

int launch_step_append(const DecodeArgs& a, const StepArgs& s, int fmt, int d_k, cudaStream_t st) {
    if (fmt == BDFP4_NVFP4)
        return d_k == 128 ? launch_step_append_t<BDFP4_NVFP4, 128, 128>(a, s, st)
                          : launch_step_append_t<BDFP4_NVFP4, 576, 512>(a, s, st);
    return d_k == 128 ? launch_step_append_t<BDFP4_MXFP4, 128, 128>(a, s, st)
                      : launch_step_append_t<BDFP4_MXFP4, 576, 512>(a, s, st);
}

template <int FMT, int DK>
__global__ void __launch_bounds__(256) quantize_q_kernel(const __nv_bfloat16* __restrict__ q, int rows, int H_q,
                                                         int G, const float* __restrict__ smooth, int flags,
                                                         uint8_t* q1_codes, uint8_t* q1_scales, uint8_t* q2_codes,
                                                         uint8_t* q2_scales, float* g_q) {
    using RG = RowGeom<FMT, DK>;
    constexpr int B = RG::beta;
    constexpr int rows_per_block = 256 / RG::rt;
    __shared__ int row_amax[rows_per_block];
    const int j = threadIdx.x % RG::rt;
    const int rl = threadIdx.x / RG::rt;
    const int row = blockIdx.x * rows_per_block + rl;
    const bool active = row < rows && j < RG::tpr;
    if (threadIdx.x < rows_per_block) row_amax[threadIdx.x] = 0;
    float x[B];
    if (active) {
        load_bf16_block<B>(q + (int64_t)row * DK, j * B, x);
    } else {
#pragma unroll
        for (int i = 0; i < B; ++i) x[i] = 0.0f;
    }
    const int hk = active ? (row % H_q) / G : 0;
    transform_block<FMT, DK, false>(x, smooth + (int64_t)hk * DK, j, !(flags & BDFP4_FLAG_NO_HADAMARD));
    __syncthreads();
    if (active) atomicMax(&row_amax[rl], __float_as_int(block_amax<B>(x)));
    __syncthreads();
    if (!active) return;
    const float amax = __int_as_float(row_amax[rl]);
    const float gq = FMT == BDFP4_NVFP4 ? (amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f) : 1.0f;
    uint32_t c1, c2, p1[B / 8], p2[B / 8];
    quantize_query_block<FMT, DK>(x, gq, !(flags & BDFP4_FLAG_SINGLE_QUERY), c1, p1, c2, p2);
#pragma unroll
    for (int i = 0; i < B; ++i) {
        q1_codes[(int64_t)row * DK + j * B + i] = (uint8_t)((p1[i / 8] >> (4 * (i % 8))) & 15u);
        q2_codes[(int64_t)row * DK + j * B + i] = (uint8_t)((p2[i / 8] >> (4 * (i % 8))) & 15u);
    }
    q1_scales[(int64_t)row * (DK / B) + j] = (uint8_t)c1;
    q2_scales[(int64_t)row * (DK / B) + j] = (uint8_t)c2;
    if (j == 0) g_q[row] = gq;
}

// ---------------------------------------------------------------- calibration
// One CTA per KV head; blockDim = max(d_k, d_v) threads (a multiple of 32).
__device__ __forceinline__ int floor_log2_ratio(float a, float b) {
    int ea, eb;
    float fa = frexpf(a, &ea), fb = frexpf(b, &eb);
    return (ea - eb) + (fa >= fb ? 0 : -1);
}

__global__ void calibrate_kernel(const __nv_bfloat16* __restrict__ k_cal, const __nv_bfloat16* __restrict__ q_cal,
                                 const __nv_bfloat16* __restrict__ v_cal, int Tc, int Tq, int H_q, int H_kv, int d_k,
                                 int d_v, int flags, float* smooth, float* k_gscale, float* v_gscale) {
    extern __shared__ float sh[];  // x[d_k]
    __shared__ int amax_bits;
    __shared__ int vmax_bits;
    float* xs = sh;
    const int h = blockIdx.x, c = threadIdx.x, G = H_q / H_kv;
    const unsigned short* kb = reinterpret_cast<const unsigned short*>(k_cal);
    const unsigned short* qb = reinterpret_cast<const unsigned short*>(q_cal);
    const unsigned short* vb = reinterpret_cast<const unsigned short*>(v_cal);
    if (c == 0) {
        amax_bits = 0;
        vmax_bits = 0;
    }
    float s = 1.0f;
    if (c < d_k) {
        float kmax = 0.0f, qmax = 0.0f;
        for (int t = 0; t < Tc; ++t)
            kmax = fmaxf(kmax, fabsf(__uint_as_float((uint32_t)kb[((int64_t)t * H_kv + h) * d_k + c] << 16)));
        for (int t = 0; t < Tq; ++t)
            for (int jg = 0; jg < G; ++jg)
                qmax = fmaxf(qmax, fabsf(__uint_as_float((uint32_t)qb[((int64_t)t * H_q + h * G + jg) * d_k + c] << 16)));
        int n = 0;
        if (kmax > 0.0f && qmax > 0.0f) {
            n = (floor_log2_ratio(kmax, qmax) + 1) >> 1;
            n = n < -20 ? -20 : (n > 20 ? 20 : n);
        }
        s = __uint_as_float((uint32_t)(127 + n) << 23);
        smooth[(int64_t)h * d_k + c] = s;
    }
    const bool hadamard = !(flags & BDFP4_FLAG_NO_HADAMARD);
    const int seg0 = d_k == 576 ? 512 : d_k;
    const int seg_base = c < seg0 ? 0 : seg0;
    const int seg_len = c < seg0 ? seg0 : d_k - seg0;
    float run_max = 0.0f;
    for (int t = 0; t < Tc; ++t) {
        __syncthreads();
        if (c < d_k) xs[c] = __fdiv_rn(__uint_as_float((uint32_t)kb[((int64_t)t * H_kv + h) * d_k + c] << 16), s);
        __syncthreads();
        if (hadamard) {
            for (int hs = 1; hs < seg_len; hs <<= 1) {
                float nv = 0.0f;
                if (c < d_k) {
                    const int ci = c - seg_base;
                    nv = (ci & hs) == 0 ? __fadd_rn(xs[c], xs[c + hs]) : __fsub_rn(xs[c - hs], xs[c]);
                }
                __syncthreads();
                if (c < d_k) xs[c] = nv;
                __syncthreads();
            }
            if (c < d_k) xs[c] = __fmul_rn(xs[c], hadamard_post(seg_len, true));
        }
        if (c < d_k) run_max = fmaxf(run_max, fabsf(xs[c]));
    }
    float vmax = 0.0f;
    if (c < d_v)
        for (int t = 0; t < Tc; ++t)
            vmax = fmaxf(vmax, fabsf(__uint_as_float((uint32_t)vb[((int64_t)t * H_kv + h) * d_v + c] << 16)));
    __syncthreads();
    atomicMax(&amax_bits, __float_as_int(run_max));
    atomicMax(&vmax_bits, __float_as_int(vmax));
    __syncthreads();
    if (c == 0) {
        const float ka = __int_as_float(amax_bits), va = __int_as_float(vmax_bits);
        k_gscale[h] = ka > 0.0f ? __fdiv_rn(ka, 2688.0f) : 1.0f;
        v_gscale[h] = va > 0.0f ? __fdiv_rn(va, 2688.0f) : 1.0f;
    }
}

// ---------------------------------------------------------------- key weights
// Channel weights of the attention-aware key scale search, one CTA per KV
// head.  Each pass transforms R calibration query rows of the head's group
// (a thread per 16-channel block, butterflies across the row's threads) into
// shared memory; then the thread owning channel c adds the rows' squares of
// that channel in query order (token, then head) to its fp64 sum.
template <int DK>
__global__ void __launch_bounds__(256) key_weights_kernel(const __nv_bfloat16* __restrict__ q_cal, int Tq, int H_q,
                                                          int H_kv, int flags, const float* __restrict__ smooth,
                                                          float* w) {
    using RG = RowGeom<BDFP4_NVFP4, DK>;
    constexpr int B = RG::beta;
    constexpr int R = 256 / RG::rt;
    constexpr int NCH = (DK + 255) / 256;   // channels per thread: threadIdx.x + 256 i
    __shared__ float xs[R][DK];
    const int hk = blockIdx.x, G = H_q / H_kv;
    const int r = threadIdx.x / RG::rt, j = threadIdx.x % RG::rt;
    const int64_t nrows = (int64_t)Tq * G;
    const bool hadamard = !(flags & BDFP4_FLAG_NO_HADAMARD);
    double acc[NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) acc[i] = 0.0;
    for (int64_t q0 = 0; q0 < nrows; q0 += R) {
        const int64_t qi = q0 + r;
        const bool act = qi < nrows && j < RG::tpr;
        float x[B];
        if (act) {
            const int64_t t = qi / G, jg = qi % G;
            load_bf16_block<B>(q_cal + (t * H_q + (int64_t)hk * G + jg) * DK, j * B, x);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i) x[i] = 0.0f;
        }
        transform_block<BDFP4_NVFP4, DK, false>(x, smooth + (int64_t)hk * DK, j, hadamard);
        __syncthreads();   // the previous pass's rows have been read
        if (act) {
#pragma unroll
            for (int i = 0; i < B; ++i) xs[r][j * B + i] = x[i];
        }
        __syncthreads();
        const int nr = (int)(nrows - q0 < R ? nrows - q0 : R);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = threadIdx.x + 256 * i;
            if (c < DK)
                for (int rr = 0; rr < nr; ++rr) {
                    const double v = (double)xs[rr][c];
                    acc[i] = __dadd_rn(acc[i], __dmul_rn(v, v));
                }
        }
    }
    const double n = (double)Tq * (double)G;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = threadIdx.x + 256 * i;
        if (c < DK) w[(int64_t)hk * DK + c] = __double2float_rn(__ddiv_rn(acc[i], n));
    }
}

}  // namespace bdfp4

using namespace bdfp4;

// ================================================================ host API
extern "C" int bdfp4_calibrate(const void* k_cal, const void* q_cal, const void* v_cal, int Tc, int Tq, int H_q,
                               int H_kv, int d_k, int d_v, int flags, float* smooth, float* k_gscale, float* v_gscale,
                               void* stream) {
    if (!k_cal || !q_cal || !v_cal || !smooth || !k_gscale || !v_gscale) return BDFP4_ERR_ARG;
    if (Tc <= 0 || Tq <= 0 || H_kv <= 0 || H_q <= 0) return BDFP4_ERR_ARG;
    if (H_q % H_kv) return BDFP4_ERR_SHAPE;
    if (!supported_dims(d_k, d_v)) return BDFP4_ERR_UNSUPPORTED;
    const int threads = d_k > d_v ? d_k : d_v;
    calibrate_kernel<<<H_kv, threads, d_k * sizeof(float), (cudaStream_t)stream>>>(
        (const __nv_bfloat16*)k_cal, (const __nv_bfloat16*)q_cal, (const __nv_bfloat16*)v_cal, Tc, Tq, H_q, H_kv, d_k,
        d_v, flags, smooth, k_gscale, v_gscale);
    return launch_status();
}

extern "C" int bdfp4_key_weights(const void* q_cal, int Tq, int H_q, int H_kv, int d_k, int flags,
                                 const float* smooth, float* w, void* stream) {
    if (!q_cal || !smooth || !w || Tq <= 0 || H_q <= 0 || H_kv <= 0) return BDFP4_ERR_ARG;
    if (H_q % H_kv) return BDFP4_ERR_SHAPE;
    if (d_k != 128 && d_k != 576) return BDFP4_ERR_UNSUPPORTED;
    if (!aligned(q_cal, 16)) return BDFP4_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    if (d_k == 128)
        key_weights_kernel<128><<<H_kv, 256, 0, st>>>((const __nv_bfloat16*)q_cal, Tq, H_q, H_kv, flags, smooth, w);
    else
        key_weights_kernel<576><<<H_kv, 256, 0, st>>>((const __nv_bfloat16*)q_cal, Tq, H_q, H_kv, flags, smooth, w);
    return launch_status();
}

template <int FMT, int DK, int DV>
static void launch_quantize_kv(const void* k, const void* v, const int64_t* slot_mapping, int T, int H_kv,
                               const bdfp4_kv_params* kv, void* k_pages, void* k_scales, void* v_pages,
                               void* v_scales, int64_t num_pages, int flags, int32_t* dev_status, cudaStream_t st) {
    const int64_t rows = (int64_t)T * H_kv;
    const int64_t kblocks = (rows + KGeom<FMT, DK>::R - 1) / KGeom<FMT, DK>::R;
    quantize_k_kernel<FMT, DK><<<(unsigned)kblocks, 256, 0, st>>>(
        (const __nv_bfloat16*)k, slot_mapping, T, H_kv, kv->smooth, kv->k_gscale, kv->k_weight, (uint8_t*)k_pages,
        (uint8_t*)k_scales, num_pages, flags, dev_status);
    const int64_t vthreads = ((int64_t)T + Fmt<FMT>::beta - 1) / Fmt<FMT>::beta * H_kv * (DV / VAppend<FMT>::VC);
    quantize_v_kernel<FMT, DV><<<(unsigned)((vthreads + 255) / 256), 256, 0, st>>>(
        (const __nv_bfloat16*)v, slot_mapping, T, H_kv, kv->v_gscale, (uint8_t*)v_pages, (uint8_t*)v_scales,
        num_pages);
}

extern "C" int bdfp4_quantize_kv(const void* k, const void* v, const int64_t* slot_mapping, int T, int H_kv, int d_k,
                                 int d_v, bdfp4_fmt fmt, int flags, const bdfp4_kv_params* kv, void* k_pages,
                                 void* k_scales, void* v_pages, void* v_scales, int64_t num_pages,
                                 int32_t* dev_status, void* stream) {
    if (T < 0 || H_kv <= 0 || num_pages < 0) return BDFP4_ERR_ARG;
    if (fmt != BDFP4_NVFP4 && fmt != BDFP4_MXFP4) return BDFP4_ERR_ARG;
    if (!supported_dims(d_k, d_v)) return BDFP4_ERR_UNSUPPORTED;
    if (T == 0) return BDFP4_OK;
    if (!k || !v || !slot_mapping || !kv || !kv->smooth || !k_pages || !k_scales || !v_pages || !v_scales)
        return BDFP4_ERR_ARG;
    if (fmt == BDFP4_NVFP4 && (!kv->k_gscale || !kv->v_gscale)) return BDFP4_ERR_ARG;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_pages, 128) || !aligned(k_scales, 128) ||
        !aligned(v_pages, 128) || !aligned(v_scales, 128))
        return BDFP4_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    if (fmt == BDFP4_NVFP4) {
        if (d_k == 128)
            launch_quantize_kv<BDFP4_NVFP4, 128, 128>(k, v, slot_mapping, T, H_kv, kv, k_pages, k_scales, v_pages,
                                                      v_scales, num_pages, flags, dev_status, st);
        else
            launch_quantize_kv<BDFP4_NVFP4, 576, 512>(k, v, slot_mapping, T, H_kv, kv, k_pages, k_scales, v_pages,
                                                      v_scales, num_pages, flags, dev_status, st);
    } else {
        if (d_k == 128)
            launch_quantize_kv<BDFP4_MXFP4, 128, 128>(k, v, slot_mapping, T, H_kv, kv, k_pages, k_scales, v_pages,
                                                      v_scales, num_pages, flags, dev_status, st);
        else
            launch_quantize_kv<BDFP4_MXFP4, 576, 512>(k, v, slot_mapping, T, H_kv, kv, k_pages, k_scales, v_pages,
                                                      v_scales, num_pages, flags, dev_status, st);
    }
    return launch_status();
}

// The key half and the value half of bdfp4_quantize_kv on their own token lists.
extern "C" int bdfp4_quantize_k(const void* k, const int64_t* slot_mapping, int T, int H_kv, int d_k, bdfp4_fmt fmt,
                                int flags, const bdfp4_kv_params* kv, void* k_pages, void* k_scales,
                                int64_t num_pages, int32_t* dev_status, void* stream) {
    if (T < 0 || H_kv <= 0 || num_pages < 0) return BDFP4_ERR_ARG;
    if (fmt != BDFP4_NVFP4 && fmt != BDFP4_MXFP4) return BDFP4_ERR_ARG;
    if (d_k != 128 && d_k != 576) return BDFP4_ERR_UNSUPPORTED;
    if (T == 0) return BDFP4_OK;
    if (!k || !slot_mapping || !kv || !kv->smooth || !k_pages || !k_scales) return BDFP4_ERR_ARG;
    if (fmt == BDFP4_NVFP4 && !kv->k_gscale) return BDFP4_ERR_ARG;
    if (!aligned(k, 16) || !aligned(k_pages, 128) || !aligned(k_scales, 128)) return BDFP4_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t rows = (int64_t)T * H_kv;
    auto launch = [&](auto kernel, int R) {
        kernel<<<(unsigned)((rows + R - 1) / R), 256, 0, st>>>((const __nv_bfloat16*)k, slot_mapping, T, H_kv,
                                                              kv->smooth, kv->k_gscale, kv->k_weight,
                                                              (uint8_t*)k_pages,
                                                              (uint8_t*)k_scales, num_pages, flags, dev_status);
    };
    if (fmt == BDFP4_NVFP4) {
        if (d_k == 128) launch(quantize_k_kernel<BDFP4_NVFP4, 128>, KGeom<BDFP4_NVFP4, 128>::R);
        else launch(quantize_k_kernel<BDFP4_NVFP4, 576>, KGeom<BDFP4_NVFP4, 576>::R);
    } else {
        if (d_k == 128) launch(quantize_k_kernel<BDFP4_MXFP4, 128>, KGeom<BDFP4_MXFP4, 128>::R);
        else launch(quantize_k_kernel<BDFP4_MXFP4, 576>, KGeom<BDFP4_MXFP4, 576>::R);
    }
    return launch_status();
}

extern "C" int bdfp4_quantize_v(const void* v, const int64_t* slot_mapping, int T, int H_kv, int d_v, bdfp4_fmt fmt,
                                const bdfp4_kv_params* kv, void* v_pages, void* v_scales, int64_t num_pages,
                                void* stream) {
    if (T < 0 || H_kv <= 0 || num_pages < 0) return BDFP4_ERR_ARG;
    if (fmt != BDFP4_NVFP4 && fmt != BDFP4_MXFP4) return BDFP4_ERR_ARG;
    if (d_v != 128 && d_v != 512) return BDFP4_ERR_UNSUPPORTED;
    if (T == 0) return BDFP4_OK;
    if (!v || !slot_mapping || !kv || !v_pages || !v_scales) return BDFP4_ERR_ARG;
    if (fmt == BDFP4_NVFP4 && !kv->v_gscale) return BDFP4_ERR_ARG;
    if (!aligned(v, 16) || !aligned(v_pages, 128) || !aligned(v_scales, 128)) return BDFP4_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    auto launch = [&](auto kernel, int groups_per_row) {
        const int beta = fmt == BDFP4_NVFP4 ? 16 : 32;
        const int64_t threads = ((int64_t)T + beta - 1) / beta * H_kv * groups_per_row;
        kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>((const __nv_bfloat16*)v, slot_mapping, T, H_kv,
                                                                 kv->v_gscale, (uint8_t*)v_pages, (uint8_t*)v_scales,
                                                                 num_pages);
    };
    if (fmt == BDFP4_NVFP4) {
        if (d_v == 128) launch(quantize_v_kernel<BDFP4_NVFP4, 128>, 128 / VAppend<BDFP4_NVFP4>::VC);
        else launch(quantize_v_kernel<BDFP4_NVFP4, 512>, 512 / VAppend<BDFP4_NVFP4>::VC);
    } else {
        if (d_v == 128) launch(quantize_v_kernel<BDFP4_MXFP4, 128>, 128 / VAppend<BDFP4_MXFP4>::VC);
        else launch(quantize_v_kernel<BDFP4_MXFP4, 512>, 512 / VAppend<BDFP4_MXFP4>::VC);
    }
    return launch_status();
}

template <int FMT, int DK>
static void launch_quantize_q(const void* q, int rows, int H_q, int G, const float* smooth, int flags, uint8_t* q1c,
                              uint8_t* q1s, uint8_t* q2c, uint8_t* q2s, float* gq, cudaStream_t st) {
    using RG = RowGeom<FMT, DK>;
    const int rows_per_block = 256 / RG::rt;
    quantize_q_kernel<FMT, DK><<<(rows + rows_per_block - 1) / rows_per_block, 256, 0, st>>>(
        (const __nv_bfloat16*)q, rows, H_q, G, smooth, flags, q1c, q1s, q2c, q2s, gq);
}

extern "C" int bdfp4_quantize_q(const void* q, int B, int H_q, int H_kv, int d_k, bdfp4_fmt fmt, int flags,
                                const float* smooth, uint8_t* q1_codes, uint8_t* q1_scales, uint8_t* q2_codes,
                                uint8_t* q2_scales, float* g_q, void* stream) {
    if (B < 0 || H_q <= 0 || H_kv <= 0) return BDFP4_ERR_ARG;
    if (fmt != BDFP4_NVFP4 && fmt != BDFP4_MXFP4) return BDFP4_ERR_ARG;
    if (H_q % H_kv) return BDFP4_ERR_SHAPE;
    if (d_k != 128 && d_k != 576) return BDFP4_ERR_UNSUPPORTED;
    if (B == 0) return BDFP4_OK;
    if (!q || !smooth || !q1_codes || !q1_scales || !q2_codes || !q2_scales || !g_q) return BDFP4_ERR_ARG;
    if (!aligned(q, 16)) return BDFP4_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    const int rows = B * H_q, G = H_q / H_kv;
    if (fmt == BDFP4_NVFP4) {
        if (d_k == 128) launch_quantize_q<BDFP4_NVFP4, 128>(q, rows, H_q, G, smooth, flags, q1_codes, q1_scales, q2_codes, q2_scales, g_q, st);
        else launch_quantize_q<BDFP4_NVFP4, 576>(q, rows, H_q, G, smooth, flags, q1_codes, q1_scales, q2_codes, q2_scales, g_q, st);
    } else {
        if (d_k == 128) launch_quantize_q<BDFP4_MXFP4, 128>(q, rows, H_q, G, smooth, flags, q1_codes, q1_scales, q2_codes, q2_scales, g_q, st);
        else launch_quantize_q<BDFP4_MXFP4, 576>(q, rows, H_q, G, smooth, flags, q1_codes, q1_scales, q2_codes, q2_scales, g_q, st);
    }
    return launch_status();
}
