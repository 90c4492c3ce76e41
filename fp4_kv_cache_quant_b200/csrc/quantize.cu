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

namespace bdfp4 {

// ---------------------------------------------------------------- K append
// Work split of the K append: every scale block of a row gets NC lanes, one per
// candidate code of its search window (10 for NVFP4, 2 for MXFP4, padded), so
// the window is searched in parallel; R rows share a 256-thread CTA.
template <int FMT, int DK>
struct KGeom {
    using RG = RowGeom<FMT, DK>;
    static constexpr int B = RG::beta;
    static constexpr int NB = DK / B;                                  // scale blocks per row
    static constexpr int NC = FMT == BDFP4_NVFP4 ? 16 : 2;             // candidate lanes per block
    static constexpr int R = 256 / (NB * NC) >= 1 ? 256 / (NB * NC) : 1;
    static constexpr int PAIRS = R * NB * NC;                           // (block, candidate) pairs
    static constexpr int PAIRS_PAD = (PAIRS + 255) / 256 * 256;
    static constexpr int T1 = (R * RG::rt + 31) / 32 * 32;             // transform threads (whole warps)
    static_assert(T1 <= 256, "transform threads exceed the CTA");
};

// Phase 1 transforms R rows into shared memory (thread per block, butterflies
// across the row's threads); phase 2 quantizes every block under every code of
// its window and keeps the fp64 squared errors (each summed left to right);
// phase 3 scans each window from its largest code down, keeping the first
// least error, and stores the winner.  The choice is the sequential search's.
template <int FMT, int DK>
__global__ void __launch_bounds__(256) quantize_k_kernel(const __nv_bfloat16* __restrict__ k,
                                                         const int64_t* __restrict__ slot_mapping, int T, int H_kv,
                                                         const float* __restrict__ smooth,
                                                         const float* __restrict__ k_gscale, uint8_t* k_pages,
                                                         uint8_t* k_scales, int64_t num_pages, int flags,
                                                         int32_t* dev_status) {
    using KG = KGeom<FMT, DK>;
    using RG = typename KG::RG;
    constexpr int B = KG::B, NB = KG::NB, NC = KG::NC, R = KG::R;
    __shared__ float xs[R][DK];
    __shared__ double errs[KG::PAIRS_PAD];
    __shared__ uint32_t pks[KG::PAIRS_PAD][B / 8];
    __shared__ int win[R * NB];            // hi << 16 | lo
    __shared__ long long slots[R];
    __shared__ float gs[R];                // tensor scale of the row's head
    const int tid = threadIdx.x;
    const int64_t rows = (int64_t)T * H_kv;
    const int64_t row0 = (int64_t)blockIdx.x * R;

    if (tid < KG::T1) {
        const int r = tid / RG::rt, j = tid % RG::rt;
        const int64_t row = row0 + r;
        const bool in_range = r < R && row < rows;
        const int t = (int)(in_range ? row / H_kv : 0);
        const int h = (int)(in_range ? row % H_kv : 0);
        int64_t sm = in_range ? __ldg(slot_mapping + t) : -1;
        if (sm >= num_pages * kPageSlots) {
            if (j == 0) set_status(dev_status, BDFP4_DEV_BAD_SLOT);
            sm = -1;
        }
        // whole warps stay converged through the shuffles; inactive rows compute on zeros
        // the row is loaded whatever its slot id, so the two loads overlap
        float x[B];
        if (in_range && j < RG::tpr) {
            load_bf16_block<B>(k + ((int64_t)t * H_kv + h) * DK, j * B, x);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i) x[i] = 0.0f;
        }
        if (sm < 0) {
#pragma unroll
            for (int i = 0; i < B; ++i) x[i] = 0.0f;
        }
        const bool active = sm >= 0 && j < RG::tpr;
        transform_block<FMT, DK, true>(x, smooth + (int64_t)h * DK, j, !(flags & BDFP4_FLAG_NO_HADAMARD));
        if (active) {
#pragma unroll
            for (int i = 0; i < B; ++i) xs[r][j * B + i] = x[i];
        }
        if (r < R && j == 0) {
            slots[r] = sm;
            gs[r] = FMT == BDFP4_NVFP4 ? __ldg(k_gscale + h) : 1.0f;
        }
    }
    __syncthreads();

    for (int p = tid; p < KG::PAIRS; p += 256) {
        const int r = p / (NB * NC), bk = (p / NC) % NB, ci = p % NC;
        if (slots[r] < 0) continue;
        const float g = gs[r];
        float x[B];
#pragma unroll
        for (int i = 0; i < B; ++i) x[i] = xs[r][bk * B + i];
        const float amax = block_amax<B>(x);
        const int c0 = (int)plain_scale_code<FMT>(amax, g);
        int hi = c0, lo = c0;   // all-zero blocks and the plain rule keep c0
        if (amax != 0.0f && !(flags & BDFP4_FLAG_NO_SCALE_SEARCH)) {
            const int top = FMT == BDFP4_NVFP4 ? 126 : 254;
            hi = min(c0 + (FMT == BDFP4_NVFP4 ? 7 : 1), top);
            lo = max(c0 - (FMT == BDFP4_NVFP4 ? 2 : 0), 0);
        }
        if (ci == 0) win[r * NB + bk] = (hi << 16) | lo;
        const int c = hi - ci;
        if (c >= lo) errs[p] = quantize_block<B>(x, block_sigma<FMT>((uint32_t)c, g), pks[p]);
    }
    __syncthreads();

    for (int q = tid; q < R * NB; q += 256) {
        const int r = q / NB, bk = q % NB;
        const int64_t sm = slots[r];
        if (sm < 0) continue;
        const int h = (int)((row0 + r) % H_kv);
        const int hi = win[q] >> 16, lo = win[q] & 0xffff;
        const int base = q * NC;
        int best = 0;
        double best_err = errs[base];
        for (int ci = 1; ci <= hi - lo; ++ci) {
            if (errs[base + ci] < best_err) {
                best = ci;
                best_err = errs[base + ci];
            }
        }
        const int64_t page = sm / kPageSlots;
        const int slot = (int)(sm % kPageSlots);
        uint8_t* kp = k_pages + (page * H_kv + h) * (int64_t)(kPageSlots * DK / 2);
        uint8_t* dst = kp + k_nib_offset(DK, slot, bk * B);
        const uint32_t* pk = pks[base + best];
        if constexpr (B == 16) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
        } else {
            *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        uint8_t* ks = k_scales + (page * H_kv + h) * (int64_t)k_scale_page_bytes(DK, B);
        ks[k_scale_offset<B>(DK, slot, bk)] = (uint8_t)(hi - best);
    }
}

// ---------------------------------------------------------------- V append
// One thread per (token, head, channel); only the first token of each run
// within a beta-slot block does work (see bdfp4_quantize_kv in bdfp4.h), for
// the whole block of its channel.
template <int DV>
struct VGeom {
    static constexpr int TPR = DV < 256 ? DV : 256;   // threads of a row in one CTA
    static constexpr int RPC = 256 / TPR;             // rows per CTA
    static constexpr int CPR = DV / TPR;              // CTAs per row
};

template <int FMT, int DV>
__global__ void __launch_bounds__(256) quantize_v_kernel(const __nv_bfloat16* __restrict__ v,
                                                         const int64_t* __restrict__ slot_mapping, int T, int H_kv,
                                                         const float* __restrict__ v_gscale, uint8_t* v_pages,
                                                         uint8_t* v_scales, int64_t num_pages) {
    constexpr int B = Fmt<FMT>::beta;
    using VG = VGeom<DV>;
    const int64_t row = (int64_t)(blockIdx.x / VG::CPR) * VG::RPC + threadIdx.x / VG::TPR;
    const int c = (int)(blockIdx.x % VG::CPR) * VG::TPR + threadIdx.x % VG::TPR;
    if (row >= (int64_t)T * H_kv) return;
    const int t = (int)(row / H_kv), h = (int)(row % H_kv);
    // two rounds of independent loads: this token's and its predecessor's slot
    // ids (the leader test), then the next B - 1 slot ids with the B rows a run can cover
    const int64_t sm = __ldg(slot_mapping + t);
    const int64_t sm_prev = t > 0 ? __ldg(slot_mapping + t - 1) : -2;
    if (sm < 0 || sm >= num_pages * kPageSlots) return;  // bad slots are reported by the K kernel
    const int slot = (int)(sm % kPageSlots);
    const bool leader = (slot % B == 0) || t == 0 || sm_prev != sm - 1;
    if (!leader) return;
    int64_t sm_next[B - 1];
#pragma unroll
    for (int i = 1; i < B; ++i) sm_next[i - 1] = t + i < T ? __ldg(slot_mapping + t + i) : -2;
    const unsigned short* vb = reinterpret_cast<const unsigned short*>(v);
    uint32_t raw[B];
#pragma unroll
    for (int i = 0; i < B; ++i) raw[i] = t + i < T ? (uint32_t)__ldg(vb + ((int64_t)(t + i) * H_kv + h) * DV + c) : 0u;
    const float g = FMT == BDFP4_NVFP4 ? __ldg(v_gscale + h) : 1.0f;
    // run: the following tokens on consecutive slots of the same block
    int n = 1;
    bool run = true;
#pragma unroll
    for (int i = 1; i < B; ++i) {
        run = run && sm_next[i - 1] == sm + i && (slot + i) / B == slot / B;
        n += run ? 1 : 0;
    }
    const int first = slot - slot % B;
    const int64_t page = sm / kPageSlots;
    uint8_t* vp = v_pages + (page * H_kv + h) * (int64_t)(DV * kPageSlots / 2);
    uint8_t* vs = v_scales + (page * H_kv + h) * (int64_t)(DV * kPageSlots / B);
    // slot first + i holds token t + (first + i - slot) when that lies in the run
    float x[B];
#pragma unroll
    for (int i = 0; i < B; ++i) {
        const int jt = first + i - slot;
        uint32_t w = 0u;
#pragma unroll
        for (int u = 0; u < B; ++u) w = (u == jt) ? raw[u] : w;
        x[i] = (jt >= 0 && jt < n) ? __uint_as_float(w << 16) : 0.0f;
    }
    const uint32_t code = plain_scale_code<FMT>(block_amax<B>(x), g);
    uint32_t packed[B / 8];
    quantize_block<B>(x, block_sigma<FMT>(code, g), packed);
    uint8_t* dst = vp + v_nib_offset(c, first);
    if constexpr (B == 16) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    vs[v_scale_offset<B>(c, first / B)] = (uint8_t)code;
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

template <int FMT, int DK, int DV>
static void launch_quantize_kv(const void* k, const void* v, const int64_t* slot_mapping, int T, int H_kv,
                               const bdfp4_kv_params* kv, void* k_pages, void* k_scales, void* v_pages,
                               void* v_scales, int64_t num_pages, int flags, int32_t* dev_status, cudaStream_t st) {
    const int64_t rows = (int64_t)T * H_kv;
    const int64_t kblocks = (rows + KGeom<FMT, DK>::R - 1) / KGeom<FMT, DK>::R;
    quantize_k_kernel<FMT, DK><<<(unsigned)kblocks, 256, 0, st>>>(
        (const __nv_bfloat16*)k, slot_mapping, T, H_kv, kv->smooth, kv->k_gscale, (uint8_t*)k_pages,
        (uint8_t*)k_scales, num_pages, flags, dev_status);
    using VG = VGeom<DV>;
    const int64_t vblocks = (rows + VG::RPC - 1) / VG::RPC * VG::CPR;
    quantize_v_kernel<FMT, DV><<<(unsigned)vblocks, 256, 0, st>>>((const __nv_bfloat16*)v, slot_mapping, T, H_kv,
                                                                  kv->v_gscale, (uint8_t*)v_pages,
                                                                  (uint8_t*)v_scales, num_pages);
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
                                                              kv->smooth, kv->k_gscale, (uint8_t*)k_pages,
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
    const int64_t rows = (int64_t)T * H_kv;
    auto launch = [&](auto kernel, int RPC, int CPR) {
        kernel<<<(unsigned)((rows + RPC - 1) / RPC * CPR), 256, 0, st>>>((const __nv_bfloat16*)v, slot_mapping, T,
                                                                        H_kv, kv->v_gscale, (uint8_t*)v_pages,
                                                                        (uint8_t*)v_scales, num_pages);
    };
    if (fmt == BDFP4_NVFP4) {
        if (d_v == 128) launch(quantize_v_kernel<BDFP4_NVFP4, 128>, VGeom<128>::RPC, VGeom<128>::CPR);
        else launch(quantize_v_kernel<BDFP4_NVFP4, 512>, VGeom<512>::RPC, VGeom<512>::CPR);
    } else {
        if (d_v == 128) launch(quantize_v_kernel<BDFP4_MXFP4, 128>, VGeom<128>::RPC, VGeom<128>::CPR);
        else launch(quantize_v_kernel<BDFP4_MXFP4, 512>, VGeom<512>::RPC, VGeom<512>::CPR);
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
