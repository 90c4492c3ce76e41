// quant_device.cuh -- device steps shared by the quantizer kernels and the
// decode prologue: the key/query transform (smoothing + Hadamard), block
// quantization with its fp64 squared error, the key scale search and the
// dual-residual query quantization (BitDecoding-FP4, Article Summary).
#pragma once

#include "bdfp4_device.cuh"

namespace bdfp4 {

// Packed fp32 pairs (sm_100 f32x2 instructions: each lane an IEEE fp32 operation, round
// to nearest, subnormals kept) and an approximate reciprocal (the special-function unit,
// relative error below 2^-22; subnormal inputs and results flushed to zero).
using f32x2 = unsigned long long;
__device__ __forceinline__ f32x2 f32x2_pack(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f32x2_unpack(f32x2 v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return make_float2(lo, hi);
}
__device__ __forceinline__ f32x2 f32x2_mul(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 f32x2_fma(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ float rcp_approx_ftz(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Row geometry: threads per row (padded), active threads, segment split.
template <int FMT, int DK>
struct RowGeom {
    static constexpr int beta = Fmt<FMT>::beta;
    static constexpr int tpr = DK / beta;                        // active threads
    static constexpr int seg0 = (DK == 576) ? 512 : DK;          // first Hadamard segment
    static constexpr int seg0_thr = seg0 / beta;
    static constexpr int seg1_thr = (DK - seg0) / beta;           // rope segment threads (MLA)
    static constexpr int rt = (DK == 576) ? ((seg0_thr == 32) ? 64 : 32) : tpr;   // padded threads per row
};

// Loads `beta` bf16 values starting at element e0 of a row into x.
template <int BETA>
__device__ __forceinline__ void load_bf16_block(const __nv_bfloat16* row, int e0, float* x) {
    const uint4* p = reinterpret_cast<const uint4*>(row + e0);
#pragma unroll
    for (int v = 0; v < BETA / 8; ++v) {
        uint4 w = __ldg(p + v);
        x[8 * v + 0] = bf16_lo(w.x);
        x[8 * v + 1] = bf16_hi(w.x);
        x[8 * v + 2] = bf16_lo(w.y);
        x[8 * v + 3] = bf16_hi(w.y);
        x[8 * v + 4] = bf16_lo(w.z);
        x[8 * v + 5] = bf16_hi(w.z);
        x[8 * v + 6] = bf16_lo(w.w);
        x[8 * v + 7] = bf16_hi(w.w);
    }
}

// Smoothing + Hadamard of one thread's block (in place).  j = thread index in
// the row; all lanes of the warp must call this (shuffles are warp-wide).
template <int FMT, int DK, bool IS_KEY>
__device__ __forceinline__ void transform_block(float* x, const float* smooth_row, int j, bool hadamard) {
    using RG = RowGeom<FMT, DK>;
    constexpr int B = RG::beta;
    const int e0 = j * B;
    const bool active = j < RG::tpr;
#pragma unroll
    for (int i = 0; i < B; ++i) {
        float s = active ? __ldg(smooth_row + e0 + i) : 1.0f;
        if constexpr (IS_KEY) {
            // a power of two 2^k whose reciprocal is normal: x / 2^k and x * 2^-k round alike
            const uint32_t u = __float_as_uint(s), e = (u >> 23) & 0xffu;
            if ((u & 0x807fffffu) == 0u && e >= 1u && e <= 253u) x[i] = __fmul_rn(x[i], __uint_as_float((254u - e) << 23));
            else x[i] = __fdiv_rn(x[i], s);
        } else {
            x[i] = __fmul_rn(x[i], s);
        }
    }
    if (!hadamard) return;
    fwht_local<B>(x);
    const int seg = (j >= RG::seg0_thr) ? 1 : 0;
    const int seg_thr = seg ? RG::seg1_thr : RG::seg0_thr;
#pragma unroll
    for (int lb = 1; lb < RG::seg0_thr; lb <<= 1) {
        // every lane shuffles; only lanes whose segment spans this stage keep the result
        float y[B];
#pragma unroll
        for (int i = 0; i < B; ++i) y[i] = x[i];
        fwht_cross<B>(y, lb, 0xffffffffu);
        if (active && lb < seg_thr) {
#pragma unroll
            for (int i = 0; i < B; ++i) x[i] = y[i];
        }
    }
    const float post = hadamard_post(seg ? (DK - RG::seg0) : RG::seg0, IS_KEY);
#pragma unroll
    for (int i = 0; i < B; ++i) x[i] = __fmul_rn(x[i], post);
}

// E2M1 codes of x / sigma (sigma = 0 -> zeros), packed two per byte (even
// element low), and the block's squared error summed left to right in fp64.
// With W, element i's squared error is weighted: w[i] * (d_i * d_i).  POW2:
// sigma is a power of two and inv = 1 / sigma (exact), so x / sigma rounded to
// fp32 is x * inv rounded (both are the correctly rounded value of the same
// real quotient).
template <int B, bool W = false, bool POW2 = false>
__device__ __forceinline__ double quantize_block(const float* x, float sigma, uint32_t* packed /* B/8 words */,
                                                 const float* w = nullptr, float inv = 0.0f) {
    double err = 0.0;
#pragma unroll
    for (int k = 0; k < B / 8; ++k) packed[k] = 0u;
    const double sd = (double)sigma;
#pragma unroll
    for (int i = 0; i < B; i += 2) {
        uint32_t pair = 0u;
        if (sigma != 0.0f) {
            if constexpr (POW2) pair = e2m1x2_encode(__fmul_rn(x[i], inv), __fmul_rn(x[i + 1], inv));
            else pair = e2m1x2_encode(__fdiv_rn(x[i], sigma), __fdiv_rn(x[i + 1], sigma));
        }
        packed[i / 8] |= pair << (4 * (i % 8));
        // e sigma is exact in fp64, so x - e sigma rounds once either way
        const double d0 = __dsub_rn((double)x[i], __dmul_rn(e2m1_value_f64(pair & 15u), sd));
        const double d1 = __dsub_rn((double)x[i + 1], __dmul_rn(e2m1_value_f64(pair >> 4), sd));
        if constexpr (W) {
            err = __dadd_rn(err, __dmul_rn((double)w[i], __dmul_rn(d0, d0)));
            err = __dadd_rn(err, __dmul_rn((double)w[i + 1], __dmul_rn(d1, d1)));
        } else {
            err = __dadd_rn(err, __dmul_rn(d0, d0));
            err = __dadd_rn(err, __dmul_rn(d1, d1));
        }
    }
    return err;
}

template <int B>
__device__ __forceinline__ float block_amax(const float* x) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < B; ++i) a = fmaxf(a, fabsf(x[i]));
    return a;
}

// Exact scoring of window codes hi .. lo (those whose bit k = hi - c is set in
// `take`, taken from the largest code down): least (W: weighted) fp64 squared
// error, ties to the larger code.  Returns the code (-1 if none), `packed` its
// E2M1 codes.  The loop walks the thread's own set bits, so a warp whose
// threads take different codes runs as many iterations as its busiest thread.
template <int FMT, bool W>
__device__ __forceinline__ int search_exact(const float* x, float g, const float* w, int hi, uint32_t take,
                                            uint32_t* packed) {
    constexpr int B = Fmt<FMT>::beta;
    if (take && !(take & (take - 1u))) {
        // one code left: nothing to compare, only its elements are needed
        const int c = hi - (__ffs(take) - 1);
        const float sg = block_sigma<FMT>((uint32_t)c, g);
        if constexpr (FMT == BDFP4_MXFP4) {
            const float inv = __uint_as_float(c == 254 ? 0x00400000u : (uint32_t)(254 - c) << 23);
            quantize_block<B, false, true>(x, sg, packed, nullptr, inv);
        } else {
            quantize_block<B>(x, sg, packed);
        }
        return c;
    }
    int best = -1;
    double best_err = 0.0;
#pragma unroll 1
    while (take) {
        const int c = hi - (__ffs(take) - 1);
        take &= take - 1u;
        uint32_t cand[B / 8];
        const float sg = block_sigma<FMT>((uint32_t)c, g);
        double err;
        if constexpr (FMT == BDFP4_MXFP4) {
            // sigma = 2^(c - 127): dividing by it is multiplying by 2^(127 - c), exactly
            const float inv = __uint_as_float(c == 254 ? 0x00400000u : (uint32_t)(254 - c) << 23);
            err = quantize_block<B, W, true>(x, sg, cand, w, inv);
        } else {
            err = quantize_block<B, W>(x, sg, cand, w);
        }
        if (best < 0 || err < best_err) {
            best = c;
            best_err = err;
#pragma unroll
            for (int k = 0; k < B / 8; ++k) packed[k] = cand[k];
        }
    }
    return best;
}

// Scale search of one key block: the window NVFP4 c0+7 .. c0-2 (E4M3 codes,
// within [0, 126]) or MXFP4 c0+1, c0 (E8M0, within [0, 254]) around the plain
// code c0; least (W: weighted) squared error in fp64 summed left to right, ties
// to the larger code.  An all-zero block keeps c0.  Returns the code; `packed`
// gets its E2M1 codes.
//
// NVFP4 scores every candidate cheaply first: x times an approximate 1 / sigma
// (rcp.approx, relative error below 2^-22) for the codes, the squared error in
// fp32, two elements per packed f32x2 instruction (two partial sums).  Against
// the exact score (fp32 RN division, fp64 sums) the cheap one moves an
// element's code only within a few ulps of a rounding midpoint, where the two
// codes' errors agree to about 5e-5 relative, and rounds the sum to about 1e-6
// relative, so the exact winner always scores within 2^-10 (relative) of the
// cheapest candidate.  Only those candidates are scored exactly, in window
// order -- the same winner as scoring all of them exactly.  A candidate whose
// 1 / sigma is not finite (sigma zero or below the normal range) is always
// scored exactly.
template <int FMT, bool W>
__device__ __forceinline__ uint32_t search_scale(const float* x, float g, const float* w, uint32_t* packed) {
    constexpr int B = Fmt<FMT>::beta;
    const float amax = block_amax<B>(x);
    const int c0 = (int)plain_scale_code<FMT>(amax, g);
    if (amax == 0.0f) {
        quantize_block<B>(x, block_sigma<FMT>((uint32_t)c0, g), packed);
        return (uint32_t)c0;
    }
    const int top = FMT == BDFP4_NVFP4 ? 126 : 254;
    int hi = c0 + (FMT == BDFP4_NVFP4 ? 7 : 1);
    int lo = c0 - (FMT == BDFP4_NVFP4 ? 2 : 0);
    hi = hi > top ? top : hi;
    lo = lo < 0 ? 0 : lo;
    const uint32_t all = (1u << (hi - lo + 1)) - 1u;
    if constexpr (FMT == BDFP4_MXFP4) {
        return (uint32_t)search_exact<FMT, W>(x, g, w, hi, all, packed);
    } else {
        constexpr int NW = 10;   // window length
        float score[NW];
        uint32_t force = 0u;
        float best = INFINITY;
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            const int c = hi - k;
            score[k] = INFINITY;
            if (c < lo) continue;
            const float sg = block_sigma<FMT>((uint32_t)c, g);
            const float r = rcp_approx_ftz(sg);
            if (!(sg > 0.0f) || !(r < INFINITY)) {
                force |= 1u << k;
                continue;
            }
            const f32x2 r2 = f32x2_pack(r, r), ns2 = f32x2_pack(-sg, -sg);
            f32x2 e2 = f32x2_pack(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < B; i += 2) {
                const f32x2 xp = f32x2_pack(x[i], x[i + 1]);
                const float2 y = f32x2_unpack(f32x2_mul(xp, r2));
                const float2 v = e2m1x2_value(e2m1x2_encode(y.x, y.y));
                const f32x2 dp = f32x2_fma(f32x2_pack(v.x, v.y), ns2, xp);   // x - v sigma
                e2 = f32x2_fma(W ? f32x2_mul(f32x2_pack(w[i], w[i + 1]), dp) : dp, dp, e2);
            }
            const float2 ep = f32x2_unpack(e2);
            const float e = ep.x + ep.y;
            score[k] = e;
            best = fminf(best, e);
        }
        const float lim = best + best * (1.0f / 1024.0f);
        uint32_t take = force;
#pragma unroll
        for (int k = 0; k < NW; ++k)
            if (score[k] <= lim) take |= 1u << k;
        take &= all;
        // nothing comparable (non-finite scores): score the whole window exactly
        return (uint32_t)search_exact<FMT, W>(x, g, w, hi, take ? take : all, packed);
    }
}

// ---------------------------------------------------------------- query
// Dual-residual quantization of one query row by its row thread group.  The
// row amax (for g_q) is a max over the row's threads through shared memory.
template <int FMT, int DK>
__device__ __forceinline__ void quantize_query_block(float* x, float gq, bool dual, uint32_t& c1, uint32_t* p1,
                                                     uint32_t& c2, uint32_t* p2) {
    constexpr int B = Fmt<FMT>::beta;
    c1 = plain_scale_code<FMT>(block_amax<B>(x), gq);
    const float s1 = block_sigma<FMT>(c1, gq);
    quantize_block<B>(x, s1, p1);
    float r[B];
#pragma unroll
    for (int i = 0; i < B; ++i) {
        const uint32_t e = (p1[i / 8] >> (4 * (i % 8))) & 15u;
        r[i] = __fsub_rn(x[i], __fmul_rn(e2m1_value(e), s1));
    }
    if (dual) {
        c2 = plain_scale_code<FMT>(block_amax<B>(r), gq);
        quantize_block<B>(r, block_sigma<FMT>(c2, gq), p2);
    } else {
        c2 = 0u;
#pragma unroll
        for (int w = 0; w < B / 8; ++w) p2[w] = 0u;
    }
}

}  // namespace bdfp4
