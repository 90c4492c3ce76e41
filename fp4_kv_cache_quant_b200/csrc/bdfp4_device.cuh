// bdfp4_device.cuh -- device-side number formats, cache layout and the
// fixed fp32 transform of the FP4 KV cache (BitDecoding-FP4, "Native FP4 KV
// Cache Decoding via Algorithm-System Co-Design", Article Summary).
//
// Formats: E2M1 elements (OCP MX v1.0), E4M3FN block scales with an FP32
// tensor scale (NVFP4, 16-element blocks), E8M0 block scales (MXFP4,
// 32-element blocks).  Every operation that decides a stored code is a single
// IEEE round-to-nearest-even fp32/fp64 operation (the __f*_rn / __d*_rn
// intrinsics, never contracted into FMAs), so the quantized cache is a pure
// function of its inputs.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/bdfp4.h"

namespace bdfp4 {

constexpr int kPageSlots = 64;    // tokens per page
constexpr int kTileTokens = 128;  // tokens per online-softmax step (two pages)
constexpr float kAlphaNV = 2048.0f;  // underflow-aware probability pre-scale (NVFP4)

template <int FMT>
struct Fmt;
template <>
struct Fmt<BDFP4_NVFP4> {
    static constexpr int beta = 16;
};
template <>
struct Fmt<BDFP4_MXFP4> {
    static constexpr int beta = 32;
};

// ------------------------------------------------------------------ E2M1
// Value of a 4-bit E2M1 code (sign bit 3): 0, 0.5, 1, 1.5, 2, 3, 4, 6.  The
// normal codes m = 2..7 (1, 1.5, 2, 3, 4, 6) step by 2^22 in their fp32 bits,
// 0x3F000000 + m 2^22; code 1 is 0.5 = 0x3F000000.
__device__ __forceinline__ float e2m1_value(uint32_t code) {
    const uint32_t m = code & 7u;
    const uint32_t mag = m >= 2u ? 0x3F000000u + (m << 22) : (m ? 0x3F000000u : 0u);
    return __uint_as_float(mag | ((code & 8u) << 28));
}

// The same value as an fp64: the high word of codes 2..7 steps by 2^19 from
// 0x3FE00000 (0.5, code 1).
__device__ __forceinline__ double e2m1_value_f64(uint32_t code) {
    const uint32_t m = code & 7u;
    const uint32_t hi = m >= 2u ? 0x3FE00000u + (m << 19) : (m ? 0x3FE00000u : 0u);
    return __hiloint2double((int)(hi | ((code & 8u) << 28)), 0);
}

// Round two fp32 values to E2M1 (nearest, ties to even, saturating at +-6,
// sign kept); returns lo | hi << 4.
__device__ __forceinline__ uint32_t e2m1x2_encode(float lo, float hi) {
    uint32_t packed;
    asm volatile(
        "{\n"
        ".reg .b8 b0;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %1, %2;\n"
        "cvt.u32.u8 %0, b0;\n"
        "}\n"
        : "=r"(packed)
        : "f"(hi), "f"(lo));
    return packed;   // cvt.u32.u8 zero-extends
}

__device__ __forceinline__ uint32_t e2m1_encode(float x) { return e2m1x2_encode(x, 0.0f) & 0xfu; }

// Eight fp32 values to E2M1 (nearest, ties to even, saturating at +-6, sign kept),
// packed v[0] in bits 0..3 up to v[7] in bits 28..31 (the byte order of a K-major row).
__device__ __forceinline__ uint32_t e2m1x8_encode(const float* v) {
    uint32_t r;
    asm("{\n .reg .b8 b0, b1, b2, b3;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
        " mov.b32 %0, {b0, b1, b2, b3};\n}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Values of the E2M1 pair lo | hi << 4 (as e2m1x2_encode packs it) through the
// hardware conversion: .x the low code's, .y the high code's (exact: E2M1 is a
// subset of fp16).
__device__ __forceinline__ float2 e2m1x2_value(uint32_t pair) {
    uint32_t h2;
    asm("{\n .reg .b8 t;\n .reg .b16 u;\n cvt.u16.u32 u, %1;\n cvt.u8.u16 t, u;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}\n"
        : "=r"(h2)
        : "r"(pair));
    return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// ------------------------------------------------------------------ E4M3
// Value of an E4M3FN code (0..0x7e used; bias 7, subnormals m * 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    uint32_t e = (code >> 3) & 15u, m = code & 7u;
    float mag = (e == 0) ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return (code & 0x80u) ? -mag : mag;
}

// E4M3 value through the hardware conversion (exact: E4M3 is a subset of fp16).
__device__ __forceinline__ float e4m3_value_hw(uint32_t code) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(code & 0xffu)));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

// Unsigned E4M3 encode: nearest, ties to even, >= 448 saturates to 448.
__device__ __forceinline__ uint32_t e4m3_encode(float u) {
    uint16_t packed;
    asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(packed) : "f"(0.0f), "f"(u));
    return packed & 0xffu;
}

// ------------------------------------------------------------------ E8M0
__device__ __forceinline__ float e8m0_value(uint32_t code) {
    // 2^(code - 127); codes 0 and 1 are fp32 subnormals 2^-127, 2^-126 (normal)
    return code == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(code << 23);
}

// OCP MX shared scale: 2^(floor(log2 amax) - 2) clamped to E8M0; 0 -> code 0.
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
    if (amax == 0.0f) return 0u;
    int E;
    frexpf(amax, &E);  // amax = f 2^E, f in [0.5, 1)
    int code = (E - 1) - 2 + 127;
    code = code < 0 ? 0 : (code > 254 ? 254 : code);
    return (uint32_t)code;
}

// fp32 divisor of block scale code c (NVFP4: fp32(E4M3(c) * g); MXFP4: 2^(c-127)).
template <int FMT>
__device__ __forceinline__ float block_sigma(uint32_t code, float g) {
    if constexpr (FMT == BDFP4_NVFP4) return __fmul_rn(e4m3_value(code), g);
    else return e8m0_value(code);
}

template <int FMT>
__device__ __forceinline__ float scale_value(uint32_t code) {
    if constexpr (FMT == BDFP4_NVFP4) return e4m3_value(code);
    else return e8m0_value(code);
}

// Plain scale rule: NVFP4 E4M3(fp32(amax / fp32(6 g))) (0 = all-zero block);
// MXFP4 the OCP MX shared exponent.
template <int FMT>
__device__ __forceinline__ uint32_t plain_scale_code(float amax, float g) {
    if constexpr (FMT == BDFP4_NVFP4) {
        if (amax == 0.0f) return 0u;
        return e4m3_encode(__fdiv_rn(amax, __fmul_rn(6.0f, g)));
    } else {
        return mx_scale_code(amax);
    }
}

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ------------------------------------------------------------------ layout
// Byte offsets within one (page, head) block of the cache; see bdfp4.h.
__device__ __forceinline__ uint32_t k_nib_offset(int d_k, int slot, int e) {
    return (uint32_t)((slot >> 3) * (d_k / 32) * 128 + (e >> 5) * 128 + (slot & 7) * 16 + ((e & 31) >> 1));
}
// K scales: four consecutive block codes of a slot share a 32-bit word;
// [blk/4][slot%32][slot/32][blk%4] in 256-byte chunks.
__host__ __device__ __forceinline__ int k_scale_page_bytes(int d_k, int beta) { return 256 * ((d_k / beta + 3) / 4); }
template <int BETA>
__device__ __forceinline__ uint32_t k_scale_offset(int d_k, int slot, int blk) {
    (void)d_k;
    return (uint32_t)((blk >> 2) * 256 + (slot & 31) * 8 + (slot >> 5) * 4 + (blk & 3));
}
__device__ __forceinline__ uint32_t v_nib_offset(int chan, int slot) {
    return (uint32_t)((chan >> 3) * 256 + (slot >> 5) * 128 + (chan & 7) * 16 + ((slot & 31) >> 1));
}
template <int BETA>
__device__ __forceinline__ uint32_t v_scale_offset(int chan, int blk) {
    constexpr int per_chan = kPageSlots / BETA;
    return (uint32_t)((chan >> 7) * (128 * per_chan) + (chan & 31) * (4 * per_chan) + ((chan & 127) >> 5) * per_chan +
                      blk);
}

// ------------------------------------------------------------------ transform
// Hadamard post-scale of a segment of length 2^L: keys 2^-ceil(L/2), queries 2^-floor(L/2).
__device__ __forceinline__ float hadamard_post(int seg_len, bool is_key) {
    int L = 31 - __clz(seg_len);
    int sh = is_key ? (L + 1) / 2 : L / 2;
    return __uint_as_float((uint32_t)(127 - sh) << 23);
}

// In-thread butterflies over n contiguous values (stages h = 1 .. n/2).
template <int N>
__device__ __forceinline__ void fwht_local(float* x) {
#pragma unroll
    for (int h = 1; h < N; h <<= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            if ((i & h) == 0) {
                float a = x[i], b = x[i + h];
                x[i] = __fadd_rn(a, b);
                x[i + h] = __fsub_rn(a, b);
            }
        }
    }
}

// Cross-thread butterfly stage: the thread whose group index has bit `lanebit`
// clear keeps a + b, the other keeps a - b, a being the lower-index value.
template <int N>
__device__ __forceinline__ void fwht_cross(float* x, int lanebit, unsigned mask) {
    const bool upper = (threadIdx.x & lanebit) != 0;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        float other = __shfl_xor_sync(mask, x[i], lanebit);
        float a = upper ? other : x[i];
        float b = upper ? x[i] : other;
        x[i] = upper ? __fsub_rn(a, b) : __fadd_rn(a, b);
    }
}

__device__ __forceinline__ void set_status(int32_t* dev_status, int bit) {
    if (dev_status) atomicOr(dev_status, bit);
}

}  // namespace bdfp4
