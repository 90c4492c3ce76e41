// prob_scale.cuh -- the per-tile probability pre-scale of the dynamic variant
// of the underflow-aware probability scaling (decode kernels).
#pragma once

#include <cstdint>

namespace bdfp4 {

// Exponent E of the per-tile pre-scale alpha = 2^E: the largest integer with
// p_max 2^E <= 2688 (6 x 448: the tile's largest block scale still fits E4M3),
// clamped to [11, 64].  With p_max = m 2^e, m in [1, 2), and 2688 = 1.3125 x
// 2^11: E = 11 - e, less one when m > 1.3125 -- read from the bits, so the
// decision is exact in fp32.  p_max <= 0, NaN or subnormal (below 2^-126, where
// E > 64 anyway) gives 64.
__device__ __forceinline__ int dynamic_alpha_exp(float p_max) {
    if (!(p_max > 0.0f)) return 64;
    const uint32_t u = __float_as_uint(p_max);
    const int ebits = (int)((u >> 23) & 0xffu);
    if (ebits == 0) return 64;
    const int E = 11 - (ebits - 127) - ((u & 0x7fffffu) > 0x280000u ? 1 : 0);
    return E < 11 ? 11 : (E > 64 ? 64 : E);
}

// 2^k as an fp32 for k in [-126, 127] (exact)
__device__ __forceinline__ float pow2f(int k) { return __int_as_float((127 + k) << 23); }

}  // namespace bdfp4
