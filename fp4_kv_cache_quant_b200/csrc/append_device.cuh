// append_device.cuh -- the KV-append quantizers as CTA-level device functions
// (BitDecoding-FP4, Article Summary: Outlier-Aware Key Quantization; values
// take the plain block rule), shared by the stand-alone append kernels and the
// fused decode-step prologue.  Each function does the work of one CTA of 256
// threads, given its block index inside its own role.
#pragma once

#include "bdfp4_device.cuh"
#include "quant_device.cuh"

namespace bdfp4 {

// ---------------------------------------------------------------- keys
// Work split of the K append: one thread per scale block of a row (its beta
// channels), R rows per 256-thread CTA; the thread transforms its block and
// searches the block's whole window itself, so nothing leaves registers.
template <int FMT, int DK>
struct KGeom {
    using RG = RowGeom<FMT, DK>;
    static constexpr int B = RG::beta;
    static constexpr int NB = DK / B;                                  // scale blocks per row
    static constexpr int R = 256 / RG::rt;                             // rows per CTA
    static_assert(256 % RG::rt == 0, "rows tile the CTA");
};

// Slot of token t from a slot mapping (page * 64 + slot, negative = skip);
// slots past the cache are reported and skipped.
struct MappedSlot {
    const int64_t* slot_mapping;
    int64_t num_pages;
    int32_t* dev_status;
    __device__ __forceinline__ int64_t operator()(int t, bool report) const {
        const int64_t sm = __ldg(slot_mapping + t);
        if (sm >= num_pages * kPageSlots) {
            if (report) set_status(dev_status, BDFP4_DEV_BAD_SLOT);
            return -1;
        }
        return sm;
    }
};

// Slot of the newest token of sequence t in a decode step: position N - 1 of
// the sequence (N = seq_lens[t] counts the new token), through its block table
// row.  Empty or over-long sequences append nothing (the decode reports the
// latter); a page id outside the cache is reported and skipped.
struct NewestSlot {
    const int32_t* block_table;
    const int32_t* seq_lens;
    int max_pages;
    int64_t num_pages;
    int32_t* dev_status;
    __device__ __forceinline__ int64_t operator()(int t, bool report) const {
        const int N = __ldg(seq_lens + t);
        if (N <= 0 || N > max_pages * kPageSlots) return -1;
        const int pg = __ldg(block_table + (int64_t)t * max_pages + (N - 1) / kPageSlots);
        if (pg < 0 || pg >= num_pages) {
            if (report) set_status(dev_status, BDFP4_DEV_BAD_PAGE);
            return -1;
        }
        return (int64_t)pg * kPageSlots + (N - 1) % kPageSlots;
    }
};

// Key rows [blk * R, blk * R + R) of k [rows / H_kv][H_kv][DK] (row = token *
// H_kv + head).  Each thread transforms its scale block (butterflies across
// the row's threads, which share a warp), then quantizes the block under every
// code of its window in turn, keeping the least fp64 squared error (summed left
// to right; with k_weight, each element's term weighted by its channel's
// weight) and the larger code on a tie -- the sequential search -- and stores
// the winner.  k_weight [H_kv][DK] or null (the plain objective).
template <int FMT, int DK, class SlotOf>
__device__ __forceinline__ void append_k_cta(int blk, const __nv_bfloat16* __restrict__ k, int64_t rows, int H_kv,
                                             const SlotOf& slot_of, const float* __restrict__ smooth,
                                             const float* __restrict__ k_gscale, const float* __restrict__ k_weight,
                                             uint8_t* k_pages, uint8_t* k_scales, int flags) {
    using KG = KGeom<FMT, DK>;
    using RG = typename KG::RG;
    constexpr int B = KG::B;
    const int r = threadIdx.x / RG::rt, j = threadIdx.x % RG::rt;
    const int64_t row = (int64_t)blk * KG::R + r;
    const bool in_range = row < rows;
    const int t = (int)(in_range ? row / H_kv : 0);
    const int h = (int)(in_range ? row % H_kv : 0);
    const int64_t sm = in_range ? slot_of(t, j == 0) : -1;
    // whole warps stay converged through the shuffles; inactive rows compute on zeros.
    // The row is loaded whatever its slot id, so the two loads overlap
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
    transform_block<FMT, DK, true>(x, smooth + (int64_t)h * DK, j, !(flags & BDFP4_FLAG_NO_HADAMARD));
    if (sm < 0 || j >= RG::tpr) return;
    const float g = FMT == BDFP4_NVFP4 ? __ldg(k_gscale + h) : 1.0f;
    uint32_t pk[B / 8];
    uint32_t code;
    if (flags & BDFP4_FLAG_NO_SCALE_SEARCH) {
        code = plain_scale_code<FMT>(block_amax<B>(x), g);
        quantize_block<B>(x, block_sigma<FMT>(code, g), pk);
    } else if (k_weight) {
        float w[B];
#pragma unroll
        for (int i = 0; i < B; ++i) w[i] = __ldg(k_weight + (int64_t)h * DK + j * B + i);
        code = search_scale<FMT, true>(x, g, w, pk);
    } else {
        code = search_scale<FMT, false>(x, g, nullptr, pk);
    }
    const int64_t page = sm / kPageSlots;
    const int slot = (int)(sm % kPageSlots);
    uint8_t* kp = k_pages + (page * H_kv + h) * (int64_t)(kPageSlots * DK / 2);
    uint8_t* dst = kp + k_nib_offset(DK, slot, j * B);
    if constexpr (B == 16) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
    } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    uint8_t* ks = k_scales + (page * H_kv + h) * (int64_t)k_scale_page_bytes(DK, B);
    ks[k_scale_offset<B>(DK, slot, j)] = (uint8_t)code;
}

// Low-latency K append for few rows (a decode step's new tokens): every scale
// block of a row gets NC lanes, one per candidate code of its search window, so
// the window is scored in parallel -- each lane quantizes the block under its
// code exactly (fp32 RN division, fp64 error left to right) -- and a shuffle
// argmin over the block's lanes keeps the least error, the larger code on a
// tie, as the sequential search.  R rows share a 256-thread CTA.
template <int FMT, int DK>
struct KWideGeom {
    using RG = RowGeom<FMT, DK>;
    static constexpr int B = RG::beta;
    static constexpr int NB = DK / B;                                  // scale blocks per row
    static constexpr int NC = FMT == BDFP4_NVFP4 ? 16 : 2;             // candidate lanes per block (10 or 2 used)
    static constexpr int R = 256 / (NB * NC) >= 1 ? 256 / (NB * NC) : 1;
    static constexpr int PAIRS = R * NB * NC;                          // (block, candidate) lanes
    static constexpr int T1 = (R * RG::rt + 31) / 32 * 32;             // transform threads (whole warps)
    static_assert(T1 <= 256 && 32 % NC == 0, "work split");
};

template <int FMT, int DK, class SlotOf>
__device__ __forceinline__ void append_k_cta_wide(int blk, const __nv_bfloat16* __restrict__ k, int64_t rows,
                                                  int H_kv, const SlotOf& slot_of, const float* __restrict__ smooth,
                                                  const float* __restrict__ k_gscale,
                                                  const float* __restrict__ k_weight, uint8_t* k_pages,
                                                  uint8_t* k_scales, int flags) {
    using KG = KWideGeom<FMT, DK>;
    using RG = typename KG::RG;
    constexpr int B = KG::B, NB = KG::NB, NC = KG::NC, R = KG::R;
    __shared__ float xs[R][DK];
    __shared__ long long slots[R];
    __shared__ float gs[R];
    const int tid = threadIdx.x;
    const int64_t row0 = (int64_t)blk * R;
    // phase 1: the rows' transform into shared memory (thread per block)
    if (tid < KG::T1) {
        const int r = tid / RG::rt, j = tid % RG::rt;
        const int64_t row = row0 + r;
        const bool in_range = r < R && row < rows;
        const int t = (int)(in_range ? row / H_kv : 0);
        const int h = (int)(in_range ? row % H_kv : 0);
        const int64_t sm = in_range ? slot_of(t, j == 0) : -1;
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
        transform_block<FMT, DK, true>(x, smooth + (int64_t)h * DK, j, !(flags & BDFP4_FLAG_NO_HADAMARD));
        if (sm >= 0 && j < RG::tpr) {
#pragma unroll
            for (int i = 0; i < B; ++i) xs[r][j * B + i] = x[i];
        }
        if (r < R && j == 0) {
            slots[r] = sm;
            gs[r] = FMT == BDFP4_NVFP4 ? __ldg(k_gscale + h) : 1.0f;
        }
    }
    __syncthreads();
    // phase 2: lane (row, block, candidate); whole warps take part in the shuffles
    for (int p0 = 0; p0 < KG::PAIRS; p0 += 256) {
        const int p = p0 + tid;
        const bool live = p < KG::PAIRS;
        const int r = live ? p / (NB * NC) : 0, bk = live ? (p / NC) % NB : 0, ci = p % NC;
        const int64_t sm = live ? slots[r] : -1;
        const float g = gs[r];
        float x[B];
#pragma unroll
        for (int i = 0; i < B; ++i) x[i] = xs[r][bk * B + i];
        const int h = (int)((row0 + r) % H_kv);
        const float amax = block_amax<B>(x);
        const int c0 = (int)plain_scale_code<FMT>(amax, g);
        int hi = c0, lo = c0;   // all-zero blocks and the plain rule keep c0
        if (amax != 0.0f && !(flags & BDFP4_FLAG_NO_SCALE_SEARCH)) {
            const int top = FMT == BDFP4_NVFP4 ? 126 : 254;
            hi = min(c0 + (FMT == BDFP4_NVFP4 ? 7 : 1), top);
            lo = max(c0 - (FMT == BDFP4_NVFP4 ? 2 : 0), 0);
        }
        const int c = hi - ci;
        uint32_t pk[B / 8];
        double err = INFINITY;
        if (sm >= 0 && c >= lo) {
            if (k_weight) {
                float w[B];
#pragma unroll
                for (int i = 0; i < B; ++i) w[i] = __ldg(k_weight + (int64_t)h * DK + bk * B + i);
                err = quantize_block<B, true>(x, block_sigma<FMT>((uint32_t)c, g), pk, w);
            } else {
                err = quantize_block<B>(x, block_sigma<FMT>((uint32_t)c, g), pk);
            }
        }
        // argmin over the block's NC lanes: least error, then smallest ci (the larger code)
        double be = err;
        int bci = ci;
#pragma unroll
        for (int off = NC / 2; off > 0; off >>= 1) {
            const double oe = __shfl_xor_sync(0xffffffffu, be, off);
            const int oc = __shfl_xor_sync(0xffffffffu, bci, off);
            if (oe < be || (oe == be && oc < bci)) {
                be = oe;
                bci = oc;
            }
        }
        if (sm >= 0 && ci == bci) {
            const int64_t page = sm / kPageSlots;
            const int slot = (int)(sm % kPageSlots);
            uint8_t* dst = k_pages + (page * H_kv + h) * (int64_t)(kPageSlots * DK / 2) + k_nib_offset(DK, slot, bk * B);
            if constexpr (B == 16) {
                *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
            } else {
                *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            k_scales[(page * H_kv + h) * (int64_t)k_scale_page_bytes(DK, B) + k_scale_offset<B>(DK, slot, bk)] =
                (uint8_t)c;
        }
    }
}

// ---------------------------------------------------------------- values
// One thread per (row, channel): TPR threads of a row per CTA, RPC rows per
// CTA, CPR CTAs per row.
template <int DV>
struct VGeom {
    static constexpr int TPR = DV < 256 ? DV : 256;   // threads of a row in one CTA
    static constexpr int RPC = 256 / TPR;             // rows per CTA
    static constexpr int CPR = DV / TPR;              // CTAs per row
};

// Decode-step value append for rows (sequence b, head h) = blk's rows of the
// [B][H_kv] grid.  v_open [B][beta][H_kv][DV] bf16 holds each sequence's open
// beta-token block (row i = slot first + i of the block that holds position
// N - 1): the new value v_new [B][H_kv][DV] goes into row (N - 1) % beta, and
// the block is quantized from rows 0 .. (N - 1) % beta (later slots of the
// block become zero), exactly as the append of that run of tokens.
template <int FMT, int DV>
__device__ __forceinline__ void append_v_open_cta(int blk, const __nv_bfloat16* __restrict__ v_new,
                                                  __nv_bfloat16* v_open, const NewestSlot& slot_of, int nseq,
                                                  int H_kv, const float* __restrict__ v_gscale, uint8_t* v_pages,
                                                  uint8_t* v_scales) {
    constexpr int B = Fmt<FMT>::beta;
    using VG = VGeom<DV>;
    const int64_t row = (int64_t)(blk / VG::CPR) * VG::RPC + threadIdx.x / VG::TPR;
    const int c = (int)(blk % VG::CPR) * VG::TPR + threadIdx.x % VG::TPR;
    if (row >= (int64_t)nseq * H_kv) return;
    const int b = (int)(row / H_kv), h = (int)(row % H_kv);
    // the whole open block and the new value are loaded with the slot lookup in flight
    const unsigned short* ob = reinterpret_cast<const unsigned short*>(v_open);
    const unsigned short vn = __ldg(reinterpret_cast<const unsigned short*>(v_new) + row * DV + c);
    uint32_t raw[B];
#pragma unroll
    for (int i = 0; i < B; ++i) raw[i] = ob[(((int64_t)b * B + i) * H_kv + h) * DV + c];
    const int64_t sm = slot_of(b, false);
    if (sm < 0) return;
    const int slot = (int)(sm % kPageSlots);
    const int last = slot % B;   // row of the new value in the open block
    const int first = slot - last;
    reinterpret_cast<unsigned short*>(v_open)[(((int64_t)b * B + last) * H_kv + h) * DV + c] = vn;
    float x[B];
#pragma unroll
    for (int i = 0; i < B; ++i) {
        const uint32_t w = i == last ? (uint32_t)vn : raw[i];
        x[i] = i <= last ? __uint_as_float(w << 16) : 0.0f;
    }
    const float g = FMT == BDFP4_NVFP4 ? __ldg(v_gscale + h) : 1.0f;
    const uint32_t code = plain_scale_code<FMT>(block_amax<B>(x), g);
    uint32_t packed[B / 8];
    quantize_block<B>(x, block_sigma<FMT>(code, g), packed);
    const int64_t page = sm / kPageSlots;
    uint8_t* vp = v_pages + (page * H_kv + h) * (int64_t)(DV * kPageSlots / 2);
    uint8_t* vs = v_scales + (page * H_kv + h) * (int64_t)(DV * kPageSlots / B);
    uint8_t* dst = vp + v_nib_offset(c, first);
    if constexpr (B == 16) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    vs[v_scale_offset<B>(c, first / B)] = (uint8_t)code;
}

// CTAs of each append role for nrows (token, head) rows.
template <int FMT, int DK>
__host__ __device__ constexpr int64_t k_append_ctas(int64_t nrows) {
    return (nrows + KGeom<FMT, DK>::R - 1) / KGeom<FMT, DK>::R;
}
template <int FMT, int DK>
__host__ __device__ constexpr int64_t k_append_ctas_wide(int64_t nrows) {
    return (nrows + KWideGeom<FMT, DK>::R - 1) / KWideGeom<FMT, DK>::R;
}
template <int DV>
__host__ __device__ constexpr int64_t v_append_ctas(int64_t nrows) {
    return (nrows + VGeom<DV>::RPC - 1) / VGeom<DV>::RPC * VGeom<DV>::CPR;
}

}  // namespace bdfp4
