// merge.cuh -- log-sum-exp merge of split-KV partial outputs, shared by the
// FP4 and BF16 decode paths.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "decode_common.cuh"

namespace bdfp4 {

// One CTA (128 threads) per (sequence, query head) row with more than one split:
//   out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
template <int DV>
__global__ void __launch_bounds__(128) merge_splits_kernel(const float* __restrict__ ws_o,
                                                           const float* __restrict__ ws_ml,
                                                           const int32_t* __restrict__ seq_lens, int H_q,
                                                           int max_pages, int chunk_tiles, int max_splits,
                                                           __nv_bfloat16* out) {
    // launched as a programmatic dependent of the decode grid: wait for its partials
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int row = blockIdx.x;
    const int b = row / H_q;
    int N = seq_lens[b];
    if (N < 0 || N > max_pages * kPageSlots) N = 0;
    const int ns = num_splits(N, chunk_tiles);
    if (ns <= 1) return;   // written by the decode kernel
    // split weights 2^(m_s - M) and L = sum_s 2^(m_s - M) l_s, every split's (m, l) pair
    // loaded by its own thread (the loads overlap instead of following one another)
    extern __shared__ float sw[];   // [ns] weights
    __shared__ float red[2][4];
    const float* ml = ws_ml + (int64_t)row * max_splits * 2;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    float M = -INFINITY;
    for (int s = threadIdx.x; s < ns; s += blockDim.x) M = fmaxf(M, ml[2 * s]);
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) red[0][wid] = M;
    __syncthreads();
    M = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
    // every split saw only masked tokens (all of the sequence's pages bad): m = -inf
    // everywhere, so take 0 as the reference -- the weights become 0, L = 0 and the
    // row is written as zeros, as a single-split row is
    if (M == -INFINITY) M = 0.0f;
    float Lp = 0.0f;
    for (int s = threadIdx.x; s < ns; s += blockDim.x) {
        const float w = exp2f(ml[2 * s] - M);
        sw[s] = w;
        Lp += ml[2 * s + 1] * w;
    }
    for (int off = 16; off > 0; off >>= 1) Lp += __shfl_xor_sync(0xffffffffu, Lp, off);
    if (lane == 0) red[1][wid] = Lp;
    __syncthreads();
    const float L = (red[1][0] + red[1][1]) + (red[1][2] + red[1][3]);
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    for (int c = threadIdx.x; c < DV; c += blockDim.x) {
        const float* o = ws_o + (int64_t)row * max_splits * DV + c;
        float acc = 0.0f;
#pragma unroll 4
        for (int s = 0; s < ns; ++s) acc += o[(int64_t)s * DV] * sw[s];
        out[(int64_t)row * DV + c] = __float2bfloat16(acc * inv);
    }
}

// Dynamic shared memory of merge_splits_kernel: a weight per split.
inline size_t merge_smem(int max_splits) { return (size_t)max_splits * sizeof(float); }

// Launches the merge as a programmatic dependent of the decode grid just before
// it on the stream: its CTAs are scheduled as the decode's last CTAs retire and
// wait (griddepcontrol.wait) for the whole decode grid, so the launch latency
// overlaps the decode's tail.  Returns the CUDA launch status.
template <int DV>
inline cudaError_t launch_merge(const float* ws_o, const float* ws_ml, const int32_t* seq_lens, int B, int H_q,
                                int max_pages, int chunk_tiles, int max_splits, __nv_bfloat16* out, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(B * H_q);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = merge_smem(max_splits);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, merge_splits_kernel<DV>, ws_o, ws_ml, seq_lens, H_q, max_pages, chunk_tiles,
                              max_splits, out);
}

}  // namespace bdfp4
