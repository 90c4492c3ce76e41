// decode_common.cuh -- arguments and split arithmetic shared by the decode
// kernels (CUDA-core path for MLA shapes, tcgen05 path for d = 128).
#pragma once

#include <cuda_runtime.h>

#include "bdfp4_device.cuh"

namespace bdfp4 {

struct DecodeArgs {
    const __nv_bfloat16* q;
    const uint8_t* k_pages;
    const uint8_t* k_scales;
    const uint8_t* v_pages;
    const uint8_t* v_scales;
    const int32_t* block_table;
    const int32_t* seq_lens;
    const float* smooth;
    const float* k_gscale;
    const float* v_gscale;
    const float* k_weight;   // [H_kv][d_k] channel weights of the key scale search, or null
    float* ws_o;   // [B][H_q][max_splits][d_v] unnormalised partial outputs
    float* ws_ml;  // [B][H_q][max_splits][2]  (m in log2 units, l)
    uint8_t* qpack;  // [B][H_kv] query images of the tensor-core path (written before the decode)
    __nv_bfloat16* out;
    int32_t* dev_status;
    int B, H_q, H_kv, max_pages, flags, chunk_tiles, max_splits;
    int append_wait;   // 1: a decode-step prologue grid writes each sequence's last page (tensor-core path)
    int T_q;           // query tokens per sequence (1: single-token decode); q, out are [B][T_q][H_q][d]
    // d = 128 tensor-core decode: the bound of every in-kernel wait (clock cycles), and the
    // unwind test's switch (1: every CTA withholds its first K tile, see bdfp4_debug.h)
    long long wait_limit;
    int test_stall;
    int64_t num_pages;
    float sm_scale;
};

// The new token of each sequence in a decode step: its key and value, and the
// bf16 values of each sequence's open beta-token value block, all appended
// into the cache (through these writable views of it) before the decode.
struct StepArgs {
    const __nv_bfloat16* k_new;   // [B][H_kv][d_k]
    const __nv_bfloat16* v_new;   // [B][H_kv][d_v]
    __nv_bfloat16* v_open;        // [B][beta][H_kv][d_v]
    uint8_t* k_pages;
    uint8_t* k_scales;
    uint8_t* v_pages;
    uint8_t* v_scales;
};

constexpr int kThreads = 128;
constexpr long long kWaitLimitDefault = 1LL << 32;   // clock cycles (about 2 s)
constexpr float kLog2e = 1.4426950408889634f;

// Workspace bytes reserved per query head for the query images of the
// tensor-core decodes (an image of a (sequence, KV head) or head slice of h
// heads takes at most h times this; each layout static_asserts it).
constexpr int kQueryImageBytes = 656;

// Row of the query, output and split-partial arrays ([B][T_q][H_q]) of stacked
// query row v of (sequence b, KV head hk): the T_q tokens' query heads of the
// KV group stack token-major, v = i G + g for token i and head g of the group.
__device__ __forceinline__ int64_t stacked_row(const DecodeArgs& a, int b, int hk, int v) {
    const int G = a.H_q / a.H_kv;
    return ((int64_t)b * a.T_q + v / G) * a.H_q + (int64_t)hk * G + v % G;
}

// Splits of a sequence of N tokens.
__host__ __device__ __forceinline__ int num_splits(int N, int chunk_tiles) {
    const int ntiles = (N + kTileTokens - 1) / kTileTokens;
    return (ntiles + chunk_tiles - 1) / chunk_tiles;
}

// Tiles per split.  Each split of c tiles of a sequence is `items` CTAs (one per
// KV head and head slice); at ctas_per_sm resident CTAs per SM the grid runs in
// ceil(CTAs / (ctas_per_sm num_sms)) waves of about c + 3 tile-times (the 3: a
// CTA's set-up, its partial write and the merge work it adds).  The plan takes the
// c in [16, 64] -- at most the longest sequence's tile count -- that minimises that
// product, the longer c on a tie (fewer partials); tiles_of(b) is sequence b's tile
// count.  Sweeps on the GQA and MLA shapes put this pick at or next to the fastest
// measured split length.
template <class TilesOf>
inline int plan_chunk_tiles(int B, const TilesOf& tiles_of, int items, int num_sms, int ctas_per_sm) {
    int max_tiles = 0;
    for (int b = 0; b < B; ++b) max_tiles = tiles_of(b) > max_tiles ? tiles_of(b) : max_tiles;
    if (max_tiles <= 16) return max_tiles < 1 ? 1 : max_tiles;
    const int64_t slots = (int64_t)(ctas_per_sm > 0 ? ctas_per_sm : 1) * (num_sms > 0 ? num_sms : 1);
    int best = 16;
    int64_t best_cost = -1;
    for (int c = 16; c <= 64 && c <= max_tiles; ++c) {
        int64_t ctas = 0;
        for (int b = 0; b < B; ++b) ctas += (tiles_of(b) + c - 1) / c;
        ctas *= items;
        const int64_t cost = (ctas + slots - 1) / slots * (c + 3);
        if (best_cost < 0 || cost <= best_cost) {
            best_cost = cost;
            best = c;
        }
    }
    return best;
}

// Which decode kernel runs a shape: G query heads per KV head, T query tokens
// per sequence (their G T rows stack per (sequence, KV head)), head dims d_k /
// d_v.
enum class DecodePath { kTensorCore128, kTensorCoreMla, kCudaCore };
inline DecodePath decode_path(int d_k, int d_v, int G, int T) {
    const int rows = G * T;
    if (d_k == 128 && d_v == 128 && rows <= 16 && (rows & (rows - 1)) == 0) return DecodePath::kTensorCore128;
    if (d_k == 576 && d_v == 512 && T == 1 && (G == 16 || G == 32 || G == 64 || G == 128))
        return DecodePath::kTensorCoreMla;
    return DecodePath::kCudaCore;
}

// Rows per CTA of the CUDA-core decode for `rows` stacked rows: the largest
// power of two up to 16 that divides them.
inline int cuda_core_rows(int rows) {
    int hg = 16;
    while (rows % hg) hg >>= 1;
    return hg;
}

// CTAs per SM and CTAs per (sequence, split, KV head) of the decode kernel that
// runs this shape (decode_path).
struct DecodeShape {
    int ctas_per_sm, items_per_kv_head;
};
inline DecodeShape decode_shape(int d_k, int d_v, int G, int T = 1) {
    switch (decode_path(d_k, d_v, G, T)) {
        case DecodePath::kTensorCore128: return {G * T <= 4 ? 4 : 3, 1};                  // decode_tc.cu
        case DecodePath::kTensorCoreMla: return {1, G > 64 ? G / 64 : 1};                   // decode_mla_tc.cu
        default: return {8, G * T / cuda_core_rows(G * T)};                                 // CUDA-core decode
    }
}

// tcgen05 decode for d_k = d_v = 128 (decode_tc.cu); returns a host status.
// With a step, one prologue grid appends the new tokens and builds the query
// images, and the decode overlaps it (programmatic dependent launch).
int launch_decode_tc(const DecodeArgs& a, int fmt, int G, cudaStream_t st, const StepArgs* step = nullptr);

// tcgen05 decode for MLA shapes (d_k = 576, d_v = 512, G in {16, 32, 64, 128};
// decode_mla_tc.cu): a prologue grid (query images, and a step's append) and
// the decode, overlapped the same way.
bool mla_tc_supported(int d_k, int d_v, int G);
int mla_query_image_bytes(int fmt, int G);
int launch_decode_mla_tc(const DecodeArgs& a, int fmt, int G, cudaStream_t st, const StepArgs* step = nullptr);

// Decode-step append on its own (quantize.cu), for the CUDA-core decode path.
int launch_step_append(const DecodeArgs& a, const StepArgs& s, int fmt, int d_k, cudaStream_t st);

}  // namespace bdfp4
