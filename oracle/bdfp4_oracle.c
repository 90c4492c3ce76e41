/*
 * bdfp4_oracle.c -- CPU oracle for native-FP4 paged decode attention.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and
 * the CPU-baseline leg of the benchmark may load this library.  It shares no
 * code, header, table or helper with the CUDA library: every format, layout
 * and step below is written out again here from its definition.
 *
 * It is a plain, slow restatement of what the method computes, in the order
 * the pages give it, with every floating-point decision spelled out:
 *   - fp32 steps that decide an integer code (the rotation, the scale codes,
 *     the E2M1 codes of K, V and q) are done in fp32 with one IEEE
 *     round-to-nearest-even operation per C operator (build with
 *     -ffp-contract=off, no fast-math), so the CUDA path can match them bit
 *     for bit;
 *   - everything else (logits, softmax, probabilities and their FP4
 *     quantization, the attention sums, the split merge) is done in fp64.
 *
 * Sources, by page title and section:
 *   [ABS]  "BitDecoding-FP4: Native FP4 KV Cache Decoding via Algorithm-System
 *          Co-Design" -- Article Summary (the paper's abstract): NVFP4/MXFP4
 *          KV cache, Dual-Residual Query Quantization, Underflow-Aware
 *          Probability Scaling with E4M3 scales, Outlier-Aware Key
 *          Quantization (static smoothing + Hadamard rotation + scale search)
 *          under token-wise scaling, transposed softmax with fused probability
 *          quantization, stacked query MMA on paged KV caches.
 *   [SNS]  "BitDecoding-FP4 : decodage natif du KV cache FP4" -- "Analyse
 *          approfondie": the second query tensor encodes the residual left by
 *          the first; a block whose E4M3 probability scale rounds to zero
 *          collapses; smoothing and rotation spread outlier energy before the
 *          scale search picks a better factor per group.
 *   [BLOG] "FP4 KV Cache Done Right: What BitDecoding-FP4 Changes for
 *          Long-Context Serving" -- "What is actually new in BitDecoding-FP4?"
 *   Number formats: OCP Microscaling Formats (MX) v1.0 (E2M1 elements, E8M0
 *   shared scale, 32-element blocks) and the OCP 8-bit floating point
 *   specification (E4M3FN); NVFP4 = E2M1 elements in 16-element blocks with
 *   an E4M3 block scale and an FP32 tensor scale.
 *
 * Where the pages leave a step open, the reading used is stated at the step;
 * the CUDA library applies the same readings.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORA_NVFP4 0
#define ORA_MXFP4 1

#define ORA_FLAG_NO_HADAMARD     1   /* ablation: no rotation of K and q          */
#define ORA_FLAG_NO_SCALE_SEARCH 2   /* ablation: plain amax rule for K blocks     */
#define ORA_FLAG_SINGLE_QUERY    4   /* ablation: q2 = 0 (vanilla single FP4 query) */
#define ORA_FLAG_NO_UNDERFLOW    8   /* ablation: alpha = 1 (vanilla P scaling)    */
#define ORA_FLAG_EXACT_P        16   /* oracle only: probabilities left unquantized,
                                        to pin the softmax against textbook attention */
#define ORA_FLAG_DYNAMIC_ALPHA  32   /* variant: alpha chosen per tile and head     */

#define PAGE_SLOTS 64   /* tokens per KV page                       */
#define TILE_TOKENS 128 /* tokens per online-softmax step (2 pages) */

/* =========================================================================
 * 1. Number formats
 * ========================================================================= */

/* E2M1 (OCP MX v1.0): sign bit 3, two exponent bits, one mantissa bit. */
static const double e2m1_magnitude[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double ora_e2m1_value(int code)
{
    double m = e2m1_magnitude[code & 7];
    return (code & 8) ? -m : m;
}

/* Round to the nearest E2M1 magnitude, ties to the even code, saturating at 6;
 * the sign bit is kept, so a negative value that rounds to zero gives -0 (8). */
int ora_e2m1_encode(double x)
{
    double a = fabs(x);
    int best = 7;
    if (!(a >= 6.0)) {
        double best_d = a;
        best = 0;
        for (int c = 1; c < 8; ++c) {
            double d = fabs(a - e2m1_magnitude[c]);
            if (d < best_d || (d == best_d && (c & 1) == 0)) {
                best = c;
                best_d = d;
            }
        }
    }
    return signbit(x) ? (best | 8) : best;
}

/* E4M3FN (OCP 8-bit FP): bias 7, no infinities, S.1111.111 is NaN, max 448,
 * subnormals m * 2^-9. */
double ora_e4m3_value(int code)
{
    int e = (code >> 3) & 15, m = code & 7;
    double v;
    if ((code & 0x7f) == 0x7f) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -v : v;
}

static double e4m3_table[128];
static int tables_ready = 0;

static void init_tables(void)
{
    if (tables_ready) return;
    for (int c = 0; c < 128; ++c) e4m3_table[c] = ora_e4m3_value(c);
    tables_ready = 1;
}

/* Unsigned E4M3 encode (block scales are never negative): nearest finite
 * code, ties to the even code, values at or above 448 saturate to 448. */
int ora_e4m3_encode(double u)
{
    init_tables();
    if (u >= 448.0) return 0x7e;
    int best = 0;
    double best_d = fabs(u);
    for (int c = 1; c <= 0x7e; ++c) {
        double d = fabs(u - e4m3_table[c]);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return best;
}

/* E8M0 (OCP MX v1.0): 2^(code-127), 0xFF is NaN. */
double ora_e8m0_value(int code)
{
    if (code == 0xff) return NAN;
    return ldexp(1.0, code - 127);
}

/* MX shared scale (OCP MX v1.0, conversion rule): X = 2^(floor(log2 amax) - 2),
 * 2 being the largest exponent of E2M1; clamped to the E8M0 range.  An
 * all-zero block takes code 0. */
int ora_mx_scale_code(double amax)
{
    if (amax == 0.0) return 0;
    int E;
    frexp(amax, &E);            /* amax = f * 2^E, f in [0.5, 1) */
    int code = (E - 1) - 2 + 127;
    if (code < 0) code = 0;
    if (code > 254) code = 254;
    return code;
}

/* bf16 <-> float */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp64 -> bf16, round to nearest even (NaN not expected). */
uint16_t ora_f64_to_bf16(double x)
{
    if (x == 0.0) return signbit(x) ? 0x8000 : 0;
    int neg = x < 0;
    double a = fabs(x);
    int E;
    frexp(a, &E);                   /* a in [2^(E-1), 2^E) */
    int e = E - 1;
    if (e < -126) e = -126;         /* bf16 subnormal spacing 2^-133 */
    double ulp = ldexp(1.0, e - 7);
    double q = a / ulp;             /* exact: scaling by a power of two */
    double fl = floor(q);
    double r = q - fl;
    double n = fl;
    if (r > 0.5 || (r == 0.5 && fmod(fl, 2.0) != 0.0)) n = fl + 1.0;
    double v = n * ulp;
    float f = (float)v;             /* exact: v has <= 9 significant bits */
    if (v >= 3.3895313892515355e38) f = INFINITY;
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t h = (uint16_t)(u >> 16);
    return neg ? (uint16_t)(h | 0x8000) : h;
}

/* =========================================================================
 * 2. Cache layout (the library's ABI), written out from its definition.
 *    A page holds 64 token slots for every KV head.
 * ========================================================================= */

/* K nibbles of (page, head): 64 slots x d_k elements, stored as 8-slot x
 * 32-element core blocks of 128 bytes: [slot/8][elem/32][slot%8][16 bytes],
 * two elements per byte, the even element in the low nibble. */
static size_t k_nib_byte(int64_t page, int head, int H_kv, int d_k, int slot, int e)
{
    size_t base = ((size_t)page * H_kv + head) * (size_t)(PAGE_SLOTS * d_k / 2);
    size_t in = (size_t)(slot / 8) * (size_t)(d_k / 32) * 128 + (size_t)(e / 32) * 128
              + (size_t)(slot % 8) * 16 + (size_t)((e % 32) / 2);
    return base + in;
}

/* K scales of (page, head): groups of four consecutive block codes of a slot
 * share a 4-byte word; 256-byte chunks per group index:
 * [blk/4][slot%32][slot/32][blk%4], i.e. 64 * 4 * ceil(d_k / (4 beta)) bytes
 * per (page, head). */
static size_t k_scale_page_bytes(int d_k, int beta)
{
    return (size_t)256 * (size_t)((d_k / beta + 3) / 4);
}

static size_t k_scale_byte(int64_t page, int head, int H_kv, int d_k, int beta, int slot, int blk)
{
    size_t base = ((size_t)page * H_kv + head) * k_scale_page_bytes(d_k, beta);
    size_t in = (size_t)(blk / 4) * 256 + (size_t)(slot % 32) * 8 + (size_t)(slot / 32) * 4 + (size_t)(blk % 4);
    return base + in;
}

/* V nibbles of (page, head): d_v channels x 64 slots, stored as 8-channel x
 * 32-slot core blocks of 128 bytes: [chan/8][slot/32][chan%8][16 bytes], two
 * slots per byte, the even slot in the low nibble. */
static size_t v_nib_byte(int64_t page, int head, int H_kv, int d_v, int chan, int slot)
{
    size_t base = ((size_t)page * H_kv + head) * (size_t)(d_v * PAGE_SLOTS / 2);
    size_t in = (size_t)(chan / 8) * 256 + (size_t)(slot / 32) * 128
              + (size_t)(chan % 8) * 16 + (size_t)((slot % 32) / 2);
    return base + in;
}

/* V scales of (page, head): 64/beta codes per channel (one per beta slots):
 * [chan/128][chan%32][(chan%128)/32][block]. */
static size_t v_scale_byte(int64_t page, int head, int H_kv, int d_v, int beta, int chan, int blk)
{
    int per_chan = PAGE_SLOTS / beta;
    size_t base = ((size_t)page * H_kv + head) * (size_t)(d_v * per_chan);
    size_t in = (size_t)(chan / 128) * (size_t)(128 * per_chan) + (size_t)(chan % 32) * (size_t)(4 * per_chan)
              + (size_t)((chan % 128) / 32) * (size_t)per_chan + (size_t)blk;
    return base + in;
}

static void put_nibble(uint8_t* buf, size_t byte, int high, int code)
{
    if (high) buf[byte] = (uint8_t)((buf[byte] & 0x0f) | ((code & 15) << 4));
    else buf[byte] = (uint8_t)((buf[byte] & 0xf0) | (code & 15));
}

static int get_nibble(const uint8_t* buf, size_t byte, int high)
{
    return high ? (buf[byte] >> 4) & 15 : buf[byte] & 15;
}

/* =========================================================================
 * 3. Outlier-aware key transform: static smoothing + Hadamard rotation
 *    ([ABS]; [SNS]: smoothing and rotation spread outlier energy).
 *
 * Readings:
 *  - smoothing is per KV head and channel, s_c = 2^n_c; keys are divided by
 *    s_c and queries multiplied by it, so q.k is unchanged;
 *  - the rotation is the unnormalised Sylvester Hadamard matrix over each
 *    power-of-two segment of the head dim (128 -> one H128; 576 -> H512 on the
 *    latent part and H64 on the rope part), computed as the fixed butterfly
 *    network below in fp32;
 *  - the segment of length n = 2^L is post-scaled by 2^-ceil(L/2) for keys and
 *    2^-floor(L/2) for queries, so (H q)(H k)/2^L = q.k exactly in reals.
 * ========================================================================= */

/* Segments of a head dim: greedy powers of two from the largest. */
static int head_segments(int d, int* seg_len)
{
    int n = 0;
    while (d > 0) {
        int p = 1;
        while (p * 2 <= d) p *= 2;
        seg_len[n++] = p;
        d -= p;
    }
    return n;
}

/* In-place Walsh-Hadamard butterflies in fp32: stages h = 1, 2, 4, ..., n/2;
 * each pair (i, i+h) with bit h of i clear becomes (x_i + x_{i+h}, x_i - x_{i+h}). */
void ora_fwht_f32(float* x, int n)
{
    for (int h = 1; h < n; h <<= 1)
        for (int i = 0; i < n; ++i)
            if ((i & h) == 0) {
                float a = x[i], b = x[i + h];
                x[i] = a + b;
                x[i + h] = a - b;
            }
}

static int ilog2i(int n)
{
    int L = 0;
    while ((1 << L) < n) ++L;
    return L;
}

/* is_key = 1: x = H (k / s) * 2^-ceil(L/2); is_key = 0: x = H (q * s) * 2^-floor(L/2). */
void ora_transform(const float* in, const float* smooth, int d, int is_key, int hadamard, float* x)
{
    for (int c = 0; c < d; ++c) x[c] = is_key ? in[c] / smooth[c] : in[c] * smooth[c];
    if (!hadamard) return;
    int seg[8];
    int nseg = head_segments(d, seg), off = 0;
    for (int s = 0; s < nseg; ++s) {
        int L = ilog2i(seg[s]);
        int sh = is_key ? (L + 1) / 2 : L / 2;
        float post = ldexpf(1.0f, -sh);
        ora_fwht_f32(x + off, seg[s]);
        for (int i = 0; i < seg[s]; ++i) x[off + i] = x[off + i] * post;
        off += seg[s];
    }
}

/* =========================================================================
 * 4. Block quantization (NVFP4 / MXFP4)
 * ========================================================================= */

/* fp32 scale sigma that divides the elements for block scale code c.
 * NVFP4: sigma = E4M3(c) * g (fp32 product); MXFP4: sigma = 2^(c-127). */
float ora_block_sigma(int fmt, int code, float g)
{
    if (fmt == ORA_NVFP4) return (float)ora_e4m3_value(code) * g;
    return ldexpf(1.0f, code - 127);
}

/* Elements of one block under scale sigma: e_i = E2M1(fp32(x_i / sigma));
 * a zero sigma (NVFP4 scale code 0) is the all-zero block.  Returns the block
 * squared error sum_i (x_i - e_i sigma)^2, accumulated left to right in fp64. */
double ora_quantize_block(const float* x, int n, float sigma, uint8_t* codes)
{
    double err = 0.0;
    for (int i = 0; i < n; ++i) {
        int e = 0;
        if (sigma != 0.0f) {
            float r = x[i] / sigma;
            e = ora_e2m1_encode((double)r);
        }
        codes[i] = (uint8_t)e;
        double d = (double)x[i] - ora_e2m1_value(e) * (double)sigma;
        err = err + d * d;
    }
    return err;
}

static float block_amax(const float* x, int n)
{
    float a = 0.0f;
    for (int i = 0; i < n; ++i) {
        float v = fabsf(x[i]);
        if (v > a) a = v;
    }
    return a;
}

/* Plain scale rule.  NVFP4: code = E4M3(fp32(amax / fp32(6 g))) -- the block
 * maximum maps to the E2M1 maximum 6; a code of 0 means an all-zero block.
 * MXFP4: the OCP MX shared exponent. */
int ora_plain_scale_code(int fmt, float amax, float g)
{
    if (fmt == ORA_NVFP4) {
        if (amax == 0.0f) return 0;
        float six_g = 6.0f * g;
        float u = amax / six_g;
        return ora_e4m3_encode((double)u);
    }
    return ora_mx_scale_code((double)amax);
}

/* Scale search for key blocks ([ABS] "scale search"; [SNS] picks a better
 * factor for each group).  Reading: start from the plain code c0 and try the
 * window c0+7, c0+6, ..., c0-2 (NVFP4: ten E4M3 codes, clamped to [0, 126];
 * it lets the block maximum land on the E2M1 points 6, 4 or 3) or c0+1, c0
 * (MXFP4, clamped to [0, 254]); keep the code with the least block squared
 * error, ties to the larger code.  An all-zero block keeps code 0. */
int ora_search_scale_code(int fmt, const float* x, int n, float g)
{
    float amax = block_amax(x, n);
    int c0 = ora_plain_scale_code(fmt, amax, g);
    if (amax == 0.0f) return c0;
    int hi, lo, top = (fmt == ORA_NVFP4) ? 126 : 254;
    hi = (fmt == ORA_NVFP4) ? c0 + 7 : c0 + 1;
    lo = (fmt == ORA_NVFP4) ? c0 - 2 : c0;
    if (hi > top) hi = top;
    if (lo < 0) lo = 0;
    uint8_t tmp[64];
    int best = hi;
    double best_err = 0.0;
    for (int c = hi; c >= lo; --c) {
        double err = ora_quantize_block(x, n, ora_block_sigma(fmt, c, g), tmp);
        if (c == hi || err < best_err) {
            best = c;
            best_err = err;
        }
    }
    return best;
}

/* Attention-aware variant of the search (the pages leave its objective open):
 * the same window and tie rule, with each element's squared error weighted by
 * w_i, the calibration queries' mean square of that transformed channel -- for
 * independent channels, the expected square of the logit error q'.(k' - k^')
 * the block adds.  w = NULL is the plain objective (a weight of 1 changes no
 * sum).  Sums run left to right in fp64. */
int ora_search_scale_code_weighted(int fmt, const float* x, int n, float g, const float* w)
{
    if (!w) return ora_search_scale_code(fmt, x, n, g);
    float amax = block_amax(x, n);
    int c0 = ora_plain_scale_code(fmt, amax, g);
    if (amax == 0.0f) return c0;
    int top = (fmt == ORA_NVFP4) ? 126 : 254;
    int hi = (fmt == ORA_NVFP4) ? c0 + 7 : c0 + 1;
    int lo = (fmt == ORA_NVFP4) ? c0 - 2 : c0;
    if (hi > top) hi = top;
    if (lo < 0) lo = 0;
    int best = hi;
    double best_err = 0.0;
    for (int c = hi; c >= lo; --c) {
        float sigma = ora_block_sigma(fmt, c, g);
        double err = 0.0;
        for (int i = 0; i < n; ++i) {
            int e = sigma != 0.0f ? ora_e2m1_encode((double)(x[i] / sigma)) : 0;
            double d = (double)x[i] - ora_e2m1_value(e) * (double)sigma;
            err = err + (double)w[i] * (d * d);
        }
        if (c == hi || err < best_err) {
            best = c;
            best_err = err;
        }
    }
    return best;
}

static int fmt_beta(int fmt) { return fmt == ORA_NVFP4 ? 16 : 32; }

/* =========================================================================
 * 5. Static calibration (smoothing factors and FP32 tensor scales).
 *
 * Readings (the pages say only "static smoothing"):
 *  - s_c = 2^n, n = round-half-up(log2(kmax_c / qmax_c) / 2), i.e. the square
 *    root of the channel's key/query range ratio rounded to a power of two
 *    (SmoothQuant migration strength 1/2).  n is found exactly: with
 *    L = floor(log2(kmax/qmax)), n = floor((L + 1) / 2); clamped to [-20, 20];
 *    0 when either maximum is 0.  qmax is taken over the query heads that
 *    share the KV head.
 *  - NVFP4 tensor scales g_k, g_v per KV head: fp32(amax / 2688) of the
 *    transformed calibration keys / raw calibration values (2688 = 6 * 448,
 *    so the calibration maximum sits at the top of both E2M1 and E4M3);
 *    1 when the amax is 0.
 * ========================================================================= */

static int floor_log2_ratio(float a, float b)  /* a, b > 0 */
{
    int ea, eb;
    double fa = frexp((double)a, &ea), fb = frexp((double)b, &eb);
    return (ea - eb) + (fa >= fb ? 0 : -1);
}

int ora_calibrate(const uint16_t* k_cal, const uint16_t* q_cal, const uint16_t* v_cal,
                  int Tc, int Tq, int H_q, int H_kv, int d_k, int d_v, int flags,
                  float* smooth, float* k_g, float* v_g)
{
    if (H_kv <= 0 || H_q % H_kv != 0 || d_k > 1024) return -1;
    int G = H_q / H_kv;
    int hadamard = !(flags & ORA_FLAG_NO_HADAMARD);
    for (int h = 0; h < H_kv; ++h) {
        for (int c = 0; c < d_k; ++c) {
            float kmax = 0.0f, qmax = 0.0f;
            for (int t = 0; t < Tc; ++t) {
                float v = fabsf(bf16_to_f32(k_cal[((size_t)t * H_kv + h) * d_k + c]));
                if (v > kmax) kmax = v;
            }
            for (int t = 0; t < Tq; ++t)
                for (int j = 0; j < G; ++j) {
                    float v = fabsf(bf16_to_f32(q_cal[((size_t)t * H_q + h * G + j) * d_k + c]));
                    if (v > qmax) qmax = v;
                }
            int n = 0;
            if (kmax > 0.0f && qmax > 0.0f) {
                int L = floor_log2_ratio(kmax, qmax);
                n = (int)floor((L + 1) / 2.0);
                if (n < -20) n = -20;
                if (n > 20) n = 20;
            }
            smooth[(size_t)h * d_k + c] = ldexpf(1.0f, n);
        }
        float in[1024], x[1024], amax = 0.0f;
        for (int t = 0; t < Tc; ++t) {
            for (int c = 0; c < d_k; ++c) in[c] = bf16_to_f32(k_cal[((size_t)t * H_kv + h) * d_k + c]);
            ora_transform(in, smooth + (size_t)h * d_k, d_k, 1, hadamard, x);
            float a = block_amax(x, d_k);
            if (a > amax) amax = a;
        }
        k_g[h] = amax > 0.0f ? amax / 2688.0f : 1.0f;
        float vmax = 0.0f;
        for (int t = 0; t < Tc; ++t)
            for (int c = 0; c < d_v; ++c) {
                float v = fabsf(bf16_to_f32(v_cal[((size_t)t * H_kv + h) * d_v + c]));
                if (v > vmax) vmax = v;
            }
        v_g[h] = vmax > 0.0f ? vmax / 2688.0f : 1.0f;
    }
    return 0;
}

/* Channel weights of the attention-aware search: per KV head h and channel c
 * of the transformed key space, the mean over the calibration queries of the
 * KV group (Tq tokens x G heads) of q'_c^2, q' = the query transform (smoothing
 * and rotation as the decode applies them).  fp64 sums, stored as fp32. */
int ora_key_weights(const uint16_t* q_cal, int Tq, int H_q, int H_kv, int d_k, int flags, const float* smooth,
                    float* w)
{
    if (H_kv <= 0 || H_q % H_kv != 0 || d_k > 1024 || d_k % 64 || Tq <= 0) return -1;
    int G = H_q / H_kv;
    int hadamard = !(flags & ORA_FLAG_NO_HADAMARD);
    for (int h = 0; h < H_kv; ++h) {
        double acc[1024];
        for (int c = 0; c < d_k; ++c) acc[c] = 0.0;
        for (int t = 0; t < Tq; ++t)
            for (int j = 0; j < G; ++j) {
                float in[1024], x[1024];
                for (int c = 0; c < d_k; ++c) in[c] = bf16_to_f32(q_cal[((size_t)t * H_q + h * G + j) * d_k + c]);
                ora_transform(in, smooth + (size_t)h * d_k, d_k, 0, hadamard, x);
                for (int c = 0; c < d_k; ++c) acc[c] += (double)x[c] * (double)x[c];
            }
        for (int c = 0; c < d_k; ++c) w[(size_t)h * d_k + c] = (float)(acc[c] / ((double)Tq * G));
    }
    return 0;
}

/* =========================================================================
 * 6. KV-append quantization into the paged cache.
 *
 * K (token-wise scaling, [ABS]): per token and head, transform, then blocks of
 * beta consecutive channels, each with its searched scale code.
 *
 * V: blocks run along tokens (beta consecutive slots of one page, per
 * channel), because the PV product reduces over tokens; plain scale rule, no
 * transform.  Reading for appends: a V block is re-quantized from the tokens
 * of this call that land in it; the tokens of one block must form one run of
 * consecutive tokens with consecutive slots (a run starts where the slot is
 * the first of its block, at the first token, or where the previous token's
 * slot is not this slot minus one); slots of the block outside the run are
 * zero.  slot_mapping[t] = page * 64 + slot, or -1 to skip the token.
 * ========================================================================= */

static void quantize_key_row(const float* x, int d_k, int fmt, int search, float g, const float* w,
                             int64_t page, int head, int H_kv, int slot,
                             uint8_t* k_pages, uint8_t* k_scales)
{
    int beta = fmt_beta(fmt);
    uint8_t codes[64];
    for (int b = 0; b < d_k / beta; ++b) {
        const float* xb = x + b * beta;
        int sc = search ? ora_search_scale_code_weighted(fmt, xb, beta, g, w ? w + b * beta : NULL)
                        : ora_plain_scale_code(fmt, block_amax(xb, beta), g);
        ora_quantize_block(xb, beta, ora_block_sigma(fmt, sc, g), codes);
        k_scales[k_scale_byte(page, head, H_kv, d_k, beta, slot, b)] = (uint8_t)sc;
        for (int i = 0; i < beta; ++i) {
            int e = b * beta + i;
            put_nibble(k_pages, k_nib_byte(page, head, H_kv, d_k, slot, e), e & 1, codes[i]);
        }
    }
}

/* k_weight: [H_kv][d_k] channel weights of the attention-aware search, or
 * NULL for the plain objective (ora_quantize_kv). */
int ora_quantize_kv_weighted(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping, int T,
                             int H_kv, int d_k, int d_v, int fmt, int flags,
                             const float* smooth, const float* k_g, const float* v_g, const float* k_weight,
                             uint8_t* k_pages, uint8_t* k_scales, uint8_t* v_pages, uint8_t* v_scales,
                             int64_t num_pages)
{
    init_tables();
    if (d_k % 64 || d_v % 128 || d_k > 1024 || (fmt != ORA_NVFP4 && fmt != ORA_MXFP4)) return -1;
    int beta = fmt_beta(fmt);
    int hadamard = !(flags & ORA_FLAG_NO_HADAMARD);
    int search = !(flags & ORA_FLAG_NO_SCALE_SEARCH);
    for (int t = 0; t < T; ++t)
        if (slot_mapping[t] >= num_pages * PAGE_SLOTS) return -2;

    /* K: one row per (token, head). */
#pragma omp parallel for schedule(dynamic, 64)
    for (int t = 0; t < T; ++t) {
        int64_t sm = slot_mapping[t];
        if (sm < 0) continue;
        int64_t page = sm / PAGE_SLOTS;
        int slot = (int)(sm % PAGE_SLOTS);
        float in[1024], x[1024];
        for (int h = 0; h < H_kv; ++h) {
            for (int c = 0; c < d_k; ++c) in[c] = bf16_to_f32(k[((size_t)t * H_kv + h) * d_k + c]);
            ora_transform(in, smooth + (size_t)h * d_k, d_k, 1, hadamard, x);
            float g = fmt == ORA_NVFP4 ? k_g[h] : 1.0f;
            quantize_key_row(x, d_k, fmt, search, g, k_weight ? k_weight + (size_t)h * d_k : NULL, page, h, H_kv,
                             slot, k_pages, k_scales);
        }
    }

    /* V: one block per run leader. */
#pragma omp parallel for schedule(dynamic, 16)
    for (int t = 0; t < T; ++t) {
        int64_t sm = slot_mapping[t];
        if (sm < 0) continue;
        int slot = (int)(sm % PAGE_SLOTS);
        int leader = (slot % beta == 0) || t == 0 || slot_mapping[t - 1] != sm - 1;
        if (!leader) continue;
        int64_t page = sm / PAGE_SLOTS;
        int first = slot - slot % beta;   /* first slot of the block */
        int n = 1;
        while (t + n < T && slot_mapping[t + n] == sm + n && (slot + n) / beta == slot / beta) ++n;
        int blk = first / beta;
        for (int h = 0; h < H_kv; ++h) {
            float g = fmt == ORA_NVFP4 ? v_g[h] : 1.0f;
            for (int c = 0; c < d_v; ++c) {
                float x[32];
                uint8_t codes[32];
                for (int i = 0; i < beta; ++i) {
                    int j = first + i - slot;   /* token offset within the run */
                    x[i] = (j >= 0 && j < n) ? bf16_to_f32(v[((size_t)(t + j) * H_kv + h) * d_v + c]) : 0.0f;
                }
                int sc = ora_plain_scale_code(fmt, block_amax(x, beta), g);
                ora_quantize_block(x, beta, ora_block_sigma(fmt, sc, g), codes);
                v_scales[v_scale_byte(page, h, H_kv, d_v, beta, c, blk)] = (uint8_t)sc;
                for (int i = 0; i < beta; ++i) {
                    int s = first + i;
                    put_nibble(v_pages, v_nib_byte(page, h, H_kv, d_v, c, s), s & 1, codes[i]);
                }
            }
        }
    }
    return 0;
}

int ora_quantize_kv(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping, int T,
                    int H_kv, int d_k, int d_v, int fmt, int flags,
                    const float* smooth, const float* k_g, const float* v_g,
                    uint8_t* k_pages, uint8_t* k_scales, uint8_t* v_pages, uint8_t* v_scales,
                    int64_t num_pages)
{
    return ora_quantize_kv_weighted(k, v, slot_mapping, T, H_kv, d_k, d_v, fmt, flags, smooth, k_g, v_g, NULL,
                                    k_pages, k_scales, v_pages, v_scales, num_pages);
}

/* =========================================================================
 * 7. Dual-Residual Query Quantization ([ABS]; [SNS]: the second FP4 tensor
 *    carries the residual of the first so that their sum approaches q).
 *
 * Readings: the query gets the key transform's counterpart (times s, rotated,
 * post-scaled); NVFP4 uses one dynamic FP32 tensor scale per query head,
 * g_q = fp32(amax / 2688) (1 when amax is 0), shared by q1 and q2 so that both
 * feed one accumulator; q1 = plain-rule FP4 of q'; r = fp32(q' - fp32(e1 *
 * sigma1)); q2 = plain-rule FP4 of r.  MXFP4: no tensor scale.
 * Outputs are logical: one code per byte, [B, H_q, d_k]; scale codes
 * [B, H_q, d_k / beta].
 * ========================================================================= */

static void quantize_query_row(const float* x, int d_k, int fmt, int dual, float gq,
                               uint8_t* c1, uint8_t* s1, uint8_t* c2, uint8_t* s2)
{
    int beta = fmt_beta(fmt);
    float r[1024];
    for (int b = 0; b < d_k / beta; ++b) {
        const float* xb = x + b * beta;
        int sc = ora_plain_scale_code(fmt, block_amax(xb, beta), gq);
        float sigma = ora_block_sigma(fmt, sc, gq);
        ora_quantize_block(xb, beta, sigma, c1 + b * beta);
        s1[b] = (uint8_t)sc;
        for (int i = 0; i < beta; ++i) {
            float deq = (float)ora_e2m1_value(c1[b * beta + i]) * sigma;
            r[b * beta + i] = xb[i] - deq;
        }
    }
    for (int b = 0; b < d_k / beta; ++b) {
        if (!dual) {
            memset(c2 + b * beta, 0, (size_t)beta);
            s2[b] = 0;
            continue;
        }
        const float* rb = r + b * beta;
        int sc = ora_plain_scale_code(fmt, block_amax(rb, beta), gq);
        ora_quantize_block(rb, beta, ora_block_sigma(fmt, sc, gq), c2 + b * beta);
        s2[b] = (uint8_t)sc;
    }
}

static float query_gscale(int fmt, const float* x, int d_k)
{
    if (fmt != ORA_NVFP4) return 1.0f;
    float a = block_amax(x, d_k);
    return a > 0.0f ? a / 2688.0f : 1.0f;
}

int ora_quantize_q(const uint16_t* q, int B, int H_q, int H_kv, int d_k, int fmt, int flags,
                   const float* smooth, uint8_t* q1_codes, uint8_t* q1_scales,
                   uint8_t* q2_codes, uint8_t* q2_scales, float* g_q, float* xq)
{
    init_tables();
    if (d_k % 64 || d_k > 1024 || H_q % H_kv) return -1;
    int G = H_q / H_kv, beta = fmt_beta(fmt);
    int hadamard = !(flags & ORA_FLAG_NO_HADAMARD);
    int dual = !(flags & ORA_FLAG_SINGLE_QUERY);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H_q; ++h) {
            size_t row = (size_t)b * H_q + h;
            float in[1024], x[1024];
            for (int c = 0; c < d_k; ++c) in[c] = bf16_to_f32(q[row * d_k + c]);
            ora_transform(in, smooth + (size_t)(h / G) * d_k, d_k, 0, hadamard, x);
            float gq = query_gscale(fmt, x, d_k);
            quantize_query_row(x, d_k, fmt, dual, gq, q1_codes + row * d_k, q1_scales + row * (d_k / beta),
                               q2_codes + row * d_k, q2_scales + row * (d_k / beta));
            g_q[row] = gq;
            if (xq) memcpy(xq + row * d_k, x, sizeof(float) * (size_t)d_k);
        }
    return 0;
}

/* =========================================================================
 * 8. Paged decode attention.
 *
 * Per (sequence b, query head h):
 *   logits s_t = sm_scale * g_q * g_k * sum_i (deq q1_i + deq q2_i) deq k_ti,
 *   over tokens t < N_b read through block_table[b, t / 64];
 *   online softmax over 128-token tiles aligned to the sequence start; the
 *   tiles are cut into splits of chunk_tiles tiles, each with its own running
 *   max m, sum l and output O; per tile:
 *     m_new = max(m, max_t s_t); p_t = exp(s_t - m_new);
 *     l = l exp(m - m_new) + sum_t p_t              (unquantized p)
 *     P^ = FP4 of p in blocks of beta tokens        (fused P quantization)
 *     O = O exp(m - m_new) + sum_t P^_t deq v_t
 *   Underflow-Aware Probability Scaling ([ABS]; [SNS]: an E4M3 probability
 *   scale that rounds to zero collapses the whole block).  Reading: NVFP4
 *   quantizes y = alpha p with alpha = 2^11, the largest power of two whose
 *   block scale alpha/6 stays inside E4M3 (<= 448), and divides alpha back out
 *   exactly: scale code c = E4M3(amax_y / 6), code 0 = collapsed block,
 *   e_t = E2M1(y_t / E4M3(c)), P^_t = e_t E4M3(c) / alpha.  Vanilla ablation:
 *   alpha = 1.  MXFP4 (E8M0 scale, no underflow at these magnitudes): alpha = 1.
 *   Dynamic variant (NVFP4): the pages place the underflow at long contexts
 *   ([BLOG] What is actually new; [SNS] Analyse approfondie), where a tile far
 *   below the running maximum has only tiny probabilities.
 *   Reading: per tile and head, alpha = 2^E with E the largest integer such
 *   that p_max 2^E <= 2688 (= 6 x 448, so the largest block scale still fits
 *   E4M3), p_max the tile's largest p, E clamped to [11, 64] (64 also for
 *   p_max = 0); P^ is divided by that tile's alpha, so O needs no other change.
 *   A tile that raises the running maximum has p_max = 1 and E = 11, the
 *   static choice.
 *   merge: m* = max m_s, O = sum_s O_s e^(m_s - m*) / sum_s l_s e^(m_s - m*),
 *   rounded to bf16.  An empty sequence gives 0.
 * The probabilities' codes are decided in fp64 here (the GPU decides them in
 * fp32 on MMA logits), so this step is compared within a tolerance.
 * ========================================================================= */

static double deq_key(const uint8_t* k_pages, const uint8_t* k_scales, int fmt, int64_t page, int head,
                      int H_kv, int d_k, int slot, int e)
{
    int beta = fmt_beta(fmt);
    int code = get_nibble(k_pages, k_nib_byte(page, head, H_kv, d_k, slot, e), e & 1);
    int sc = k_scales[k_scale_byte(page, head, H_kv, d_k, beta, slot, e / beta)];
    double s = fmt == ORA_NVFP4 ? ora_e4m3_value(sc) : ora_e8m0_value(sc);
    return ora_e2m1_value(code) * s;
}

static double deq_value(const uint8_t* v_pages, const uint8_t* v_scales, int fmt, int64_t page, int head,
                        int H_kv, int d_v, int chan, int slot)
{
    int beta = fmt_beta(fmt);
    int code = get_nibble(v_pages, v_nib_byte(page, head, H_kv, d_v, chan, slot), slot & 1);
    int sc = v_scales[v_scale_byte(page, head, H_kv, d_v, beta, chan, slot / beta)];
    double s = fmt == ORA_NVFP4 ? ora_e4m3_value(sc) : ora_e8m0_value(sc);
    return ora_e2m1_value(code) * s;
}

/* Dequantized key row (d_k values, without the tensor scale) of one cached token. */
void ora_dequant_key_row(const uint8_t* k_pages, const uint8_t* k_scales, int fmt, int64_t page, int head,
                         int H_kv, int d_k, int slot, double* out)
{
    init_tables();
    for (int e = 0; e < d_k; ++e) out[e] = deq_key(k_pages, k_scales, fmt, page, head, H_kv, d_k, slot, e);
}

/* Dequantized value row (d_v values, without the tensor scale) of one cached token. */
void ora_dequant_value_row(const uint8_t* v_pages, const uint8_t* v_scales, int fmt, int64_t page, int head,
                           int H_kv, int d_v, int slot, double* out)
{
    init_tables();
    for (int c = 0; c < d_v; ++c) out[c] = deq_value(v_pages, v_scales, fmt, page, head, H_kv, d_v, c, slot);
}

/* Exponent E of the per-tile alpha = 2^E of the dynamic variant: the largest
 * integer with p_max 2^E <= 2688, clamped to [11, 64]; every product here is
 * exact in fp64 (a power-of-two scaling). */
int ora_dynamic_alpha_exp(double p_max)
{
    if (!(p_max > 0.0)) return 64;
    int E = 11;
    while (E < 64 && ldexp(p_max, E + 1) <= 2688.0) ++E;
    while (E > 11 && ldexp(p_max, E) > 2688.0) --E;
    return E;
}

/* FP4 quantization of one block of probabilities y (already times alpha),
 * decided in fp64; returns the dequantized values (still times alpha). */
static void quantize_probs(int fmt, const double* y, int n, double* yq)
{
    double amax = 0.0;
    for (int i = 0; i < n; ++i)
        if (y[i] > amax) amax = y[i];
    double sigma;
    if (fmt == ORA_NVFP4) {
        int c = amax > 0.0 ? ora_e4m3_encode(amax / 6.0) : 0;
        sigma = ora_e4m3_value(c);
    } else {
        sigma = ora_e8m0_value(ora_mx_scale_code(amax));
    }
    for (int i = 0; i < n; ++i) {
        int e = sigma > 0.0 ? ora_e2m1_encode(y[i] / sigma) : 0;
        yq[i] = ora_e2m1_value(e) * sigma;
    }
}

int ora_decode(const uint16_t* q, const uint8_t* k_pages, const uint8_t* k_scales,
               const uint8_t* v_pages, const uint8_t* v_scales,
               const int32_t* block_table, const int32_t* seq_lens,
               int B, int H_q, int H_kv, int d_k, int d_v, int max_pages, int64_t num_pages,
               int fmt, int flags, const float* smooth, const float* k_g, const float* v_g,
               double sm_scale, int chunk_tiles, uint16_t* out_bf16, double* out_f64)
{
    init_tables();
    if (d_k % 64 || d_v % 128 || d_k > 1024 || d_v > 1024 || H_q % H_kv || chunk_tiles <= 0) return -1;
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 0 || seq_lens[b] > max_pages * PAGE_SLOTS) return -2;
        for (int p = 0; p < (seq_lens[b] + PAGE_SLOTS - 1) / PAGE_SLOTS; ++p)
            if (block_table[(size_t)b * max_pages + p] < 0 || block_table[(size_t)b * max_pages + p] >= num_pages)
                return -3;
    }
    int G = H_q / H_kv, beta = fmt_beta(fmt);
    int hadamard = !(flags & ORA_FLAG_NO_HADAMARD);
    int dual = !(flags & ORA_FLAG_SINGLE_QUERY);
    double alpha = (fmt == ORA_NVFP4 && !(flags & ORA_FLAG_NO_UNDERFLOW)) ? 2048.0 : 1.0;
    if ((flags & ORA_FLAG_DYNAMIC_ALPHA) && (flags & ORA_FLAG_NO_UNDERFLOW)) return -1;
    int dynamic = fmt == ORA_NVFP4 && (flags & ORA_FLAG_DYNAMIC_ALPHA);

    /* One (sequence, KV head) at a time; the G query heads of the group each
     * run the steps above.  A tile's keys and values are dequantized once
     * into fp64 and shared by the heads (no change to any head's arithmetic). */
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < H_kv; ++hk) {
            int N = seq_lens[b];
            double* kt = malloc(sizeof(double) * TILE_TOKENS * (size_t)d_k);
            double* vt = malloc(sizeof(double) * TILE_TOKENS * (size_t)d_v);
            double* dq = malloc(sizeof(double) * (size_t)G * d_k);
            double* lsc = malloc(sizeof(double) * (size_t)G);
            double* m = malloc(sizeof(double) * (size_t)G);
            double* l = malloc(sizeof(double) * (size_t)G);
            double* M_all = malloc(sizeof(double) * (size_t)G);
            double* L_all = malloc(sizeof(double) * (size_t)G);
            double* o_split = calloc((size_t)G * d_v, sizeof(double));
            double* o_merged = calloc((size_t)G * d_v, sizeof(double));
            int valid[TILE_TOKENS];
            double s[TILE_TOKENS], y[TILE_TOKENS], yq[TILE_TOKENS];
            double vg = fmt == ORA_NVFP4 ? (double)v_g[hk] : 1.0;

            /* queries: transform + dual-residual FP4, dequantized in fp64 */
            for (int j = 0; j < G; ++j) {
                size_t row = (size_t)b * H_q + (size_t)hk * G + j;
                float in[1024], x[1024];
                uint8_t c1[1024], c2[1024], s1[64], s2[64];
                for (int c = 0; c < d_k; ++c) in[c] = bf16_to_f32(q[row * d_k + c]);
                ora_transform(in, smooth + (size_t)hk * d_k, d_k, 0, hadamard, x);
                float gq = query_gscale(fmt, x, d_k);
                quantize_query_row(x, d_k, fmt, dual, gq, c1, s1, c2, s2);
                for (int i = 0; i < d_k; ++i) {
                    double sc1 = fmt == ORA_NVFP4 ? ora_e4m3_value(s1[i / beta]) : ora_e8m0_value(s1[i / beta]);
                    double sc2 = fmt == ORA_NVFP4 ? ora_e4m3_value(s2[i / beta]) : ora_e8m0_value(s2[i / beta]);
                    dq[(size_t)j * d_k + i] = ora_e2m1_value(c1[i]) * sc1 + ora_e2m1_value(c2[i]) * sc2;
                }
                lsc[j] = sm_scale * (fmt == ORA_NVFP4 ? (double)gq * (double)k_g[hk] : 1.0);
                M_all[j] = -INFINITY;
                L_all[j] = 0.0;
            }

            int ntiles = (N + TILE_TOKENS - 1) / TILE_TOKENS;
            for (int sp0 = 0; sp0 < ntiles; sp0 += chunk_tiles) {
                int sp1 = sp0 + chunk_tiles < ntiles ? sp0 + chunk_tiles : ntiles;
                for (int j = 0; j < G; ++j) {
                    m[j] = -INFINITY;
                    l[j] = 0.0;
                }
                memset(o_split, 0, sizeof(double) * (size_t)G * d_v);
                for (int tile = sp0; tile < sp1; ++tile) {
                    int t0 = tile * TILE_TOKENS;
                    for (int jt = 0; jt < TILE_TOKENS; ++jt) {
                        int t = t0 + jt;
                        valid[jt] = t < N;
                        if (!valid[jt]) continue;
                        int64_t page = block_table[(size_t)b * max_pages + t / PAGE_SLOTS];
                        int slot = t % PAGE_SLOTS;
                        for (int i = 0; i < d_k; ++i)
                            kt[(size_t)jt * d_k + i] = deq_key(k_pages, k_scales, fmt, page, hk, H_kv, d_k, slot, i);
                        for (int c = 0; c < d_v; ++c)
                            vt[(size_t)jt * d_v + c] =
                                deq_value(v_pages, v_scales, fmt, page, hk, H_kv, d_v, c, slot) * vg;
                    }
                    for (int j = 0; j < G; ++j) {
                        const double* dqj = dq + (size_t)j * d_k;
                        double* oj = o_split + (size_t)j * d_v;
                        double m_tile = -INFINITY;
                        for (int jt = 0; jt < TILE_TOKENS; ++jt) {
                            s[jt] = -INFINITY;
                            if (!valid[jt]) continue;
                            double acc = 0.0;
                            for (int i = 0; i < d_k; ++i) acc += dqj[i] * kt[(size_t)jt * d_k + i];
                            s[jt] = acc * lsc[j];
                            if (s[jt] > m_tile) m_tile = s[jt];
                        }
                        double m_new = m[j] > m_tile ? m[j] : m_tile;
                        double corr = exp(m[j] - m_new);   /* 0 on a split's first tile */
                        double psum = 0.0, p_max = 0.0;
                        for (int jt = 0; jt < TILE_TOKENS; ++jt) {
                            y[jt] = valid[jt] ? exp(s[jt] - m_new) : 0.0;
                            if (y[jt] > p_max) p_max = y[jt];
                        }
                        double alpha_t = dynamic ? ldexp(1.0, ora_dynamic_alpha_exp(p_max)) : alpha;
                        for (int jt = 0; jt < TILE_TOKENS; ++jt) {
                            psum += y[jt];
                            y[jt] *= alpha_t;
                        }
                        if (flags & ORA_FLAG_EXACT_P) memcpy(yq, y, sizeof(y));
                        else
                            for (int j0 = 0; j0 < TILE_TOKENS; j0 += beta) quantize_probs(fmt, y + j0, beta, yq + j0);
                        l[j] = l[j] * corr + psum;
                        for (int c = 0; c < d_v; ++c) oj[c] *= corr;
                        for (int jt = 0; jt < TILE_TOKENS; ++jt) {
                            if (!valid[jt] || yq[jt] == 0.0) continue;
                            double w = yq[jt] / alpha_t;
                            for (int c = 0; c < d_v; ++c) oj[c] += w * vt[(size_t)jt * d_v + c];
                        }
                        m[j] = m_new;
                    }
                }
                /* merge this split into the running merge state */
                for (int j = 0; j < G; ++j) {
                    double M_new = M_all[j] > m[j] ? M_all[j] : m[j];
                    double a_old = exp(M_all[j] - M_new), a_new = exp(m[j] - M_new);
                    L_all[j] = L_all[j] * a_old + l[j] * a_new;
                    for (int c = 0; c < d_v; ++c)
                        o_merged[(size_t)j * d_v + c] = o_merged[(size_t)j * d_v + c] * a_old +
                                                        o_split[(size_t)j * d_v + c] * a_new;
                    M_all[j] = M_new;
                }
            }
            for (int j = 0; j < G; ++j) {
                size_t row = (size_t)b * H_q + (size_t)hk * G + j;
                for (int c = 0; c < d_v; ++c) {
                    double o = L_all[j] > 0.0 ? o_merged[(size_t)j * d_v + c] / L_all[j] : 0.0;
                    if (out_f64) out_f64[row * d_v + c] = o;
                    if (out_bf16) out_bf16[row * d_v + c] = ora_f64_to_bf16(o);
                }
            }
            free(kt); free(vt); free(dq); free(lsc); free(m); free(l);
            free(M_all); free(L_all); free(o_split); free(o_merged);
        }
    return 0;
}

/* =========================================================================
 * 9. Reference arm: unquantized attention on the bf16 inputs in fp64
 *    (the "BF16 KV" accuracy reference of [ABS]).  K and V are token-major
 *    [T, H_kv, d] with sequence b owning tokens [cu_seqlens[b], cu_seqlens[b+1]).
 * ========================================================================= */
int ora_attention_ref(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int64_t* cu_seqlens,
                      int B, int H_q, int H_kv, int d_k, int d_v, double sm_scale, double* out_f64)
{
    if (H_q % H_kv) return -1;
    int G = H_q / H_kv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H_q; ++h) {
            int hk = h / G;
            int64_t t0 = cu_seqlens[b], N = cu_seqlens[b + 1] - cu_seqlens[b];
            size_t row = (size_t)b * H_q + h;
            double* s = malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
            double mx = -INFINITY;
            for (int64_t t = 0; t < N; ++t) {
                double acc = 0.0;
                for (int c = 0; c < d_k; ++c)
                    acc += (double)bf16_to_f32(q[row * d_k + c]) *
                           (double)bf16_to_f32(k[((size_t)(t0 + t) * H_kv + hk) * d_k + c]);
                s[t] = acc * sm_scale;
                if (s[t] > mx) mx = s[t];
            }
            double l = 0.0;
            for (int64_t t = 0; t < N; ++t) {
                s[t] = exp(s[t] - mx);
                l += s[t];
            }
            for (int c = 0; c < d_v; ++c) {
                double acc = 0.0;
                for (int64_t t = 0; t < N; ++t)
                    acc += s[t] * (double)bf16_to_f32(v[((size_t)(t0 + t) * H_kv + hk) * d_v + c]);
                out_f64[row * d_v + c] = N > 0 ? acc / l : 0.0;
            }
            free(s);
        }
    return 0;
}

/* Thread count the OpenMP regions above use (for the CPU-baseline record). */
int ora_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
