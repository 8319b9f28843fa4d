/*
 * bitlinear_oracle.c -- plain, slow, obviously-correct CPU statement of the
 * BitNet b1.58 BitLinear forward computation.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library; the two meet only through the seeded synthetic inputs.
 *
 * Source of every step (cited as [MF]):
 *   "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
 *    Absmean Scaling, and Multiplication-Free LLM Architectures" (llms.blog),
 *   section 2 "Mathematical Formulation of the BitLinear b1.58 Layer" with its
 *   three parts "Weight Quantization: Absmean Scaling", "Activation
 *   Quantization: Absmax Scaling" and "The Linear Transformation and
 *   Rescaling"; section 6 "Implementation Considerations and Inference
 *   Engines", part "Vectorized Ternary GEMV with SIMD" (sign / zero masks,
 *   masked addition, scale-factor fusion).
 *
 * Precision: reductions (the absmean sum, the RMS sum of squares) and the
 * final rescale are carried in double.  The quantities that feed an integer
 * code (z = W / (gamma + eps), n = x * r, v = n * 127 / (beta + eps)) are
 * formed in IEEE binary32, one correctly rounded operation at a time, because
 * that is the precision in which the GPU kernels form them; the rounding
 * floor(z + 0.5) itself is then evaluated exactly.  This file is compiled
 * with -ffp-contract=off and without fast-math so no operation is fused.
 *
 * Readings taken where the page is silent or inconsistent:
 *   - Q_b - 1 = 127 is both the activation multiplier and the clip bound; the
 *     code range is the symmetric [-127, 127].
 *   - The activation absmax beta is taken per token (one row of X).
 *   - RMSNorm is x * r * g with r = 1 / sqrt(mean(x^2) + norm_eps) (the
 *     reciprocal formed once per token) and g = 1 unless a gain vector is
 *     given; the page names RMSNorm but prints no formula.
 *   - The rescale is the literal beta*gamma/(Q_b-1), without the epsilons used
 *     inside the two quantisers.
 *   - RoundClip rounds with floor(z + 0.5), i.e. halves go toward +infinity,
 *     evaluated exactly on the binary32 value z.
 *
 * Packed weight layout (this library's own format; the page only says
 * "packed 2-bit"): a d_out x d_in ternary matrix is cut into tiles of 16 rows
 * by 256 columns, stored tile-row-major; inside a tile the 16 rows follow one
 * another, each as 16 little-endian 32-bit words; word kw of a row holds
 * columns 16*kw .. 16*kw+15 and the 2-bit code c = W~ + 1 of column
 * 16*kw + 4*s + j sits at bits 8*j + 2*s.  Code 3 is never produced and is
 * rejected on unpack.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_QB_MINUS_1 127

/* ---------------------------------------------------------------- bf16 --- */

/* bf16 -> binary32 is exact: the bf16 pattern is the top half of the float. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even (finite inputs). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------ weight quantisation ([MF] §2) */

/* Sum over all entries of |W_ij|, in double, in index order. */
double oracle_abs_sum(const float *W, int64_t n_out, int64_t n_in)
{
    double s = 0.0;
    for (int64_t i = 0; i < n_out * n_in; ++i)
        s += fabs((double)W[i]);
    return s;
}

/* gamma = (1 / (d_out d_in)) * sum |W_ij|   ([MF] §2, absmean scale). */
float oracle_absmean_gamma(const float *W, int64_t n_out, int64_t n_in)
{
    double s = oracle_abs_sum(W, n_out, n_in);
    return (float)(s / ((double)n_out * (double)n_in));
}

/* RoundClip(z, a, b) = max(a, min(b, floor(z + 0.5)))   ([MF] §2).
 * z arrives in binary32; floor(z + 0.5) is then taken exactly: the sum is
 * formed in double, which holds z + 0.5 without rounding whenever it lies
 * near an integer (|z| >= 0.5 there, so z has no bits below 2^-24 of its
 * leading bit).  A binary32 sum would round 0.5 - 2^-25 + 0.5 up to 1. */
static float round_clip_f32(float z, float a, float b)
{
    double u = (double)z + 0.5;
    float r = (float)floor(u);
    if (r > b) r = b;
    if (r < a) r = a;
    return r;
}

/* W~_ij = RoundClip(W_ij / (gamma + eps), -1, 1)   ([MF] §2). */
void oracle_ternarize(const float *W, int64_t count, float gamma, float eps,
                      int8_t *wq)
{
    float den = gamma + eps;   /* binary32 addition */
    for (int64_t i = 0; i < count; ++i) {
        float z = W[i] / den;  /* binary32 division */
        wq[i] = (int8_t)round_clip_f32(z, -1.0f, 1.0f);
    }
}

/* ------------------------------------------------------- packed layout --- */

/* Index of the word holding weight (o, k) and the bit offset of its code. */
static void packed_position(int64_t n_in, int64_t o, int64_t k,
                            int64_t *word, int *shift)
{
    int64_t tiles_per_row = n_in / 256;
    int64_t rb = o / 16, r = o % 16;
    int64_t kb = k / 256, kw = (k % 256) / 16;
    int s = (int)((k % 16) / 4), j = (int)(k % 4);
    *word = ((rb * tiles_per_row + kb) * 16 + r) * 16 + kw;
    *shift = 8 * j + 2 * s;
}

/* Returns 0, or -1 if a shape is not a whole number of tiles or a code is
 * outside {-1, 0, 1}. */
int oracle_pack(const int8_t *wq, int64_t n_out, int64_t n_in, uint32_t *packed)
{
    if (n_out % 16 != 0 || n_in % 256 != 0) return -1;
    memset(packed, 0, (size_t)(n_out * n_in / 16) * sizeof(uint32_t));
    for (int64_t o = 0; o < n_out; ++o) {
        for (int64_t k = 0; k < n_in; ++k) {
            int v = wq[o * n_in + k];
            if (v < -1 || v > 1) return -1;
            int64_t word;
            int shift;
            packed_position(n_in, o, k, &word, &shift);
            packed[word] |= ((uint32_t)(v + 1)) << shift;
        }
    }
    return 0;
}

/* Inverse of oracle_pack.  Returns -1 on the unused code 3. */
int oracle_unpack(const uint32_t *packed, int64_t n_out, int64_t n_in, int8_t *wq)
{
    if (n_out % 16 != 0 || n_in % 256 != 0) return -1;
    for (int64_t o = 0; o < n_out; ++o) {
        for (int64_t k = 0; k < n_in; ++k) {
            int64_t word;
            int shift;
            packed_position(n_in, o, k, &word, &shift);
            uint32_t c = (packed[word] >> shift) & 3u;
            if (c == 3u) return -1;
            wq[o * n_in + k] = (int8_t)((int)c - 1);
        }
    }
    return 0;
}

/* One row of codes read back out of the packed buffer (for sampled checks on
 * matrices too large to unpack whole).  Returns -1 on code 3. */
int oracle_unpack_row(const uint32_t *packed, int64_t n_out, int64_t n_in,
                      int64_t o, int8_t *row)
{
    if (n_out % 16 != 0 || n_in % 256 != 0 || o < 0 || o >= n_out) return -1;
    for (int64_t k = 0; k < n_in; ++k) {
        int64_t word;
        int shift;
        packed_position(n_in, o, k, &word, &shift);
        uint32_t c = (packed[word] >> shift) & 3u;
        if (c == 3u) return -1;
        row[k] = (int8_t)((int)c - 1);
    }
    return 0;
}

/* ------------------------------------ base-3 packed layout ([MF] §4) --- */

/* [MF] §4, "Memory Bandwidth and Latency Bounds": five ternary values fit in
 * one byte because 3^5 = 243 < 256.  This library's base-3 format (its own;
 * the page fixes only the five-per-byte count):
 *   - each row is padded with W~ = 0 to a whole number of 160 columns;
 *   - the matrix is cut into tiles of 16 rows x 160 columns (512 bytes),
 *     stored tile-row-major like the 2-bit format, each row of a tile as 32
 *     consecutive bytes;
 *   - byte B of a tile row belongs to the 20-column group g = B / 4 and, with
 *     j = B % 4, holds the codes c_i = W~ + 1 of the columns 20*g + 4*i + j,
 *     i = 0..4, as the base-3 number c_0 + 3 c_1 + 9 c_2 + 27 c_3 + 81 c_4.
 * So a byte never exceeds 242, and a full row costs 8/5 = 1.6 bits per
 * weight. */
int64_t oracle_base3_cols(int64_t n_in)
{
    return (n_in + 159) / 160 * 160;
}

/* Byte holding weight (o, k) (k < padded width) and the power of 3 of its
 * digit. */
static void base3_position(int64_t n_in, int64_t o, int64_t k, int64_t *byte, int *power)
{
    int64_t tiles_per_row = oracle_base3_cols(n_in) / 160;
    int64_t rb = o / 16, r = o % 16;
    int64_t kb = k / 160, col = k % 160;
    int64_t g = col / 20, in_group = col % 20;
    int i = (int)(in_group / 4), j = (int)(in_group % 4);
    *byte = ((rb * tiles_per_row + kb) * 16 + r) * 32 + g * 4 + j;
    *power = i;
}

static const int kPow3[5] = {1, 3, 9, 27, 81};

/* Returns 0, or -1 if d_out is not a multiple of 16, d_in < 1 or a code is
 * outside {-1, 0, 1}.  packed holds d_out * padded width / 5 bytes. */
int oracle_pack_base3(const int8_t *wq, int64_t n_out, int64_t n_in, uint8_t *packed)
{
    if (n_out % 16 != 0 || n_in < 1) return -1;
    const int64_t kp = oracle_base3_cols(n_in);
    memset(packed, 0, (size_t)(n_out * kp / 5));
    for (int64_t o = 0; o < n_out; ++o) {
        for (int64_t k = 0; k < kp; ++k) {
            int v = k < n_in ? wq[o * n_in + k] : 0;
            if (v < -1 || v > 1) return -1;
            int64_t byte;
            int power;
            base3_position(n_in, o, k, &byte, &power);
            packed[byte] = (uint8_t)(packed[byte] + (v + 1) * kPow3[power]);
        }
    }
    return 0;
}

/* Inverse of oracle_pack_base3: digit i of byte b is (b / 3^i) mod 3.
 * Returns -1 on a byte above 242 or a padding column that is not W~ = 0. */
int oracle_unpack_base3(const uint8_t *packed, int64_t n_out, int64_t n_in, int8_t *wq)
{
    if (n_out % 16 != 0 || n_in < 1) return -1;
    const int64_t kp = oracle_base3_cols(n_in);
    for (int64_t b = 0; b < n_out * kp / 5; ++b)
        if (packed[b] > 242) return -1;
    for (int64_t o = 0; o < n_out; ++o) {
        for (int64_t k = 0; k < kp; ++k) {
            int64_t byte;
            int power;
            base3_position(n_in, o, k, &byte, &power);
            int c = (packed[byte] / kPow3[power]) % 3;
            if (k < n_in)
                wq[o * n_in + k] = (int8_t)(c - 1);
            else if (c != 1)
                return -1;
        }
    }
    return 0;
}

/* ----------------------------------------- binary weights (W1A4, [EoMM]) */

/* W1: the binary alphabet {-1, +1} of [MF] section 1 (BitNet b1), used by the
 * W1A4 regime that "The End of Matrix Multiplications: Welcome to Addition"
 * names (1-bit weights, 4-bit activations).  The pages give no binarisation
 * rule; the reading taken: W~ = +1 where W >= 0 and -1 elsewhere (so +0 and
 * -0 both map to +1), scaled by the same absmean gamma as the ternary layer,
 * which is the least-squares scale of a sign code: d/da sum (W - a sign W)^2
 * = 0 at a = mean |W|. */
void oracle_binarize(const float *W, int64_t count, int8_t *wq)
{
    for (int64_t i = 0; i < count; ++i) wq[i] = (int8_t)(W[i] >= 0.0f ? 1 : -1);
}

/* This library's 1-bit format: rows padded with W~ = -1 to a multiple of 512
 * columns; tiles of 16 rows x 512 columns (1 KiB), tile-row-major; each tile
 * row is 16 little-endian 32-bit words; word kw covers columns 32 kw .. 32 kw
 * + 31, and the bit c = (W~ + 1) / 2 of column 32 kw + 4 s + j sits at bit
 * 8 j + s.  So (word >> s) & 0x01010101 is the four bits of four consecutive
 * columns. */
int64_t oracle_w1_cols(int64_t n_in)
{
    return (n_in + 511) / 512 * 512;
}

static void w1_position(int64_t n_in, int64_t o, int64_t k, int64_t *word, int *bit)
{
    int64_t tiles_per_row = oracle_w1_cols(n_in) / 512;
    int64_t rb = o / 16, r = o % 16;
    int64_t kb = k / 512, kw = (k % 512) / 32;
    int s = (int)((k % 32) / 4), j = (int)(k % 4);
    *word = ((rb * tiles_per_row + kb) * 16 + r) * 16 + kw;
    *bit = 8 * j + s;
}

/* Returns 0, or -1 if d_out is not a multiple of 16, d_in < 1 or a code is
 * not -1 or +1.  packed holds d_out * padded width / 32 words. */
int oracle_pack_w1(const int8_t *wq, int64_t n_out, int64_t n_in, uint32_t *packed)
{
    if (n_out % 16 != 0 || n_in < 1) return -1;
    const int64_t kp = oracle_w1_cols(n_in);
    memset(packed, 0, (size_t)(n_out * kp / 32) * sizeof(uint32_t));
    for (int64_t o = 0; o < n_out; ++o) {
        for (int64_t k = 0; k < n_in; ++k) {
            int v = wq[o * n_in + k];
            if (v != -1 && v != 1) return -1;
            int64_t word;
            int bit;
            w1_position(n_in, o, k, &word, &bit);
            if (v == 1) packed[word] |= 1u << bit;
        }
    }
    return 0;
}

/* Inverse of oracle_pack_w1.  Returns -1 if a padding bit is set. */
int oracle_unpack_w1(const uint32_t *packed, int64_t n_out, int64_t n_in, int8_t *wq)
{
    if (n_out % 16 != 0 || n_in < 1) return -1;
    const int64_t kp = oracle_w1_cols(n_in);
    for (int64_t o = 0; o < n_out; ++o) {
        for (int64_t k = 0; k < kp; ++k) {
            int64_t word;
            int bit;
            w1_position(n_in, o, k, &word, &bit);
            int c = (int)((packed[word] >> bit) & 1u);
            if (k < n_in)
                wq[o * n_in + k] = (int8_t)(2 * c - 1);
            else if (c)
                return -1;
        }
    }
    return 0;
}

/* Threads the OpenMP build runs its parallel loops on (1 in the plain build). */
#ifdef _OPENMP
#include <omp.h>
int oracle_threads(void) { return omp_get_max_threads(); }
#else
int oracle_threads(void) { return 1; }
#endif

/* ---------------------------------------- activation quantisation ([MF] §2) */

/* Reciprocal RMS of one token: 1 / sqrt(mean(x^2) + norm_eps), carried in
 * double (sum, mean, square root and reciprocal each correctly rounded) and
 * rounded once to binary32. */
float oracle_inv_rms(const uint16_t *x, int64_t K, float norm_eps)
{
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double v = (double)oracle_bf16_to_f32(x[k]);
        ss += v * v;
    }
    return (float)(1.0 / sqrt(ss / (double)K + (double)norm_eps));
}

/* The normalised value of one element: x * r (times g), or x unchanged. */
static float normalised(const uint16_t *x, int64_t k, int rmsnorm, float r, const float *gain)
{
    float n = oracle_bf16_to_f32(x[k]);
    if (rmsnorm) {
        n = n * r;
        if (gain) n = n * gain[k];
    }
    return n;
}

/*
 * Absmax int8 quantisation with optional RMSNorm in front.
 *   n_k   = x_k * r (binary32 multiplication) with r the token's reciprocal
 *           RMS, times g_k if a gain is given (binary32 multiplication);
 *           n_k = x_k when rmsnorm == 0
 *   beta  = max |n| over the token (per_tensor == 0), or over every element
 *           of every token (per_tensor != 0: [MF] section 2 prints the max
 *           over all i, j and allows either scope)
 *   q_k   = RoundClip(n_k * 127 / (beta + eps), -127, 127) with the scale
 *           127 / (beta + eps) formed first (binary32 add, then divide) and
 *           applied with one binary32 multiplication
 *   S     = sum_k q_k per token (the correction term of the offset-code
 *           product)
 * inv_rms_in, when not NULL, supplies the per-token reciprocal RMS instead of
 * computing it (used to compare integer codes against a GPU that computed
 * its own).  beta[t] receives the beta token t was quantised with.
 */
void oracle_quant_act_bits(const uint16_t *X, int64_t T, int64_t K, const float *gain,
                           int rmsnorm, int per_tensor, int act_bits, float eps,
                           float norm_eps, const float *inv_rms_in, int8_t *xq, float *beta,
                           int32_t *rowsum, float *inv_rms_out)
{
    /* Q_b = 2^(k-1) levels for k-bit activations ([MF] section 2); the
     * multiplier and the clip bound are Q_b - 1. */
    const int qmax = (1 << (act_bits - 1)) - 1;
    /* Statistics of every token first. */
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *x = X + t * K;
        float r = 1.0f;
        if (rmsnorm)
            r = inv_rms_in ? inv_rms_in[t] : oracle_inv_rms(x, K, norm_eps);
        if (inv_rms_out) inv_rms_out[t] = r;
        float b = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(normalised(x, k, rmsnorm, r, gain));
            if (a > b) b = a;
        }
        beta[t] = b;
    }
    if (per_tensor) {
        float m = 0.0f;
        for (int64_t t = 0; t < T; ++t)
            if (beta[t] > m) m = beta[t];
        for (int64_t t = 0; t < T; ++t) beta[t] = m;
    }
    /* Then the codes. */
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *x = X + t * K;
        float r = 1.0f;
        if (rmsnorm)
            r = inv_rms_in ? inv_rms_in[t] : oracle_inv_rms(x, K, norm_eps);
        float scale = (float)qmax / (beta[t] + eps);
        int32_t S = 0;
        for (int64_t k = 0; k < K; ++k) {
            float v = normalised(x, k, rmsnorm, r, gain) * scale;
            int q = (int)round_clip_f32(v, -(float)qmax, (float)qmax);
            xq[t * K + k] = (int8_t)q;
            S += q;
        }
        rowsum[t] = S;
    }
}

/* The int8 quantiser of [MF] section 2: 8-bit activations, Q_b - 1 = 127. */
void oracle_quant_act(const uint16_t *X, int64_t T, int64_t K, const float *gain,
                      int rmsnorm, int per_tensor, float eps, float norm_eps,
                      const float *inv_rms_in, int8_t *xq, float *beta, int32_t *rowsum,
                      float *inv_rms_out)
{
    oracle_quant_act_bits(X, T, K, gain, rmsnorm, per_tensor, 8, eps, norm_eps, inv_rms_in, xq,
                          beta, rowsum, inv_rms_out);
}

/* ---------------------------------- product and rescale ([MF] §2 and §6) */

/* acc[t][o] = sum_k W~[o][k] * X~[t][k], exact in int32. */
void oracle_int_matmul(const int8_t *wq, const int8_t *xq, int64_t T, int64_t N,
                       int64_t K, int32_t *acc)
{
    /* The outputs are independent: the OpenMP build of this file (used only
     * to time the oracle on every host core) splits them over threads; the
     * plain build ignores the pragma.  Each output is the same sum either
     * way. */
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t o = 0; o < N; ++o) {
            int32_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int32_t)wq[o * K + k] * (int32_t)xq[t * K + k];
            acc[t * N + o] = s;
        }
}

/* The same dot product written the multiplier-free way of [MF] §6: unpack a
 * sign mask and a zero mask per weight and add (x XOR sign) - sign where the
 * weight is non-zero.  sign is all ones (-1) for a -1 weight and 0 otherwise;
 * on two's-complement int8 (x ^ -1) - (-1) = ~x + 1 = -x. */
int32_t oracle_dot_masked_add(const int8_t *wrow, const int8_t *xrow, int64_t K)
{
    int32_t acc = 0;
    for (int64_t k = 0; k < K; ++k) {
        int32_t sign = (wrow[k] < 0) ? -1 : 0;
        int nonzero = (wrow[k] != 0);
        if (nonzero)
            acc += ((int32_t)xrow[k] ^ sign) - sign;
    }
    return acc;
}

/* Y = (X~ W~^T) * beta * gamma / (Q_b - 1), in double ([MF] §2). */
void oracle_rescale_bits(const int32_t *acc, int64_t T, int64_t N, float gamma,
                         const float *beta, int act_bits, double *y)
{
    const double qmax = (double)((1 << (act_bits - 1)) - 1);
    for (int64_t t = 0; t < T; ++t) {
        double scale = (double)beta[t] * (double)gamma / qmax;
        for (int64_t o = 0; o < N; ++o)
            y[t * N + o] = (double)acc[t * N + o] * scale;
    }
}

void oracle_rescale(const int32_t *acc, int64_t T, int64_t N, float gamma,
                    const float *beta, double *y)
{
    oracle_rescale_bits(acc, T, N, gamma, beta, 8, y);
}

/*
 * The dense bf16 layer that BitLinear replaces, Y = X W^T ([MF] §2, "The
 * Linear Transformation and Rescaling", without the quantisers): the context
 * the measurements compare against.  Each product of two bf16 values is
 * exact in double (8 + 8 significant bits); the K products of one output are
 * summed in double in index order.
 */
double oracle_dense_bf16_dot(const uint16_t *w, const uint16_t *x, int64_t K)
{
    double s = 0.0;
    for (int64_t k = 0; k < K; ++k)
        s += (double)oracle_bf16_to_f32(w[k]) * (double)oracle_bf16_to_f32(x[k]);
    return s;
}

void oracle_dense_bf16(const uint16_t *W, const uint16_t *X, int64_t T, int64_t N, int64_t K,
                       double *y)
{
    for (int64_t t = 0; t < T; ++t)
        for (int64_t o = 0; o < N; ++o)
            y[t * N + o] = oracle_dense_bf16_dot(W + o * K, X + t * K, K);
}

/*
 * Backward pass with the straight-through estimator ([MF] section 3,
 * "Training Dynamics and the Straight-Through Estimator"): the rounding of
 * both quantisers is bypassed, so the layer acts as Y = X^ (gamma W~)^T with
 * the dequantised activations X^ = X~ * beta / 127, gamma and beta held
 * constant.  Given dY [T][N] (bf16):
 *   dX[t][k] = gamma * sum_o dY[t][o] W~[o][k]        (gradient at X^)
 *   dW[o][k] = gamma * sum_t dY[t][o] X^[t][k]        (gradient at W~, passed
 *                                                      to the latent weights)
 * X^ is formed as the GEMM operand is: bf16 of the binary32 product
 * X~ * (beta / 127) (binary32 divide, binary32 multiply, round to nearest
 * even).  Sums in double; each product of a bf16 value and a small integer or
 * of two bf16 values is exact in double.
 */
uint16_t oracle_dequant_act_bf16(int8_t q, float beta)
{
    float s = beta / (float)ORACLE_QB_MINUS_1;
    return oracle_f32_to_bf16((float)q * s);
}

void oracle_backward(const int8_t *wq, float gamma, const int8_t *xq, const float *beta,
                     const uint16_t *dY, int64_t T, int64_t N, int64_t K, double *dX,
                     double *dW)
{
    if (dX) {
        for (int64_t t = 0; t < T; ++t)
            for (int64_t k = 0; k < K; ++k) {
                double s = 0.0;
                for (int64_t o = 0; o < N; ++o)
                    s += (double)oracle_bf16_to_f32(dY[t * N + o]) * (double)wq[o * K + k];
                dX[t * K + k] = (double)gamma * s;
            }
    }
    if (dW) {
        for (int64_t o = 0; o < N; ++o)
            for (int64_t k = 0; k < K; ++k) {
                double s = 0.0;
                for (int64_t t = 0; t < T; ++t) {
                    double xh = (double)oracle_bf16_to_f32(
                        oracle_dequant_act_bf16(xq[t * K + k], beta[t]));
                    s += (double)oracle_bf16_to_f32(dY[t * N + o]) * xh;
                }
                dW[o * K + k] = (double)gamma * s;
            }
    }
}
