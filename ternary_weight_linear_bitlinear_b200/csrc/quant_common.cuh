// quant_common.cuh -- per-token RMSNorm / absmax statistics and int8 codes,
// shared by the stand-alone quantiser and the fused decode kernel so that both
// reduce in one canonical order and produce bit-identical results.
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 2,
// "Activation Quantization: Absmax Scaling".
//
// RMSNorm is n = x * r (* g) with the reciprocal RMS r = 1 / sqrt(mean(x^2) +
// norm_eps) formed once per token (see inv_rms_from_ss) and rounded to
// binary32.
// Canonical order (a CTA of kQuantThreads threads): thread i owns the 16-byte
// vectors i, i + kQuantThreads, ... of a token row and accumulates, in double
// and in that order, each vector's sum of squares (sq_sum8); a warp
// xor-butterfly combines the 32 lanes; the kQuantWarps warp sums are added in
// warp order.  Without a gain vector
// beta = fl(max|x| * r): correctly rounded multiplication by r > 0 is
// monotone, so this is exactly max_k fl(|x_k| * r).  With a gain it is the
// max of the normalised values themselves.
//
// Tokens are processed in a loop that is not unrolled, keeping the code small
// (a fully unrolled multi-token version spent most of its time on
// instruction-cache misses).
#pragma once

#include <cstdint>

#include "common.cuh"

namespace bl {

constexpr int kQuantThreads = 128;
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kQuantBatch = 8;   // 16-byte loads in flight per thread

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 &v, float (&x)[8]) {
    x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x);
    x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
    x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z);
    x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}

// Shared scratch for the statistics of up to TMAX tokens.
template <int TMAX>
struct QuantShared {
    double ss[kQuantWarps][TMAX];
    float amax[kQuantWarps][TMAX];
    int sum[kQuantWarps][TMAX];
    float inv_rms[TMAX];
    float beta[TMAX];
    float scale[TMAX];   // qmax / (beta + eps)
    int rowsum[TMAX];
};

// Barrier over the kQuantThreads threads (warps 0..kQuantWarps-1) that run
// the quantiser; a CTA may hold further warps that do not take part.
__device__ __forceinline__ void quant_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(kQuantThreads) : "memory");
}

// Reciprocal RMS from the sum of squares: r = 1 / sqrt(ss * inv_k + norm_eps)
// rounded to binary32.  A single-precision estimate refined by one Newton
// step in double (relative error ~1e-13 before the final rounding); outside
// [1e-30, 1e30] the correctly rounded double sequence is used instead.  The
// same fixed sequence runs in every kernel that quantises, so they agree bit
// for bit; against the sequential double computation it agrees to far
// better than the 1e-6 relative the tests require.
__device__ __forceinline__ float inv_rms_from_ss(double ss, double inv_k, float norm_eps) {
    const double x = __dadd_rn(__dmul_rn(ss, inv_k), (double)norm_eps);
    if (x > 1e-30 && x < 1e30) {
        const double y0 = (double)rsqrtf((float)x);
        const double t = __dmul_rn(__dmul_rn(x, y0), y0);
        return (float)__dmul_rn(y0, __fma_rn(-0.5, t, 1.5));
    }
    return (float)__ddiv_rn(1.0, __dsqrt_rn(x));
}

// Sum of the squares of eight bf16 values, returned in double.  A bf16 value
// has an 8-bit significand, so its square is exact in binary32 whenever it
// neither overflows nor leaves the normal range; the eight squares are then
// added as a fixed pairwise tree in binary32 (relative error at most 3 x
// 2^-24).  When that sum is not finite or below 2^-100 (huge or tiny inputs)
// the squares are formed and added sequentially in double instead.
__device__ __forceinline__ double sq_sum8(const float (&x)[8]) {
    // fma(x1, x1, x0 * x0) is fl(p0 + p1) itself, since both squares are
    // exact: the pairs of the tree cost one multiply and one fma.
    float p[4];
    #pragma unroll
    for (int j = 0; j < 4; ++j)
        p[j] = __fmaf_rn(x[2 * j + 1], x[2 * j + 1], __fmul_rn(x[2 * j], x[2 * j]));
    const float s = __fadd_rn(__fadd_rn(p[0], p[1]), __fadd_rn(p[2], p[3]));
    if (s >= 0x1p-100f && s <= 3.40282347e38f) return (double)s;
    double d = 0.0;
    #pragma unroll
    for (int j = 0; j < 8; ++j) d = __dadd_rn(d, __dmul_rn((double)x[j], (double)x[j]));
    return d;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
// Maximum over the warp of non-negative finite floats: their bit patterns
// order as unsigned integers, so one integer reduction gives it exactly.
__device__ __forceinline__ float warp_max_f32(float v) {
    return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
}
__device__ __forceinline__ int warp_sum_i32(int v) {
    return __reduce_add_sync(0xffffffffu, v);
}

// The activation code floor(v + 0.5) as the bit pattern of the binary32
// value 1.5 * 2^23 + code.  u = fl_rd(v + 0.5) keeps floor(v + 0.5) (see
// round_half_up_int); adding 1.5 * 2^23 rounding down lands in [2^23, 2^24),
// where the spacing is 1, exactly at 1.5 * 2^23 + floor(u).  The low byte is
// then the code in two's complement, and the pattern minus kCodeBias is the
// code itself.  Valid for |v| < 2^22; the quantiser's v never exceeds
// qmax (1 + 2^-23) in magnitude (qmax = Q_b - 1 = 127 for 8-bit codes, 7 for
// 4-bit): |n| <= beta because beta is the absmax of the same rounded
// products, and fl(qmax / (beta + eps)) <= (qmax / beta)(1 + 2^-24), so
// floor(v + 0.5) already lies in [-qmax, qmax] and the clip is a no-op.
constexpr uint32_t kCodeBias = 0x4B400000u;   // bit pattern of 1.5 * 2^23
__device__ __forceinline__ uint32_t code_bits(float v) {
    return __float_as_uint(__fadd_rd(__fadd_rd(v, 0.5f), 12582912.0f));
}
// Low bytes of four code patterns, little-endian.
__device__ __forceinline__ uint32_t pack_code_bytes(uint32_t b0, uint32_t b1, uint32_t b2,
                                                    uint32_t b3) {
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// Statistics of tokens 0..T-1 (T <= TMAX) of X [T][K] (bf16 bits).  Threads
// 0..kQuantThreads-1 of the CTA must all call it.  inv_rms_in, when
// given, supplies the per-token reciprocal RMS.  Results: qs.inv_rms, beta,
// scale.
// Per-warp partial statistics of token rows in the canonical order (thread i
// owns vectors i, i + kQuantThreads, ...; xor-butterfly within the warp),
// written to qs.ss[warp][t] / qs.amax[warp][t].  No barrier.  X in shared
// memory.
template <int TMAX>
__device__ __forceinline__ void token_partials_smem(const uint16_t *X, int T, int K,
                                                    bool need_ss, QuantShared<TMAX> &qs) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nvec = K >> 3;
    #pragma unroll 1
    for (int t = 0; t < T; ++t) {
        const uint4 *row = reinterpret_cast<const uint4 *>(X + (size_t)t * K);
        double ss = 0.0;
        float am = 0.0f;
        for (int v = tid; v < nvec; v += kQuantThreads) {
            float x[8];
            unpack8(row[v], x);
            if (need_ss) ss = __dadd_rn(ss, sq_sum8(x));
            #pragma unroll
            for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(x[j]));
        }
        ss = warp_sum_f64(ss);
        am = warp_max_f32(am);
        if (lane == 0) {
            qs.ss[warp][t] = ss;
            qs.amax[warp][t] = am;
        }
    }
}

struct TokenScale {
    float inv_rms;   // r (1 without RMSNorm)
    float beta;      // absmax of the normalised row
    float scale;     // qmax / (beta + eps)
};

// Final statistics of token t from the warp partials (fixed warp order); any
// thread may compute them and every thread gets the same bits.  No gain.
// inv_rms_in, when given, supplies r.
template <int TMAX>
__device__ __forceinline__ TokenScale token_finalize(int t, bool rmsnorm, float eps,
                                                     float norm_eps, double inv_k, float qmax,
                                                     const float *inv_rms_in,
                                                     const QuantShared<TMAX> &qs) {
    TokenScale ts;
    ts.inv_rms = 1.0f;
    if (rmsnorm && inv_rms_in) {
        ts.inv_rms = __ldg(inv_rms_in + t);
    } else if (rmsnorm) {
        double s = qs.ss[0][t];
        #pragma unroll
        for (int w = 1; w < kQuantWarps; ++w) s += qs.ss[w][t];
        ts.inv_rms = inv_rms_from_ss(s, inv_k, norm_eps);
    }
    float m = qs.amax[0][t];
    #pragma unroll
    for (int w = 1; w < kQuantWarps; ++w) m = fmaxf(m, qs.amax[w][t]);
    ts.beta = rmsnorm ? __fmul_rn(m, ts.inv_rms) : m;
    ts.scale = __fdiv_rn(qmax, __fadd_rn(ts.beta, eps));
    return ts;
}

// Eight codes of one 16-byte vector of bf16 activations, packed little-endian
// into two words; adds their sum to *sum.  No gain.
__device__ __forceinline__ uint2 codes8(const uint4 &v, bool rmsnorm, float r, float scale,
                                        int *sum) {
    float x[8];
    unpack8(v, x);
    uint32_t b[8];
    #pragma unroll
    for (int j = 0; j < 8; ++j) {
        float n = x[j];
        if (rmsnorm) n = __fmul_rn(n, r);
        b[j] = code_bits(__fmul_rn(n, scale));
        *sum += (int)(b[j] - kCodeBias);
    }
    return make_uint2(pack_code_bytes(b[0], b[1], b[2], b[3]),
                      pack_code_bytes(b[4], b[5], b[6], b[7]));
}

// Row loads: read-only global path, or plain loads when X was staged in
// shared memory.
template <bool kSmemSrc>
__device__ __forceinline__ uint4 load_row_vec(const uint4 *row, int v) {
    if constexpr (kSmemSrc) return row[v];
    else return __ldg(row + v);
}

template <int TMAX, bool kSmemSrc = false>
__device__ __forceinline__ void token_stats(const uint16_t *__restrict__ X, int T, int K,
                                         const float *__restrict__ gain, bool rmsnorm,
                                         float eps, float norm_eps, double inv_k, float qmax,
                                         const float *__restrict__ inv_rms_in,
                                         QuantShared<TMAX> &qs) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nvec = K >> 3;
    const bool need_ss = rmsnorm && !inv_rms_in;
    #pragma unroll 1
    for (int t = 0; t < T; ++t) {
        const uint4 *row = reinterpret_cast<const uint4 *>(X + (size_t)t * K);
        double ss = 0.0;
        float am = 0.0f;
        // Loads are issued kQuantBatch at a time, then consumed in order.
        for (int v0 = tid; v0 < nvec; v0 += kQuantBatch * kQuantThreads) {
            uint4 buf[kQuantBatch];
            #pragma unroll
            for (int b = 0; b < kQuantBatch; ++b) {
                const int v = v0 + b * kQuantThreads;
                if (v < nvec) buf[b] = load_row_vec<kSmemSrc>(row, v);
            }
            #pragma unroll
            for (int b = 0; b < kQuantBatch; ++b) {
                if (v0 + b * kQuantThreads < nvec) {
                    float x[8];
                    unpack8(buf[b], x);
                    if (need_ss) ss = __dadd_rn(ss, sq_sum8(x));
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(x[j]));
                }
            }
        }
        ss = warp_sum_f64(ss);
        am = warp_max_f32(am);
        if (lane == 0) {
            qs.ss[warp][t] = ss;
            qs.amax[warp][t] = am;
        }
    }
    quant_barrier();
    if (tid < T) {
        const int t = tid;
        if (rmsnorm && inv_rms_in) {
            const float r = inv_rms_in[t];
            float m = qs.amax[0][t];
            #pragma unroll
            for (int w = 1; w < kQuantWarps; ++w) m = fmaxf(m, qs.amax[w][t]);
            qs.inv_rms[t] = r;
            qs.beta[t] = __fmul_rn(m, r);
        } else {
            const TokenScale ts =
                token_finalize<TMAX>(t, rmsnorm, eps, norm_eps, inv_k, qmax, nullptr, qs);
            qs.inv_rms[t] = ts.inv_rms;
            qs.beta[t] = ts.beta;                    // replaced below when a gain is set
        }
    }
    quant_barrier();
    if (rmsnorm && gain) {
        // With a gain the absmax is that of fl(fl(x * r) * g).
        #pragma unroll 1
        for (int t = 0; t < T; ++t) {
            const uint4 *row = reinterpret_cast<const uint4 *>(X + (size_t)t * K);
            const float r = qs.inv_rms[t];
            float a = 0.0f;
            for (int v = tid; v < nvec; v += kQuantThreads) {
                float x[8];
                unpack8(load_row_vec<kSmemSrc>(row, v), x);
                #pragma unroll
                for (int j = 0; j < 8; ++j)
                    a = fmaxf(a, fabsf(__fmul_rn(__fmul_rn(x[j], r), __ldg(gain + 8 * v + j))));
            }
            a = warp_max_f32(a);
            if (lane == 0) qs.amax[warp][t] = a;
        }
        quant_barrier();
        if (tid < T) {
            float m = qs.amax[0][tid];
            #pragma unroll
            for (int w = 1; w < kQuantWarps; ++w) m = fmaxf(m, qs.amax[w][tid]);
            qs.beta[tid] = m;
        }
        quant_barrier();
    }
    if (tid < T) qs.scale[tid] = __fdiv_rn(qmax, __fadd_rn(qs.beta[tid], eps));
    quant_barrier();
}

// Codes of tokens 0..T-1 written to dst (row stride K bytes; global or shared
// memory) and their row sums to qs.rowsum.  Call after token_stats.
template <int TMAX, bool kSmemSrc = false>
__device__ __forceinline__ void token_codes(const uint16_t *__restrict__ X, int T, int K,
                                         const float *__restrict__ gain, bool rmsnorm,
                                         int8_t *dst, QuantShared<TMAX> &qs) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nvec = K >> 3;
    const bool use_gain = rmsnorm && gain;
    #pragma unroll 1
    for (int t = 0; t < T; ++t) {
        const uint4 *row = reinterpret_cast<const uint4 *>(X + (size_t)t * K);
        uint2 *out = reinterpret_cast<uint2 *>(dst + (size_t)t * K);
        const float r = rmsnorm ? qs.inv_rms[t] : 1.0f, scale = qs.scale[t];
        int sum = 0;
        for (int v0 = tid; v0 < nvec; v0 += kQuantBatch * kQuantThreads) {
            uint4 buf[kQuantBatch];
            #pragma unroll
            for (int b = 0; b < kQuantBatch; ++b) {
                const int v = v0 + b * kQuantThreads;
                if (v < nvec) buf[b] = load_row_vec<kSmemSrc>(row, v);
            }
            #pragma unroll
            for (int b = 0; b < kQuantBatch; ++b) {
                const int v = v0 + b * kQuantThreads;
                if (v < nvec) {
                    float x[8];
                    unpack8(buf[b], x);
                    float g[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
                    if (use_gain) {
                        #pragma unroll
                        for (int j = 0; j < 8; ++j) g[j] = __ldg(gain + 8 * v + j);
                    }
                    uint32_t bb[8];
                    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float n = x[j];
                        if (rmsnorm) n = __fmul_rn(n, r);
                        if (use_gain) n = __fmul_rn(n, g[j]);
                        bb[j] = code_bits(__fmul_rn(n, scale));
                        sum += (int)(bb[j] - kCodeBias);
                    }
                    out[v] = make_uint2(pack_code_bytes(bb[0], bb[1], bb[2], bb[3]),
                                        pack_code_bytes(bb[4], bb[5], bb[6], bb[7]));
                }
            }
        }
        sum = warp_sum_i32(sum);
        if (lane == 0) qs.sum[warp][t] = sum;
    }
    quant_barrier();
    if (tid < T) {
        int s = 0;
        #pragma unroll
        for (int w = 0; w < kQuantWarps; ++w) s += qs.sum[w][tid];
        qs.rowsum[tid] = s;
    }
    quant_barrier();
}

}  // namespace bl
