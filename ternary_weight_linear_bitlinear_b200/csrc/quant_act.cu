// quant_act.cu -- fused RMSNorm + per-token absmax int8 activation codes.
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 2,
// "Activation Quantization: Absmax Scaling": activations are RMS-normalised,
// beta = max |x| (taken per token), X~ = RoundClip(x (Q_b-1)/(beta+eps),
// -(Q_b-1), Q_b-1) with Q_b - 1 = 127.
//
// One CTA per token.  The row (at most 64 KiB of bf16) is read with 16-byte
// loads; the three passes (sum of squares, absmax, codes) re-read it from
// L1.  Besides the codes the kernel writes the row sum of the codes, which
// the product kernels use to turn their offset-code sums into W~ X~.
#include <cmath>
#include <cstdint>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {

constexpr int kQThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 &v, float (&x)[8]) {
    x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x);
    x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
    x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z);
    x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, T *sh, Op op) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sh[warp] = v;
    __syncthreads();
    T r = sh[0];
    #pragma unroll
    for (int w = 1; w < kQThreads / 32; ++w) r = op(r, sh[w]);
    __syncthreads();
    return r;  // same value in every thread, fixed order
}

__global__ void __launch_bounds__(kQThreads)
quant_act_kernel(const uint16_t *__restrict__ X, int64_t T, int d_in,
                 const float *__restrict__ gain, int rmsnorm, float eps, float norm_eps,
                 const float *__restrict__ rms_in, int8_t *__restrict__ Xq,
                 float *__restrict__ beta_out, int32_t *__restrict__ rowsum,
                 float *__restrict__ rms_out) {
    __shared__ double shd[kQThreads / 32];
    __shared__ float shf[kQThreads / 32];
    __shared__ int shi[kQThreads / 32];
    const int64_t t = blockIdx.x;
    const uint4 *row = reinterpret_cast<const uint4 *>(X + t * d_in);
    const int nvec = d_in >> 3;

    // Everything enqueued before this kernel is complete past this point
    // (a no-op for an ordinary launch).  Only then may a dependent product
    // kernel start streaming weights, which nothing after this point writes.
    pdl_wait_primary();
    pdl_launch_dependents();

    float rms = 1.0f;
    if (rmsnorm) {
        if (rms_in) {
            rms = rms_in[t];
        } else {
            double ss = 0.0;
            for (int i = threadIdx.x; i < nvec; i += kQThreads) {
                float x[8];
                unpack8(__ldg(row + i), x);
                #pragma unroll
                for (int j = 0; j < 8; ++j) ss += (double)x[j] * (double)x[j];
            }
            ss = block_reduce(ss, shd, [](double a, double b) { return a + b; });
            rms = (float)__dsqrt_rn(__dadd_rn(ss / (double)d_in, (double)norm_eps));
        }
    }

    float amax = 0.0f;
    for (int i = threadIdx.x; i < nvec; i += kQThreads) {
        float x[8];
        unpack8(__ldg(row + i), x);
        #pragma unroll
        for (int j = 0; j < 8; ++j) {
            float n = x[j];
            if (rmsnorm) {
                n = __fdiv_rn(n, rms);
                if (gain) n = __fmul_rn(n, __ldg(gain + i * 8 + j));
            }
            amax = fmaxf(amax, fabsf(n));
        }
    }
    const float beta = block_reduce(amax, shf, [](float a, float b) { return fmaxf(a, b); });
    const float scale = __fdiv_rn(127.0f, __fadd_rn(beta, eps));

    int sum = 0;
    uint2 *qrow = reinterpret_cast<uint2 *>(Xq + t * d_in);
    for (int i = threadIdx.x; i < nvec; i += kQThreads) {
        float x[8];
        unpack8(__ldg(row + i), x);
        uint32_t lo = 0, hi = 0;
        #pragma unroll
        for (int j = 0; j < 8; ++j) {
            float n = x[j];
            if (rmsnorm) {
                n = __fdiv_rn(n, rms);
                if (gain) n = __fmul_rn(n, __ldg(gain + i * 8 + j));
            }
            float q = round_half_up_exact(__fmul_rn(n, scale));
            q = fminf(fmaxf(q, -127.0f), 127.0f);
            const int qi = (int)q;
            sum += qi;
            const uint32_t b = (uint32_t)(qi & 0xff);
            if (j < 4) lo |= b << (8 * j); else hi |= b << (8 * (j - 4));
        }
        qrow[i] = make_uint2(lo, hi);
    }
    sum = block_reduce(sum, shi, [](int a, int b) { return a + b; });
    if (threadIdx.x == 0) {
        beta_out[t] = beta;
        rowsum[t] = sum;
        if (rms_out) rms_out[t] = rms;
    }
}

bitlinear_status launch_quant_act(const uint16_t *X, int64_t T, int64_t d_in,
                                  const float *norm_gain, uint32_t flags, float eps,
                                  float norm_eps, const float *rms_in, int8_t *Xq, float *beta,
                                  int32_t *rowsum, float *rms_out, cudaStream_t stream) {
    const int rmsnorm = (flags & BITLINEAR_RMSNORM) ? 1 : 0;
    quant_act_kernel<<<(unsigned)T, kQThreads, 0, stream>>>(X, T, (int)d_in, norm_gain, rmsnorm,
                                                            eps, norm_eps, rms_in, Xq, beta,
                                                            rowsum, rms_out);
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

}  // namespace bl

using namespace bl;

extern "C" int bitlinear_quant_act(const uint16_t *X, int64_t T, int64_t d_in,
                                   const float *norm_gain, uint32_t flags, float eps,
                                   float norm_eps, const float *rms_in, int8_t *Xq,
                                   float *beta, int32_t *rowsum, float *rms_out,
                                   cudaStream_t stream) {
    if (T < 0 || T > (1 << 20)) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (d_in <= 0 || d_in % 256 || d_in > 65536) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (flags & ~BITLINEAR_RMSNORM) return BITLINEAR_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BITLINEAR_ERR_INVALID_ARG;
    if (!(norm_eps >= 0.0f) || !std::isfinite(norm_eps)) return BITLINEAR_ERR_INVALID_ARG;
    if (T == 0) return BITLINEAR_OK;
    if (!X || !Xq || !beta || !rowsum) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(beta, 4) || !aligned(rowsum, 4))
        return BITLINEAR_ERR_MISALIGNED;
    if ((norm_gain && !aligned(norm_gain, 4)) || (rms_in && !aligned(rms_in, 4)) ||
        (rms_out && !aligned(rms_out, 4)))
        return BITLINEAR_ERR_MISALIGNED;
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;

    return launch_quant_act(X, T, d_in, norm_gain, flags, eps, norm_eps, rms_in, Xq, beta,
                            rowsum, rms_out, stream);
}
