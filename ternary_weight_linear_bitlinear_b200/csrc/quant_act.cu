// quant_act.cu -- fused RMSNorm + absmax int8 activation codes (per token, or
// per tensor).
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 2,
// "Activation Quantization: Absmax Scaling": activations are RMS-normalised,
// beta = max |x| (taken per token), X~ = RoundClip(x (Q_b-1)/(beta+eps),
// -(Q_b-1), Q_b-1) with Q_b - 1 = 127.
//
// One CTA of kQuantThreads per token: one pass for the sum of squares and the
// absmax (one more when a gain vector is set), one pass for the codes; the
// row is re-read from L1.  RMSNorm multiplies by the token's reciprocal RMS.
// Besides the codes the kernel writes the row sum of the codes, which the
// product kernels use to turn their offset-code sums into W~ X~.  The
// reduction order is the one of quant_common.cuh, shared with the fused
// decode kernel.
//
// 4-bit codes (BITLINEAR_ACT_4BIT, the A4 of the W1A4 regime): the same
// section's Q_b = 2^(k-1) with k = 4, so the multiplier and the clip bound
// are 7 instead of 127.
//
// Per-tensor scope (the same section prints beta as the max over all i, j):
// three launches -- every token's statistics (beta[t] = its own absmax), one
// CTA folding them into beta[0] = max_t beta[t], then every token's codes on
// that one beta (recomputing its reciprocal RMS in the same order), each
// token's beta[t] set to it.
#include <cmath>
#include <cstdint>

#include "bitlinear.h"
#include "common.cuh"
#include "quant_common.cuh"

namespace bl {

enum QuantMode : int {
    kQuantPerToken = 0,     // statistics and codes of each token
    kQuantStatsOnly = 1,    // statistics only: beta[t] = the token's absmax
    kQuantSharedBeta = 2,   // codes on the one beta held in beta[0]
};

__global__ void __launch_bounds__(kQuantThreads)
quant_act_kernel(const uint16_t *__restrict__ X, int d_in, const float *__restrict__ gain,
                 int rmsnorm, float eps, float norm_eps, double inv_k, float qmax,
                 const float *__restrict__ inv_rms_in,
                 int8_t *__restrict__ Xq, float *__restrict__ beta_out,
                 int32_t *__restrict__ rowsum, float *__restrict__ inv_rms_out, int mode) {
    __shared__ QuantShared<1> qs;
    const int64_t t = blockIdx.x;

    // A dependent product kernel may launch at once: it reads nothing this
    // kernel or earlier work writes before its own dependency wait, except
    // weights its caller declared static.  This kernel reads X only after
    // everything enqueued before it is complete (a no-op for an ordinary
    // launch).
    pdl_launch_dependents();
    pdl_wait_primary();

    const uint16_t *row = X + t * d_in;
    token_stats<1>(row, 1, d_in, gain, rmsnorm != 0, eps, norm_eps, inv_k, qmax,
                   inv_rms_in ? inv_rms_in + t : nullptr, qs);
    if (mode == kQuantStatsOnly) {
        if (threadIdx.x == 0) {
            beta_out[t] = qs.beta[0];
            if (inv_rms_out) inv_rms_out[t] = qs.inv_rms[0];
        }
        return;
    }
    if (mode == kQuantSharedBeta) {
        // Every CTA reads the same beta[0] and token 0 rewrites it with the
        // same value.
        if (threadIdx.x == 0) {
            const float b = beta_out[0];
            qs.beta[0] = b;
            qs.scale[0] = __fdiv_rn(qmax, __fadd_rn(b, eps));
        }
        quant_barrier();
    }
    token_codes<1>(row, 1, d_in, gain, rmsnorm != 0, Xq + t * d_in, qs);
    if (threadIdx.x == 0) {
        beta_out[t] = qs.beta[0];
        rowsum[t] = qs.rowsum[0];
        if (inv_rms_out) inv_rms_out[t] = qs.inv_rms[0];
    }
}

// beta[0] = max_t beta[t] (non-negative values), one CTA.
constexpr int kBetaMaxThreads = 1024;
__global__ void __launch_bounds__(kBetaMaxThreads) beta_max_kernel(float *beta, int64_t T) {
    __shared__ float part[kBetaMaxThreads / 32];
    float m = 0.0f;
    for (int64_t i = threadIdx.x; i < T; i += kBetaMaxThreads) m = fmaxf(m, beta[i]);
    m = warp_max_f32(m);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = part[threadIdx.x];
        m = warp_max_f32(m);
        if (threadIdx.x == 0) beta[0] = m;
    }
}

// The per-token quantiser's launch as a launch record (parameter 0 is X).
bitlinear_status prepare_quant_act(const uint16_t *X, int64_t T, int64_t d_in,
                                   const float *norm_gain, uint32_t flags, float eps,
                                   float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                   float *beta, int32_t *rowsum, float *inv_rms_out, bool pdl,
                                   LaunchRec *rec) {
    *rec = LaunchRec();
    rec->func = (const void *)quant_act_kernel;
    rec->grid = dim3((unsigned)T);
    rec->block = dim3(kQuantThreads);
    rec->pdl = pdl;
    rec->push(X);
    rec->push((int)d_in);
    rec->push(norm_gain);
    rec->push((flags & BITLINEAR_RMSNORM) ? 1 : 0);
    rec->push(eps);
    rec->push(norm_eps);
    rec->push(1.0 / (double)d_in);
    rec->push((flags & BITLINEAR_ACT_4BIT) ? 7.0f : 127.0f);
    rec->push(inv_rms_in);
    rec->push(Xq);
    rec->push(beta);
    rec->push(rowsum);
    rec->push(inv_rms_out);
    rec->push((int)kQuantPerToken);
    return BITLINEAR_OK;
}

bitlinear_status launch_quant_act(const uint16_t *X, int64_t T, int64_t d_in,
                                  const float *norm_gain, uint32_t flags, float eps,
                                  float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                  float *beta, int32_t *rowsum, float *inv_rms_out, bool pdl,
                                  cudaStream_t stream) {
    const int rmsnorm = (flags & BITLINEAR_RMSNORM) ? 1 : 0;
    const bool per_tensor = (flags & BITLINEAR_PER_TENSOR_ABSMAX) != 0;
    if (!per_tensor) {
        LaunchRec rec;
        prepare_quant_act(X, T, d_in, norm_gain, flags, eps, norm_eps, inv_rms_in, Xq, beta,
                          rowsum, inv_rms_out, pdl, &rec);
        return rec.launch(stream) == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)T);
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const double inv_k = 1.0 / (double)d_in;
    // Q_b - 1 for 8-bit codes (127) or, under BITLINEAR_ACT_4BIT, 4-bit (7).
    const float qmax = (flags & BITLINEAR_ACT_4BIT) ? 7.0f : 127.0f;
    cudaError_t e = cudaLaunchKernelEx(&cfg, quant_act_kernel, X, (int)d_in, norm_gain, rmsnorm, eps,
                           norm_eps, inv_k, qmax, inv_rms_in, Xq, beta, rowsum, inv_rms_out,
                           (int)kQuantStatsOnly);
    if (e != cudaSuccess) return BITLINEAR_ERR_CUDA;
    beta_max_kernel<<<1, kBetaMaxThreads, 0, stream>>>(beta, T);
    if (cudaGetLastError() != cudaSuccess) return BITLINEAR_ERR_CUDA;
    cfg.numAttrs = 0;   // the codes need the folded beta: an ordinary stream-ordered launch
    e = cudaLaunchKernelEx(&cfg, quant_act_kernel, X, (int)d_in, norm_gain, rmsnorm, eps,
                           norm_eps, inv_k, qmax, inv_rms_in, Xq, beta, rowsum, inv_rms_out,
                           (int)kQuantSharedBeta);
    return e == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

}  // namespace bl

using namespace bl;

extern "C" int bitlinear_quant_act(const uint16_t *X, int64_t T, int64_t d_in,
                                   const float *norm_gain, uint32_t flags, float eps,
                                   float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                   float *beta, int32_t *rowsum, float *inv_rms_out,
                                   cudaStream_t stream) {
    if (T < 0 || T > (1 << 20)) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (d_in <= 0 || d_in % 256 || d_in > 65536) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (flags & ~(BITLINEAR_RMSNORM | BITLINEAR_PER_TENSOR_ABSMAX | BITLINEAR_ACT_4BIT))
        return BITLINEAR_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BITLINEAR_ERR_INVALID_ARG;
    if (!(norm_eps >= 0.0f) || !std::isfinite(norm_eps)) return BITLINEAR_ERR_INVALID_ARG;
    if (T == 0) return BITLINEAR_OK;
    if (!X || !Xq || !beta || !rowsum) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(beta, 4) || !aligned(rowsum, 4))
        return BITLINEAR_ERR_MISALIGNED;
    if ((norm_gain && !aligned(norm_gain, 4)) || (inv_rms_in && !aligned(inv_rms_in, 4)) ||
        (inv_rms_out && !aligned(inv_rms_out, 4)))
        return BITLINEAR_ERR_MISALIGNED;
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;

    return launch_quant_act(X, T, d_in, norm_gain, flags, eps, norm_eps, inv_rms_in, Xq, beta,
                            rowsum, inv_rms_out, false, stream);
}
