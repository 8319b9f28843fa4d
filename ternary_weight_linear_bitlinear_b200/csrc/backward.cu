// backward.cu -- BitLinear backward pass with the straight-through estimator.
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 3,
// "Training Dynamics and the Straight-Through Estimator": the rounding of
// the quantisers is bypassed in the backward pass, so the layer acts as
// Y = X^ (gamma W~)^T with X^ = X~ beta / 127 and gamma, beta held constant:
//
//   dX = gamma dY W~          [T][d_in]   (gradient at X^)
//   dW = gamma dY^T X^        [d_out][d_in] (gradient at W~, for the latent
//                                          weights)
//
// Both are dense contractions, run on the tcgen05 bf16 GEMM of
// dense_bf16.cu with gamma applied in its fp32 epilogue and the operands read
// in their natural layouts (MN-major where the reduction index is the row):
//   * dX: A = W~ [d_out][d_in] as bf16 {-1, 0, 1} (exact; expand_ternary_kernel
//     writes it from the packed codes), read MN-major; B = dY [T][d_out];
//   * dW: A = X^ [T][d_in] as bf16 of fl32(q fl32(beta / 127))
//     (dequant_kernel), B = dY [T][d_out], both read MN-major; the copies
//     zero-fill the token rows past T.
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {

bitlinear_status launch_dense_bf16(const uint16_t *W, int64_t d_out, int64_t d_in,
                                   const uint16_t *X, int64_t T, void *Y, int out_dtype,
                                   const float *alpha, cudaStream_t stream);

bitlinear_status launch_dense_gemm_mn(const uint16_t *A, bool a_mn, const uint16_t *B, bool b_mn,
                                      int64_t M, int64_t N, int64_t K, void *Y, int out_dtype,
                                      const float *alpha, cudaStream_t stream);

constexpr int kBwThreads = 256;

// W~ as bf16, [d_out][d_in]: one thread per packed word (16 weights of one
// row); word kw of a tile row holds columns 16 kw + 4 s + b in bits 8 b + 2 s
// as W~ + 1, so the 16 values are written as 32 contiguous bytes.
__global__ void __launch_bounds__(kBwThreads)
expand_ternary_kernel(const uint32_t *__restrict__ packed, int64_t d_out, int kb_total,
                      uint16_t *__restrict__ wt) {
    const int64_t nwords = d_out * kb_total * 16;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t d_in = (int64_t)kb_total * 256;
    for (int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < nwords; wi += stride) {
        const int64_t tile = wi >> 8;
        const int within = (int)(wi & 255);
        const int r = within >> 4, kw = within & 15;
        const int64_t rb = tile / kb_total, kb = tile - rb * kb_total;
        const uint32_t w = __ldg(packed + wi);
        uint32_t v[8];   // bf16 pairs of columns 16 kw + 2 i, 2 i + 1
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t h[2];
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = 2 * i + e, s = col >> 2, b = col & 3;
                const uint32_t c = (w >> (8 * b + 2 * s)) & 3u;     // W~ + 1
                h[e] = c == 1u ? 0u : (c == 0u ? 0xBF80u : 0x3F80u);  // bf16 -1, 0, +1
            }
            v[i] = h[0] | (h[1] << 16);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(wt + (rb * 16 + r) * d_in + kb * 256 + kw * 16);
        dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
        dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
    }
}

// X^ as bf16, [T][d_in]: one thread per 16 codes of one token.
__global__ void __launch_bounds__(kBwThreads)
dequant_kernel(const int8_t *__restrict__ xq, const float *__restrict__ beta, int64_t T, int K,
               uint16_t *__restrict__ xh) {
    const int64_t nvec = T * (K / 16);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t vi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; vi < nvec; vi += stride) {
        const int64_t t = vi / (K / 16);
        const uint4 q = __ldg(reinterpret_cast<const uint4 *>(xq) + vi);
        const float sc = __fdiv_rn(beta[t], 127.0f);
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
        uint32_t v[8];
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t h[2];
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int j = 2 * i + e;
                const int code = (int)(int8_t)((qw[j >> 2] >> (8 * (j & 3))) & 0xFFu);
                h[e] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)code, sc)));
            }
            v[i] = h[0] | (h[1] << 16);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(xh) + vi * 2;
        dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
        dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
    }
}

struct BackwardLayout {
    size_t wt, xh, total;   // byte offsets of the two bf16 operands, total bytes
};

static BackwardLayout backward_layout(int64_t d_out, int64_t d_in, int64_t T, bool want_dx,
                                      bool want_dw) {
    BackwardLayout l = {};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) / 256 * 256;
        return at;
    };
    l.wt = want_dx ? take((size_t)d_in * d_out * 2) : 0;
    l.xh = want_dw ? take((size_t)d_in * (T > 0 ? T : 1) * 2) : 0;
    l.total = off;
    return l;
}

static bool backward_shape_ok(int64_t d_out, int64_t d_in, int64_t T) {
    return T >= 0 && T <= 65536 && d_out > 0 && d_out % 256 == 0 && d_out <= 65536 &&
           d_in > 0 && d_in % 256 == 0 && d_in <= 65536;
}

}  // namespace bl

using namespace bl;

extern "C" size_t bitlinear_backward_workspace_bytes(int64_t d_out, int64_t d_in, int64_t T,
                                                     int want_dx, int want_dw) {
    if (!backward_shape_ok(d_out, d_in, T)) return 0;
    return backward_layout(d_out, d_in, T, want_dx != 0, want_dw != 0).total;
}

extern "C" int bitlinear_backward(const uint32_t *packed, const float *gamma, int64_t d_out,
                                  int64_t d_in, const int8_t *Xq, const float *beta, int64_t T,
                                  const uint16_t *dY, void *dX, void *dW, int out_dtype,
                                  void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!backward_shape_ok(d_out, d_in, T)) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (out_dtype != BITLINEAR_OUT_F32 && out_dtype != BITLINEAR_OUT_BF16)
        return BITLINEAR_ERR_INVALID_ARG;
    const bool want_dx = dX != nullptr, want_dw = dW != nullptr;
    if (!want_dx && !want_dw) return BITLINEAR_ERR_INVALID_ARG;
    if (!packed || !gamma) return BITLINEAR_ERR_INVALID_ARG;
    if (T > 0 && (!dY || (want_dw && (!Xq || !beta)))) return BITLINEAR_ERR_INVALID_ARG;
    const BackwardLayout lay = backward_layout(d_out, d_in, T, want_dx, want_dw);
    if (T > 0 && (!workspace || workspace_bytes < lay.total)) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(gamma, 4) || (dY && !aligned(dY, 16)) ||
        (Xq && !aligned(Xq, 16)) || (beta && !aligned(beta, 4)) || (dX && !aligned(dX, 16)) ||
        (dW && !aligned(dW, 16)) || (workspace && !aligned(workspace, 256)))
        return BITLINEAR_ERR_MISALIGNED;
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;
    const size_t esize = out_dtype == BITLINEAR_OUT_BF16 ? 2 : 4;
    if (T == 0) {
        // No tokens: dW is zero, dX has no rows.
        if (want_dw && cudaMemsetAsync(dW, 0, (size_t)d_out * d_in * esize, stream) != cudaSuccess)
            return BITLINEAR_ERR_CUDA;
        return BITLINEAR_OK;
    }
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int kb_total = (int)(d_in / 256);
    auto grid_for = [](int64_t items) {
        int64_t b = (items + kBwThreads - 1) / kBwThreads;
        return (unsigned)(b > 148 * 16 ? 148 * 16 : b);
    };
    if (want_dx) {
        uint16_t *wt = reinterpret_cast<uint16_t *>(ws + lay.wt);
        expand_ternary_kernel<<<grid_for(d_out * d_in / 16), kBwThreads, 0, stream>>>(
            packed, d_out, kb_total, wt);
        if (cudaGetLastError() != cudaSuccess) return BITLINEAR_ERR_CUDA;
        // dX[t][k] = gamma sum_o dY[t][o] W~[o][k]: A = W~ read MN-major (M = d_in).
        st = launch_dense_gemm_mn(wt, true, dY, false, d_in, T, d_out, dX, out_dtype, gamma,
                                  stream);
        if (st != BITLINEAR_OK) return st;
    }
    if (want_dw) {
        uint16_t *xh = reinterpret_cast<uint16_t *>(ws + lay.xh);
        dequant_kernel<<<grid_for(T * d_in / 16), kBwThreads, 0, stream>>>(Xq, beta, T, (int)d_in,
                                                                           xh);
        if (cudaGetLastError() != cudaSuccess) return BITLINEAR_ERR_CUDA;
        // dW[o][k] = gamma sum_t dY[t][o] X^[t][k]: both read MN-major (M = d_in, N = d_out).
        st = launch_dense_gemm_mn(xh, true, dY, true, d_in, d_out, T, dW, out_dtype, gamma,
                                  stream);
        if (st != BITLINEAR_OK) return st;
    }
    return BITLINEAR_OK;
}
