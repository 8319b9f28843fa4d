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
// dense_bf16.cu with gamma applied in its fp32 epilogue.  Three
// memory-bound kernels put the operands in the K-major form it reads:
//   * expand_ternary_t_kernel: the packed codes -> W~^T as bf16 {-1, 0, 1}
//     (exact), [d_in][d_out];
//   * dequant_t_kernel: X~ and beta -> X^^T as bf16 of fl32(q fl32(beta/127)),
//     [d_in][Tp], zero for the padded tokens t >= T;
//   * transpose_bf16_kernel: dY -> dY^T, [d_out][Tp], zero-padded likewise;
// Tp = T rounded up to 256 (the GEMM's reduction granule).
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {

bitlinear_status launch_dense_bf16(const uint16_t *W, int64_t d_out, int64_t d_in,
                                   const uint16_t *X, int64_t T, void *Y, int out_dtype,
                                   const float *alpha, cudaStream_t stream);

constexpr int kTrThreads = 256;
constexpr int kTrTile = 64;          // 64 x 64 element tiles
constexpr int kTrPad = 8;            // row padding of the shared tile (elements)

// W~^T: one CTA per 64 weight rows (four 16-row tiles) x one 256-column
// k-block.  Thread i decodes row i mod 64's words kw = i / 64 (+ 4, 8, 12):
// word kw holds columns 16 kw + 4 s + b in bits 8 b + 2 s as W~ + 1.
__global__ void __launch_bounds__(kTrThreads)
expand_ternary_t_kernel(const uint32_t *__restrict__ packed, int d_out, int kb_total,
                        uint16_t *__restrict__ wt) {
    __shared__ __align__(16) uint16_t tile[256][kTrTile + kTrPad];   // [column][row]
    const int kb = blockIdx.y;
    const int row0 = blockIdx.x * kTrTile;
    const int row = threadIdx.x % kTrTile, kwq = threadIdx.x / kTrTile;
    const int o = row0 + row;
    const uint32_t *tile_words = packed + ((size_t)(o >> 4) * kb_total + kb) * 256 + (o & 15) * 16;
    const uint16_t lut[3] = {0xBF80u, 0x0000u, 0x3F80u};   // bf16 of -1, 0, +1
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int kw = kwq + 4 * i;
        const uint32_t w = __ldg(tile_words + kw);
        #pragma unroll
        for (int s = 0; s < 4; ++s)
            #pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t c = (w >> (8 * b + 2 * s)) & 3u;
                tile[16 * kw + 4 * s + b][row] = c < 3 ? lut[c] : (uint16_t)0x7FC0u;
            }
    }
    __syncthreads();
    // Each output row k holds 64 consecutive weight rows: 128 bytes.
    #pragma unroll
    for (int p = 0; p < 256 * kTrTile * 2 / (16 * kTrThreads); ++p) {
        const int idx = p * kTrThreads + threadIdx.x;
        const int col = idx >> 3, chunk = idx & 7;
        const uint4 v = *reinterpret_cast<const uint4 *>(&tile[col][chunk * 8]);
        *reinterpret_cast<uint4 *>(wt + (size_t)(kb * 256 + col) * d_out + row0 + chunk * 8) = v;
    }
}

// X^^T: one CTA per 64 tokens x 64 columns.
__global__ void __launch_bounds__(kTrThreads)
dequant_t_kernel(const int8_t *__restrict__ xq, const float *__restrict__ beta, int T, int K,
                 int Tp, uint16_t *__restrict__ xt) {
    __shared__ __align__(16) uint16_t tile[kTrTile][kTrTile + kTrPad];   // [k][t]
    const int t0 = blockIdx.y * kTrTile, k0 = blockIdx.x * kTrTile;
    const int tl = threadIdx.x / 4, kc = (threadIdx.x % 4) * 16;
    const int t = t0 + tl;
    uint4 q = make_uint4(0, 0, 0, 0);
    float sc = 0.0f;
    if (t < T) {
        q = __ldg(reinterpret_cast<const uint4 *>(xq + (size_t)t * K + k0 + kc));
        sc = __fdiv_rn(beta[t], 127.0f);
    }
    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
    #pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int code = (int)(int8_t)((qw[j >> 2] >> (8 * (j & 3))) & 0xFFu);
        const float v = __fmul_rn((float)code, sc);
        tile[kc + j][tl] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
    __syncthreads();
    #pragma unroll
    for (int p = 0; p < kTrTile * kTrTile * 2 / (16 * kTrThreads); ++p) {
        const int idx = p * kTrThreads + threadIdx.x;
        const int k = idx >> 3, chunk = idx & 7;
        const uint4 v = *reinterpret_cast<const uint4 *>(&tile[k][chunk * 8]);
        *reinterpret_cast<uint4 *>(xt + (size_t)(k0 + k) * Tp + t0 + chunk * 8) = v;
    }
}

// dY^T: one CTA per 64 tokens x 64 outputs.
__global__ void __launch_bounds__(kTrThreads)
transpose_bf16_kernel(const uint16_t *__restrict__ dy, int T, int N, int Tp,
                      uint16_t *__restrict__ dyt) {
    __shared__ __align__(16) uint16_t tile[kTrTile][kTrTile + kTrPad];   // [n][t]
    const int t0 = blockIdx.y * kTrTile, n0 = blockIdx.x * kTrTile;
    const int tl = threadIdx.x / 8, nc = (threadIdx.x % 8) * 8;
    #pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int tt = tl + 32 * h, t = t0 + tt;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < T) v = __ldg(reinterpret_cast<const uint4 *>(dy + (size_t)t * N + n0 + nc));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        #pragma unroll
        for (int j = 0; j < 8; ++j) tile[nc + j][tt] = (uint16_t)(w[j >> 1] >> (16 * (j & 1)));
    }
    __syncthreads();
    #pragma unroll
    for (int p = 0; p < kTrTile * kTrTile * 2 / (16 * kTrThreads); ++p) {
        const int idx = p * kTrThreads + threadIdx.x;
        const int n = idx >> 3, chunk = idx & 7;
        const uint4 v = *reinterpret_cast<const uint4 *>(&tile[n][chunk * 8]);
        *reinterpret_cast<uint4 *>(dyt + (size_t)(n0 + n) * Tp + t0 + chunk * 8) = v;
    }
}

static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

struct BackwardLayout {
    size_t wt, xt, dyt, total;   // byte offsets of the three operands, total bytes
    int64_t tp;
};

static BackwardLayout backward_layout(int64_t d_out, int64_t d_in, int64_t T, bool want_dx,
                                      bool want_dw) {
    BackwardLayout l = {};
    l.tp = round_up(T > 0 ? T : 1, 256);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) / 256 * 256;
        return at;
    };
    l.wt = want_dx ? take((size_t)d_in * d_out * 2) : 0;
    l.xt = want_dw ? take((size_t)d_in * l.tp * 2) : 0;
    l.dyt = want_dw ? take((size_t)d_out * l.tp * 2) : 0;
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
    if (want_dx) {
        uint16_t *wt = reinterpret_cast<uint16_t *>(ws + lay.wt);
        expand_ternary_t_kernel<<<dim3((unsigned)(d_out / kTrTile), (unsigned)kb_total), kTrThreads,
                                  0, stream>>>(packed, (int)d_out, kb_total, wt);
        if (cudaGetLastError() != cudaSuccess) return BITLINEAR_ERR_CUDA;
        // dX[t][k] = gamma sum_o dY[t][o] W~^T[k][o]
        st = launch_dense_bf16(wt, d_in, d_out, dY, T, dX, out_dtype, gamma, stream);
        if (st != BITLINEAR_OK) return st;
    }
    if (want_dw) {
        uint16_t *xt = reinterpret_cast<uint16_t *>(ws + lay.xt);
        uint16_t *dyt = reinterpret_cast<uint16_t *>(ws + lay.dyt);
        const unsigned tb = (unsigned)(lay.tp / kTrTile);
        dequant_t_kernel<<<dim3((unsigned)(d_in / kTrTile), tb), kTrThreads, 0, stream>>>(
            Xq, beta, (int)T, (int)d_in, (int)lay.tp, xt);
        transpose_bf16_kernel<<<dim3((unsigned)(d_out / kTrTile), tb), kTrThreads, 0, stream>>>(
            dY, (int)T, (int)d_out, (int)lay.tp, dyt);
        if (cudaGetLastError() != cudaSuccess) return BITLINEAR_ERR_CUDA;
        // dW[o][k] = gamma sum_t dY^T[o][t] X^^T[k][t]
        st = launch_dense_bf16(xt, d_in, lay.tp, dyt, d_out, dW, out_dtype, gamma, stream);
        if (st != BITLINEAR_OK) return st;
    }
    return BITLINEAR_OK;
}
