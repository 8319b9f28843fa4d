// gemv.cu -- decode-time ternary x int8 product for 1..16 tokens.
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 2,
// "The Linear Transformation and Rescaling" (Y = (X~ W~^T) beta gamma /
// (Q_b - 1), int32 accumulation), and section 4, "Memory Bandwidth and
// Latency Bounds" (a decode step costs the weight bytes over the memory
// bandwidth).  Section 6 unpacks 2-bit codes into masks for a SIMD add;
// here the unpacking feeds the int8 tensor-core MMA instead, which does the
// same additions with far fewer issued instructions.
//
// Work decomposition: one CTA per 16-row tile of W~, its 8 warps splitting
// the 256-column tiles of that row band.  A warp streams one 1 KiB packed
// tile per step with two fully coalesced 16-byte loads per lane (lane l
// reads bytes 16l.. of rows 0..7 and of rows 8..15) and keeps `D` tiles in
// flight.  Lane (g = l/4, q = l%4) then holds words 4q..4q+3 of rows g and
// g+8, i.e. the A fragments of m16n8k32 MMAs under a permutation of the
// reduction index that the activation fragments follow too:
//   MMA (p, s), p in {0,1}, s in {0..3}:
//     a0/a2 = word 4q+2p / 4q+2p+1 of row g  masked to slot s,
//     a1/a3 = the same words of row g+8,
//     b0/b1 = activation bytes 64q+32p+4s.. and 64q+32p+16+4s.. of token g.
// Masking slot s without shifting leaves the codes scaled by 4^s (at most
// 2*64 = 128, a valid u8), so each slot has its own accumulator and the
// four are combined exactly as acc0 + acc1/4 + acc2/16 + acc3/64 at the end.
// Codes are c = W~ + 1; the epilogue subtracts the activation row sum.
#include <cstdint>

#include <cuda_bf16.h>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {

constexpr int kGemvWarps = 8;

__device__ __forceinline__ uint4 ld_stream_v4(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NT, int D, bool OUT_BF16>
__global__ void __launch_bounds__(kGemvWarps * 32)
gemv_kernel(const uint4 *__restrict__ packed, const float *__restrict__ gamma_ptr, int d_out,
            int kb_total, const int8_t *__restrict__ Xq, const float *__restrict__ beta,
            const int32_t *__restrict__ rowsum, int T, void *__restrict__ Y,
            int32_t *__restrict__ acc_out) {
    __shared__ int4 red[kGemvWarps][NT][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int rt = blockIdx.x;
    const int kb_begin = (kb_total * warp) / kGemvWarps;
    const int nblk = (kb_total * (warp + 1)) / kGemvWarps - kb_begin;
    const int d_in = kb_total * 256;

    // Tile (rt, kb) starts at uint4 index (rt * kb_total + kb) * 64.
    const uint4 *wsrc = packed + ((size_t)rt * kb_total + kb_begin) * 64 + lane;

    // The weights are not written by the kernel this one may overlap with,
    // so they stream in before the dependency wait.
    uint4 wa[D], wb[D];
    #pragma unroll
    for (int d = 0; d < D; ++d) {
        if (d < nblk) {
            wa[d] = ld_stream_v4(wsrc + d * 64);
            wb[d] = ld_stream_v4(wsrc + d * 64 + 32);
        }
    }

    pdl_wait_primary();

    int acc[NT][4][4];
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt)
        #pragma unroll
        for (int s = 0; s < 4; ++s)
            #pragma unroll
            for (int r = 0; r < 4; ++r) acc[nt][s][r] = 0;

    const uint4 *xsrc[NT];
    bool xvalid[NT];
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int t = nt * 8 + g;
        xvalid[nt] = t < T;
        xsrc[nt] = reinterpret_cast<const uint4 *>(Xq + (size_t)(xvalid[nt] ? t : 0) * d_in +
                                                   (size_t)kb_begin * 256 + 64 * q);
    }

    for (int i0 = 0; i0 < nblk; i0 += D) {
        #pragma unroll
        for (int d = 0; d < D; ++d) {
            const int i = i0 + d;
            if (i < nblk) {
                uint32_t xr[NT][16];
                #pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    #pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 x = xvalid[nt] ? __ldg(xsrc[nt] + i * 16 + v) : make_uint4(0, 0, 0, 0);
                        xr[nt][4 * v + 0] = x.x;
                        xr[nt][4 * v + 1] = x.y;
                        xr[nt][4 * v + 2] = x.z;
                        xr[nt][4 * v + 3] = x.w;
                    }
                }
                const uint32_t w0[4] = {wa[d].x, wa[d].y, wa[d].z, wa[d].w};
                const uint32_t w1[4] = {wb[d].x, wb[d].y, wb[d].z, wb[d].w};
                if (i + D < nblk) {
                    wa[d] = ld_stream_v4(wsrc + (i + D) * 64);
                    wb[d] = ld_stream_v4(wsrc + (i + D) * 64 + 32);
                }
                #pragma unroll
                for (int p = 0; p < 2; ++p) {
                    #pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        const uint32_t m = 0x03030303u << (2 * s);
                        const uint32_t a0 = w0[2 * p] & m, a2 = w0[2 * p + 1] & m;
                        const uint32_t a1 = w1[2 * p] & m, a3 = w1[2 * p + 1] & m;
                        #pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_u8s8(acc[nt][s], a0, a1, a2, a3, xr[nt][8 * p + s],
                                     xr[nt][8 * p + 4 + s]);
                    }
                }
            }
        }
    }

    #pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        int c[4];
        #pragma unroll
        for (int r = 0; r < 4; ++r)
            c[r] = acc[nt][0][r] + (acc[nt][1][r] >> 2) + (acc[nt][2][r] >> 4) +
                   (acc[nt][3][r] >> 6);
        red[warp][nt][lane] = make_int4(c[0], c[1], c[2], c[3]);
    }
    __syncthreads();

    // Epilogue: thread i -> (token t = i / 16, row r = i % 16), so a warp
    // stores two tokens' 16 consecutive outputs.
    const int i = threadIdx.x;
    const int t = i >> 4, r = i & 15;
    if (t < T) {
        const int gg = r & 7, half = r >> 3;
        const int nt = t >> 3, tt = t & 7;
        const int src_lane = gg * 4 + (tt >> 1);
        const int reg = (tt & 1) + 2 * half;
        int v = 0;
        #pragma unroll
        for (int w = 0; w < kGemvWarps; ++w) {
            const int *e = reinterpret_cast<const int *>(&red[w][nt][src_lane]);
            v += e[reg];
        }
        const int a = v - rowsum[t];
        const int o = rt * 16 + r;
        const size_t idx = (size_t)t * d_out + o;
        if (acc_out) acc_out[idx] = a;
        const float scale = __fdiv_rn(__fmul_rn(*gamma_ptr, beta[t]), 127.0f);
        const float y = __fmul_rn((float)a, scale);
        if (OUT_BF16)
            reinterpret_cast<__nv_bfloat16 *>(Y)[idx] = __float2bfloat16_rn(y);
        else
            reinterpret_cast<float *>(Y)[idx] = y;
    }
}

template <int NT, bool OUT_BF16>
static cudaError_t launch_gemv_t(const uint32_t *packed, const float *gamma, int d_out, int d_in,
                                 const int8_t *Xq, const float *beta, const int32_t *rowsum,
                                 int T, void *Y, int32_t *acc_out, bool pdl,
                                 cudaStream_t stream) {
    constexpr int D = 4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(d_out / 16));
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<NT, D, OUT_BF16>,
                              reinterpret_cast<const uint4 *>(packed), gamma, d_out, d_in / 256,
                              Xq, beta, rowsum, T, Y, acc_out);
}

bitlinear_status launch_gemv(const uint32_t *packed, const float *gamma, int64_t d_out,
                             int64_t d_in, const int8_t *Xq, const float *beta,
                             const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                             int32_t *acc_out, bool pdl, cudaStream_t stream) {
    cudaError_t e;
    const bool bf = out_dtype == BITLINEAR_OUT_BF16;
    if (T <= 8)
        e = bf ? launch_gemv_t<1, true>(packed, gamma, (int)d_out, (int)d_in, Xq, beta, rowsum,
                                        (int)T, Y, acc_out, pdl, stream)
               : launch_gemv_t<1, false>(packed, gamma, (int)d_out, (int)d_in, Xq, beta, rowsum,
                                         (int)T, Y, acc_out, pdl, stream);
    else
        e = bf ? launch_gemv_t<2, true>(packed, gamma, (int)d_out, (int)d_in, Xq, beta, rowsum,
                                        (int)T, Y, acc_out, pdl, stream)
               : launch_gemv_t<2, false>(packed, gamma, (int)d_out, (int)d_in, Xq, beta, rowsum,
                                         (int)T, Y, acc_out, pdl, stream);
    return e == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

}  // namespace bl
