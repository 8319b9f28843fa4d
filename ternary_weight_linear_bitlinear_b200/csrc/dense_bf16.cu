// dense_bf16.cu -- the dense bf16 linear layer Y = X W^T that BitLinear
// replaces, as context for the measurements: "BitNet b1.58: Mathematical
// Foundations of 1.58-Bit Ternary Quantization, Absmean Scaling, and
// Multiplication-Free LLM Architectures", section 2, "The Linear
// Transformation and Rescaling" (the full-precision product the ternary one
// stands in for) and section 4, "Memory Bandwidth and Latency Bounds" (a
// decode step costs the weight bytes over the memory bandwidth: 2 bytes per
// weight here against 0.25 for the packed ternary codes).
//
// Two hand-written kernels, no library GEMM:
//   * dense_gemv_kernel (T <= 16): every warp streams two weight rows with
//     16-byte loads that bypass L1, multiplies them with the activations
//     (read through the read-only path, shared by all warps) in fp32, and
//     reduces across the warp with shuffles;
//   * dense_gemm_kernel (T > 16): a persistent tcgen05 kind::f16 GEMM.  One
//     CTA per SM walks 128 x 256 output tiles; warp 0 TMA-loads 64-column
//     stages of W (A operand, 128 rows) and X (B operand, 256 tokens), both
//     128-byte swizzled, K-major -- or, for the backward pass's GEMMs,
//     either operand MN-major (stored with the reduction index as the row,
//     loaded as 64-element panels, no transpose pass); warp 1 issues four
//     MMAs per stage into one
//     of two TMEM fp32 accumulators (2 x 256 columns); warps 2..5 read a
//     finished accumulator, round it and write it with TMA tensor stores
//     while the next tile accumulates.  Every mbarrier wait is bounded.
#include <cstdint>
#include <type_traits>

#include <cuda.h>
#include <cuda_bf16.h>

#include "bitlinear.h"
#include "common.cuh"
#include "tc_common.cuh"

namespace bl {

// ------------------------------------------------------------------ GEMV ---

constexpr int kDgThreads = 256;
constexpr int kDgRows = 2;   // weight rows per warp

__device__ __forceinline__ uint4 ld_stream_u4(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float dot8_bf16(const uint4 &w, const uint4 &x, float acc) {
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w}, xv[4] = {x.x, x.y, x.z, x.w};
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc = fmaf(__uint_as_float(wv[i] << 16), __uint_as_float(xv[i] << 16), acc);
        acc = fmaf(__uint_as_float(wv[i] & 0xffff0000u), __uint_as_float(xv[i] & 0xffff0000u), acc);
    }
    return acc;
}

template <int TT, bool OUT_BF16>
__global__ void __launch_bounds__(kDgThreads)
dense_gemv_kernel(const uint4 *__restrict__ W, const uint4 *__restrict__ X, int d_out, int kv,
                  int T, void *__restrict__ Y, const float *__restrict__ alpha) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = (blockIdx.x * (kDgThreads / 32) + warp) * kDgRows;
    if (row0 >= d_out) return;   // whole warp
    float acc[kDgRows][TT];
    #pragma unroll
    for (int r = 0; r < kDgRows; ++r)
        #pragma unroll
        for (int t = 0; t < TT; ++t) acc[r][t] = 0.0f;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    #pragma unroll 4
    for (int c = lane; c < kv; c += 32) {
        uint4 w[kDgRows];
        #pragma unroll
        for (int r = 0; r < kDgRows; ++r)
            w[r] = row0 + r < d_out ? ld_stream_u4(W + (size_t)(row0 + r) * kv + c) : zero;
        #pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t < T) {
                const uint4 x = __ldg(X + (size_t)t * kv + c);
                #pragma unroll
                for (int r = 0; r < kDgRows; ++r) acc[r][t] = dot8_bf16(w[r], x, acc[r][t]);
            }
        }
    }
    #pragma unroll
    for (int r = 0; r < kDgRows; ++r)
        #pragma unroll
        for (int t = 0; t < TT; ++t) {
            float v = acc[r][t];
            #pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[r][t] = v;
        }
    if (lane == 0) {
        const float a = alpha ? *alpha : 1.0f;
        #pragma unroll
        for (int r = 0; r < kDgRows; ++r)
            #pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < T && row0 + r < d_out) {
                    const size_t yi = (size_t)t * d_out + row0 + r;
                    const float y = alpha ? __fmul_rn(acc[r][t], a) : acc[r][t];
                    if (OUT_BF16)
                        reinterpret_cast<__nv_bfloat16 *>(Y)[yi] = __float2bfloat16_rn(y);
                    else
                        reinterpret_cast<float *>(Y)[yi] = y;
                }
            }
    }
}

// ------------------------------------------------------------------ GEMM ---

constexpr int kDM = 128;                      // weight rows per tile (MMA M)
constexpr int kDN = 256;                      // tokens per tile (MMA N)
constexpr int kDKE = 64;                      // bf16 columns per stage (128 bytes)
constexpr int kDStages = 4;
constexpr int kDATile = kDM * 128;            // 16 KiB
constexpr int kDBTile = kDN * 128;            // 32 KiB
constexpr int kDStageBytes = kDATile + kDBTile;
constexpr int kDAccCols = kDN;                // fp32 columns of one accumulator
constexpr int kDAccBufs = 2;
constexpr int kDTmemCols = 512;
constexpr int kDEpiWarps = 4;
constexpr int kDChunk = 32;                   // tokens per output block
constexpr int kDOutBufBytes = kDChunk * 32 * 4;
constexpr int kDOutBytes = kDEpiWarps * 2 * kDOutBufBytes;
constexpr int kDFirstEpiWarp = 2;
constexpr int kDThreads = 32 * (kDFirstEpiWarp + kDEpiWarps);
static_assert(kDAccBufs * kDAccCols <= kDTmemCols, "tensor memory budget");
static_assert(kDStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");

struct __align__(8) DenseBarriers {
    uint64_t full[kDStages];
    uint64_t empty[kDStages];
    uint64_t acc_full[kDAccBufs];
    uint64_t acc_empty[kDAccBufs];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
constexpr int kDSmemBytes = kDStages * kDStageBytes + kDOutBytes + 1024 + 1024;
constexpr int kDPanel = 64;                   // MN-elements of one MN-major panel (128 bytes)
constexpr int kDPanelBytes = kDPanel * 128;   // 64 K-rows of 128 bytes per stage and panel

// D[m][n] = sum_k A[m][k] B[n][k] (A: M = d_out rows, B: N = T rows, K = d_in),
// stored as Y[n][m].  A_MN / B_MN: the operand is stored MN-major, i.e. as
// [k][m] / [k][n] in memory, loaded as 64-element panels (no transpose pass).
template <bool OUT_BF16, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kDThreads, 1)
dense_gemm_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                  const __grid_constant__ CUtensorMap map_y, int d_out, int d_in, int T,
                  const float *__restrict__ alpha, DeviceCtx ctx) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *out_stage = smem + kDStages * kDStageBytes;
    DenseBarriers *bars = reinterpret_cast<DenseBarriers *>(out_stage + kDOutBytes);
    const uint32_t smem_base = smem_u32(smem);
    auto stage_a = [&](int s) { return smem_base + s * kDStageBytes; };
    auto stage_b = [&](int s) { return smem_base + s * kDStageBytes + kDATile; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tiles = (d_out + kDM - 1) / kDM;
    const int num_tiles = m_tiles * ((T + kDN - 1) / kDN);
    const int num_k = (d_in + kDKE - 1) / kDKE;   // MN-major K edges are zero-filled by the copy
    volatile int *abort_flag = &bars->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDStages; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        for (int b = 0; b < kDAccBufs; ++b) {
            mbar_init(smem_u32(&bars->acc_full[b]), 1);
            mbar_init(smem_u32(&bars->acc_empty[b]), kDEpiWarps);
        }
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort_flag = 0;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_y)) : "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&bars->tmem_base), kDTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ---
        if (lane == 0) {
            int s = 0, step = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile % m_tiles) * kDM, n0 = (tile / m_tiles) * kDN;
                for (int kt = 0; kt < num_k; ++kt) {
                    if (step >= kDStages &&
                        !wait_or_abort(smem_u32(&bars->empty[s]), ph ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&bars->full[s]);
                    mbar_arrive_expect_tx(fb, kDStageBytes);
                    if constexpr (A_MN) {
                        #pragma unroll
                        for (int p = 0; p < kDM / kDPanel; ++p)
                            tma_load_2d(stage_a(s) + p * kDPanelBytes, &map_w, m0 + p * kDPanel,
                                        kt * kDKE, fb);
                    } else {
                        tma_load_2d(stage_a(s), &map_w, kt * kDKE, m0, fb);
                    }
                    if constexpr (B_MN) {
                        #pragma unroll
                        for (int p = 0; p < kDN / kDPanel; ++p)
                            tma_load_2d(stage_b(s) + p * kDPanelBytes, &map_x, n0 + p * kDPanel,
                                        kt * kDKE, fb);
                    } else {
                        tma_load_2d(stage_b(s), &map_x, kt * kDKE, n0, fb);
                    }
                    ++step;
                    if (++s == kDStages) { s = 0; ph ^= 1u; }
                }
            }
            // Drain: every copy issued must land before the CTA may exit.
            for (int q = step > kDStages ? step - kDStages : 0; q < step; ++q)
                mbar_wait_bounded(smem_u32(&bars->full[q % kDStages]),
                                  (uint32_t)(q / kDStages) & 1u, ctx);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kDM, kDN, A_MN, B_MN);
            int s = 0, i = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++i) {
                const int buf = i & 1, use = i >> 1;
                if (use > 0 && !wait_or_abort(smem_u32(&bars->acc_empty[buf]),
                                              (uint32_t)(use - 1) & 1u, ctx, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t tmem_acc = tmem_base + buf * kDAccCols;
                for (int kt = 0; kt < num_k; ++kt) {
                    if (!wait_or_abort(smem_u32(&bars->full[s]), ph, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    #pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // K = 16 bf16 per MMA
                        // K-major: 32 bytes along each 128-byte row; MN-major:
                        // 16 K-rows of every panel (two 1024-byte atoms).
                        const uint64_t da =
                            A_MN ? smem_desc_sw128_mn(stage_a(s) + kk * 2048, kDPanelBytes)
                                 : smem_desc_sw128(stage_a(s) + kk * 32);
                        const uint64_t db =
                            B_MN ? smem_desc_sw128_mn(stage_b(s) + kk * 2048, kDPanelBytes)
                                 : smem_desc_sw128(stage_b(s) + kk * 32);
                        tc_mma_f16_ss(tmem_acc, da, db, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&bars->empty[s]));
                    if (++s == kDStages) { s = 0; ph ^= 1u; }
                }
                if (ok) tc_commit(smem_u32(&bars->acc_full[buf]));
            }
            tc_commit(smem_u32(&bars->drain));
            mbar_wait_bounded(smem_u32(&bars->drain), 0, ctx);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue ---
        const int quarter = warp & 3;
        const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
        uint8_t *my_out = out_stage + (warp - kDFirstEpiWarp) * 2 * kDOutBufBytes;
        const float a = alpha ? *alpha : 1.0f;
        int ob = 0, i = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
            const int m0 = (tile % m_tiles) * kDM, n0 = (tile / m_tiles) * kDN;
            const int buf = i & 1, use = i >> 1;
            const bool ok = wait_or_abort(smem_u32(&bars->acc_full[buf]), (uint32_t)use & 1u, ctx,
                                          abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int r0 = m0 + quarter * 32;
            #pragma unroll 1
            for (int c = 0; c < kDN / kDChunk; ++c) {
                const int t0 = n0 + c * kDChunk;
                if (t0 >= T || r0 >= d_out) break;   // uniform: nothing of this block exists
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_field + buf * kDAccCols + c * kDChunk, v);
                tmem_wait_ld();
                if (lane == 0) bulk_wait_read_1();
                __syncwarp();
                uint8_t *stg = my_out + ob * kDOutBufBytes;
                #pragma unroll
                for (int j = 0; j < kDChunk; ++j) {
                    const float y = alpha ? __fmul_rn(__uint_as_float(v[j]), a)
                                          : __uint_as_float(v[j]);
                    if (OUT_BF16)
                        reinterpret_cast<__nv_bfloat16 *>(stg)[j * 32 + lane] = __float2bfloat16_rn(y);
                    else
                        reinterpret_cast<float *>(stg)[j * 32 + lane] = y;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&map_y, smem_u32(stg), r0, t0);
                    bulk_commit_group();
                }
                ob ^= 1;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty[buf]));
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kDTmemCols);
    }
}

// ------------------------------------------------------------------ host ---

template <int TT>
static cudaError_t launch_dense_gemv_t(const uint16_t *W, int64_t d_out, int64_t d_in,
                                       const uint16_t *X, int64_t T, void *Y, bool bf,
                                       const float *alpha, cudaStream_t stream) {
    const int rows_per_cta = (kDgThreads / 32) * kDgRows;
    const unsigned grid = (unsigned)((d_out + rows_per_cta - 1) / rows_per_cta);
    auto kern = bf ? dense_gemv_kernel<TT, true> : dense_gemv_kernel<TT, false>;
    kern<<<grid, kDgThreads, 0, stream>>>(reinterpret_cast<const uint4 *>(W),
                                          reinterpret_cast<const uint4 *>(X), (int)d_out,
                                          (int)(d_in / 8), (int)T, Y, alpha);
    return cudaGetLastError();
}

// A: [d_out][d_in] (K-major) or [d_in][d_out] (a_mn); B: [T][d_in] or
// [d_in][T] (b_mn).  Y[T][d_out].
static bitlinear_status launch_dense_gemm(const uint16_t *W, int64_t d_out, int64_t d_in,
                                          const uint16_t *X, int64_t T, void *Y, bool bf,
                                          const float *alpha, cudaStream_t stream,
                                          bool a_mn = false, bool b_mn = false) {
    PFN_encodeTiled encode = get_encode_fn();
    if (!encode) return BITLINEAR_ERR_CUDA;
    DeviceCtx ctx;
    bitlinear_status st = get_ctx(&ctx);
    if (st != BITLINEAR_OK) return st;
    CUtensorMap map_w, map_x, map_y;
    const cuuint32_t estr[2] = {1, 1};
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(a_mn ? d_out : d_in), (cuuint64_t)(a_mn ? d_in : d_out)};
        const cuuint64_t strides[1] = {(cuuint64_t)(a_mn ? d_out : d_in) * 2};
        const cuuint32_t box[2] = {a_mn ? (cuuint32_t)kDPanel : (cuuint32_t)kDKE,
                                   a_mn ? (cuuint32_t)kDKE : (cuuint32_t)kDM};
        if (encode(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(W), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(b_mn ? T : d_in), (cuuint64_t)(b_mn ? d_in : T)};
        const cuuint64_t strides[1] = {(cuuint64_t)(b_mn ? T : d_in) * 2};
        const cuuint32_t box[2] = {b_mn ? (cuuint32_t)kDPanel : (cuuint32_t)kDKE,
                                   b_mn ? (cuuint32_t)kDKE : (cuuint32_t)kDN};
        if (encode(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(X), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    {
        const cuuint64_t esize = bf ? 2 : 4;
        const cuuint64_t dims[2] = {(cuuint64_t)d_out, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)d_out * esize};
        const cuuint32_t box[2] = {32, kDChunk};
        if (encode(&map_y, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   2, Y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    auto pick = [&](auto bf_tag) {
        constexpr bool B = decltype(bf_tag)::value;
        if (a_mn && b_mn) return dense_gemm_kernel<B, true, true>;
        if (a_mn) return dense_gemm_kernel<B, true, false>;
        if (b_mn) return dense_gemm_kernel<B, false, true>;
        return dense_gemm_kernel<B, false, false>;
    };
    auto kern = bf ? pick(std::true_type{}) : pick(std::false_type{});
    if (ensure_dynamic_smem((const void *)kern, kDSmemBytes) != cudaSuccess)
        return BITLINEAR_ERR_CUDA;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles = ((d_out + kDM - 1) / kDM) * ((T + kDN - 1) / kDN);
    const int grid = (int)(tiles < sms ? tiles : sms);
    kern<<<grid, kDThreads, kDSmemBytes, stream>>>(map_w, map_x, map_y, (int)d_out, (int)d_in,
                                                   (int)T, alpha, ctx);
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

// The tcgen05 GEMM with MN-major operands (see launch_dense_gemm): used by the
// backward pass so that dY, X^ and W~ are read in their natural layouts.
bitlinear_status launch_dense_gemm_mn(const uint16_t *A, bool a_mn, const uint16_t *B, bool b_mn,
                                      int64_t M, int64_t N, int64_t K, void *Y, int out_dtype,
                                      const float *alpha, cudaStream_t stream) {
    return launch_dense_gemm(A, M, K, B, N, Y, out_dtype == BITLINEAR_OUT_BF16, alpha, stream,
                             a_mn, b_mn);
}

// alpha: optional device scalar multiplying every output (in fp32, once).
bitlinear_status launch_dense_bf16(const uint16_t *W, int64_t d_out, int64_t d_in,
                                   const uint16_t *X, int64_t T, void *Y, int out_dtype,
                                   const float *alpha, cudaStream_t stream) {
    const bool bf = out_dtype == BITLINEAR_OUT_BF16;
    if (T > 16) return launch_dense_gemm(W, d_out, d_in, X, T, Y, bf, alpha, stream);
    cudaError_t e;
    if (T <= 1) e = launch_dense_gemv_t<1>(W, d_out, d_in, X, T, Y, bf, alpha, stream);
    else if (T <= 2) e = launch_dense_gemv_t<2>(W, d_out, d_in, X, T, Y, bf, alpha, stream);
    else if (T <= 4) e = launch_dense_gemv_t<4>(W, d_out, d_in, X, T, Y, bf, alpha, stream);
    else if (T <= 8) e = launch_dense_gemv_t<8>(W, d_out, d_in, X, T, Y, bf, alpha, stream);
    else e = launch_dense_gemv_t<16>(W, d_out, d_in, X, T, Y, bf, alpha, stream);
    return e == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

}  // namespace bl
