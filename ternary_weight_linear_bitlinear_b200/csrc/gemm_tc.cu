// gemm_tc.cu -- prefill ternary x int8 product on the 5th-generation tensor
// cores (tcgen05, sm_100a).
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 2,
// "The Linear Transformation and Rescaling": Y = (X~ W~^T) beta gamma /
// (Q_b - 1) with int32 accumulation.  With hundreds of tokens the product is
// a dense contraction, so it runs as an int8 MMA:
//
//   D[o][t] = sum_k C[o][k] * X~[t][k]     (C = W~ + 1 in {0,1,2}, u8 x s8)
//
// with the weight codes as the A operand (M = 128 weight rows per CTA) and
// the tokens as B (N = kBN tokens per CTA).  Per 128-column step:
//   * warp 0 (one lane) TMA-loads the token tile X~[n0..n0+kBN)[k..k+128)
//     (128-byte swizzled, K-major) and the packed 2-bit tile of the 128
//     weight rows (4 KiB) into shared memory, signalling `full`;
//   * warps 2..5 (one thread per weight row = TMEM lane) expand their row's
//     eight packed words into 128 int8 codes and store them straight into
//     tensor memory (tcgen05.st), where the MMA reads its A operand: the
//     expanded weights never touch shared memory.  They signal `afull`;
//   * warp 1 (one lane) issues four tcgen05.mma.kind::i8 (K = 32 each) into
//     the TMEM accumulator and commits to `empty`, which frees both the
//     shared-memory stage and the TMEM A slot;
//   * after the last step warps 2..5 read the accumulator (tcgen05.ld),
//     subtract the token's code sum, apply gamma beta / 127 and store Y.
// Every mbarrier wait is bounded (see common.cuh); on expiry the CTA stops
// issuing, waits for its own copies and MMAs in flight, frees its tensor
// memory and returns with the device error word set.
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {

constexpr int kBM = 128;          // weight rows per CTA (MMA M)
constexpr int kBN = 256;          // tokens per CTA (MMA N)
constexpr int kBK = 128;          // reduction columns per stage (bytes)
constexpr int kStages = 5;
constexpr int kBTile = kBN * kBK;            // 32 KiB token tile
constexpr int kPTile = kBM * kBK / 4;        // 4 KiB packed tile
constexpr int kStageBytes = kBTile + kPTile;
constexpr int kAccCols = kBN;                // int32 accumulator columns
constexpr int kACols = kBK / 4;              // TMEM columns of one A slot (4 codes each)
constexpr int kTmemCols = 512;               // >= kAccCols + kStages * kACols
constexpr int kGemmThreads = 192;            // 6 warps
static_assert(kAccCols + kStages * kACols <= kTmemCols, "tensor memory budget");

struct __align__(8) GemmBarriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t afull[kStages];
    uint64_t acc_full;
    uint32_t tmem_base;
    int abort_flag;
};
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /* barriers etc. */ + 1024 /* align */;

// ----------------------------------------------------------------- PTX ---
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// D(tmem) (+)= A(tmem) * B(smem descriptor), kind::i8.
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

#define BL_R32(v)                                                                               \
    "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),     \
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),       \
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),     \
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),     \
        "r"(v[29]), "r"(v[30]), "r"(v[31])
#define BL_W32(v)                                                                               \
    "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),         \
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),              \
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),           \
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),           \
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),           \
        "=r"(v[31])

// Each thread of the warp writes 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        BL_R32(v)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : BL_W32(v)
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows
// of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), leading
// byte offset unused for this swizzle (1), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                 // leading byte offset (16 B units)
    d |= (uint64_t)(1024u >> 4) << 32;       // stride byte offset (16 B units)
    d |= (uint64_t)1u << 46;                 // version
    d |= (uint64_t)2u << 61;                 // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::i8: D s32, A u8, B s8, both K-major.
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n) {
    return (2u << 4)                       // D format s32
           | (0u << 7)                     // A unsigned 8-bit
           | (1u << 10)                    // B signed 8-bit
           | ((uint32_t)(n >> 3) << 17)    // N / 8
           | ((uint32_t)(m >> 4) << 24);   // M / 16
}

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, const DeviceCtx &ctx,
                                              volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > ctx.wait_ns) {
            atomicOr(ctx.err, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
    }
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
               const float *__restrict__ gamma_ptr, int d_out, int d_in,
               const float *__restrict__ beta, const int32_t *__restrict__ rowsum, int T,
               void *__restrict__ Y, int32_t *__restrict__ acc_out, DeviceCtx ctx) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ float s_scale[kBN];
    __shared__ int s_rowsum[kBN];

    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    GemmBarriers *bars = reinterpret_cast<GemmBarriers *>(smem + kStages * kStageBytes);
    const uint32_t smem_base = smem_u32(smem);
    auto stage_x = [&](int s) { return smem_base + s * kStageBytes; };
    auto stage_w = [&](int s) { return smem_base + s * kStageBytes + kBTile; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kBM;   // first weight row
    const int n0 = blockIdx.y * kBN;   // first token
    const int num_k = d_in / kBK;
    volatile int *abort_flag = &bars->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
            mbar_init(smem_u32(&bars->afull[s]), 4);
        }
        mbar_init(smem_u32(&bars->acc_full), 1);
        bars->abort_flag = 0;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    if (warp >= 2) {
        // Per-token scale gamma * beta / 127 and code sums of this token tile.
        const float gamma = *gamma_ptr;
        for (int j = threadIdx.x - 64; j < kBN; j += 128) {
            const int t = n0 + j;
            s_scale[j] = t < T ? __fdiv_rn(__fmul_rn(gamma, beta[t]), 127.0f) : 0.0f;
            s_rowsum[j] = t < T ? rowsum[t] : 0;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    const uint32_t tmem_acc = tmem_base;
    const uint32_t tmem_a = tmem_base + kAccCols;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ---
        if (lane == 0) {
            int issued = 0;
            for (int kt = 0; kt < num_k; ++kt) {
                const int s = kt % kStages;
                const uint32_t ph = (uint32_t)(kt / kStages) & 1u;
                if (kt >= kStages &&
                    !wait_or_abort(smem_u32(&bars->empty[s]), ph ^ 1u, ctx, abort_flag))
                    break;
                const uint32_t fb = smem_u32(&bars->full[s]);
                mbar_arrive_expect_tx(fb, kStageBytes);
                tma_load_2d(stage_x(s), &map_x, kt * kBK, n0, fb);
                tma_load_4d(stage_w(s), &map_w, (kt & 1) * 8, 0, kt >> 1, m0 / 16, fb);
                ++issued;
            }
            // Drain: every copy issued must land before the CTA may exit.
            for (int kt = issued > kStages ? issued - kStages : 0; kt < issued; ++kt)
                mbar_wait_bounded(smem_u32(&bars->full[kt % kStages]),
                                  (uint32_t)(kt / kStages) & 1u, ctx);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, kBN);
            for (int kt = 0; kt < num_k; ++kt) {
                const int s = kt % kStages;
                const uint32_t ph = (uint32_t)(kt / kStages) & 1u;
                if (!wait_or_abort(smem_u32(&bars->afull[s]), ph, ctx, abort_flag)) break;
                if (!wait_or_abort(smem_u32(&bars->full[s]), ph, ctx, abort_flag)) break;
                tc_fence_after();
                #pragma unroll
                for (int kk = 0; kk < kBK / 32; ++kk) {
                    const uint64_t bdesc = smem_desc_sw128(stage_x(s) + kk * 32);
                    tc_mma_i8_ts(tmem_acc, tmem_a + s * kACols + kk * 8, bdesc, idesc,
                                 (kt > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(smem_u32(&bars->empty[s]));
            }
            // Completion of everything issued above (also the drain).
            tc_commit(smem_u32(&bars->acc_full));
            mbar_wait_bounded(smem_u32(&bars->acc_full), 0, ctx);
        }
        __syncwarp();
    } else {
        // ---------------------------------- expander, then epilogue ---
        const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
        const int m = quarter * 32 + lane;      // weight row within the tile
        const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        for (int kt = 0; kt < num_k && ok; ++kt) {
            const int s = kt % kStages;
            const uint32_t ph = (uint32_t)(kt / kStages) & 1u;
            ok = wait_or_abort(smem_u32(&bars->full[s]), ph, ctx, abort_flag);
            uint32_t w[8];
            if (ok) {
                const uint4 *src = reinterpret_cast<const uint4 *>(smem + s * kStageBytes + kBTile +
                                                                  m * 32);
                const uint4 lo = src[0], hi = src[1];
                w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
                w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
                if (kt >= kStages)
                    ok = wait_or_abort(smem_u32(&bars->empty[s]), ph ^ 1u, ctx, abort_flag);
            }
            // The warp stays converged: tcgen05.st is a warp-wide instruction.
            if (__all_sync(0xffffffffu, ok)) {
                uint32_t a[32];
                #pragma unroll
                for (int j = 0; j < 8; ++j)
                    #pragma unroll
                    for (int sl = 0; sl < 4; ++sl) a[4 * j + sl] = (w[j] >> (2 * sl)) & 0x03030303u;
                tmem_st_32x32b_x32(tmem_a + lane_field + s * kACols, a);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->afull[s]));
            } else {
                ok = false;
            }
        }
        // Epilogue.
        if (__all_sync(0xffffffffu, ok) &&
            wait_or_abort(smem_u32(&bars->acc_full), 0, ctx, abort_flag)) {
            tc_fence_after();
        } else {
            ok = false;
        }
        if (__all_sync(0xffffffffu, ok)) {
            const int o = m0 + m;
            const bool row_ok = o < d_out;
            #pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                if (n0 + c * 32 >= T) break;    // uniform across the warp
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_acc + lane_field + c * 32, v);
                tmem_wait_ld();
                if (row_ok) {
                    #pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int tl = c * 32 + j;
                        const int t = n0 + tl;
                        if (t < T) {
                            const int a = (int)v[j] - s_rowsum[tl];
                            const size_t idx = (size_t)t * d_out + o;
                            if (acc_out) acc_out[idx] = a;
                            const float y = __fmul_rn((float)a, s_scale[tl]);
                            if (OUT_BF16)
                                reinterpret_cast<__nv_bfloat16 *>(Y)[idx] = __float2bfloat16_rn(y);
                            else
                                reinterpret_cast<float *>(Y)[idx] = y;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------ host ---

typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                    const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                    const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode_fn() {
    static PFN_encodeTiled fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(p);
    }
    return fn;
}

bitlinear_status launch_gemm_tc(const uint32_t *packed, const float *gamma, int64_t d_out,
                                int64_t d_in, const int8_t *Xq, const float *beta,
                                const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                int32_t *acc_out, cudaStream_t stream) {
    PFN_encodeTiled encode = get_encode_fn();
    if (!encode) return BITLINEAR_ERR_CUDA;
    DeviceCtx ctx;
    bitlinear_status st = get_ctx(&ctx);
    if (st != BITLINEAR_OK) return st;

    CUtensorMap map_x, map_w;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)d_in};
        const cuuint32_t box[2] = {kBK, kBN};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(Xq), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    {
        // Packed words as a 4-D array [row tile][k tile][row in tile][word].
        const cuuint64_t kb = (cuuint64_t)(d_in / 256);
        const cuuint64_t dims[4] = {16, 16, kb, (cuuint64_t)(d_out / 16)};
        const cuuint64_t strides[3] = {64, 1024, kb * 1024};
        const cuuint32_t box[4] = {8, 16, 1, kBM / 16};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        if (encode(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint32_t *>(packed), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    const bool bf = out_dtype == BITLINEAR_OUT_BF16;
    auto kern = bf ? gemm_tc_kernel<true> : gemm_tc_kernel<false>;
    static bool attr_set[2] = {false, false};
    if (!attr_set[bf]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
            cudaSuccess)
            return BITLINEAR_ERR_CUDA;
        attr_set[bf] = true;
    }
    dim3 grid((unsigned)((d_out + kBM - 1) / kBM), (unsigned)((T + kBN - 1) / kBN));
    kern<<<grid, kGemmThreads, kSmemBytes, stream>>>(map_x, map_w, gamma, (int)d_out, (int)d_in,
                                                     beta, rowsum, (int)T, Y, acc_out, ctx);
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

}  // namespace bl
