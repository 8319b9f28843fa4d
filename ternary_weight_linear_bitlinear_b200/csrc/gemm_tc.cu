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
// with the weight codes as the A operand (M = 128 weight rows per tile) and
// the tokens as B (N = 128 tokens per tile).  The kernel is persistent: one
// CTA per SM walks the output tiles, and four roles run concurrently:
//   * warp 0 (one lane) TMA-loads, per 256-column step, the token tile
//     X~[n0..n0+128)[k..k+256) (two 128-byte swizzled, K-major halves) and
//     the eight whole 16x256 packed tiles of the 128 weight rows (8 KiB,
//     eight contiguous 1 KiB rows) into a ring of shared-memory stages,
//     signalling `full`;
//   * warps 2..5 (one thread per weight row = TMEM lane) expand their row's
//     sixteen packed words into 256 int8 codes and store them straight into
//     a tensor-memory A slot (tcgen05.st), where the MMA reads its A operand:
//     the expanded weights never touch shared memory.  They signal `afull`;
//   * warp 1 (one lane) issues eight tcgen05.mma.kind::i8 (K = 32 each) per
//     step into one of two TMEM accumulators and commits to `empty`, which
//     frees the shared-memory stage and the A slot; after a tile's last step
//     it commits to `acc_full`;
//   * warps 6..9 read a finished accumulator into registers (tcgen05.ld) and
//     hand it straight back (`acc_empty`), then subtract each token's code
//     sum, apply gamma beta / 127, stage 32x32 output blocks in shared memory
//     and write them with TMA tensor stores -- while the MMA already fills
//     the other accumulator with the next tile.
// Tensor memory: 2 x 128 accumulator columns + 4 A slots x 64 columns = 512.
// Waiting threads sleep in mbarrier.try_wait (with a suspend-time hint)
// instead of spinning, leaving issue slots to the producer and MMA lanes.
// Every mbarrier wait is bounded (see common.cuh); on expiry the CTA stops
// issuing, waits for its own copies, MMAs and stores in flight, frees its
// tensor memory and returns with the device error word set.
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {

constexpr int kBM = 128;          // weight rows per tile (MMA M = TMEM lanes)
constexpr int kBN = 128;          // tokens per tile (MMA N)
constexpr int kBK = 256;          // reduction columns per stage (one packed tile)
constexpr int kStages = 4;
constexpr int kBHalf = kBN * 128;            // 16 KiB: one 128-byte swizzle span of tokens
constexpr int kBTile = 2 * kBHalf;           // 32 KiB token tile
constexpr int kPTile = kBM * kBK / 4;        // 8 KiB packed tile
constexpr int kStageBytes = kBTile + kPTile; // 40 KiB (a multiple of 1024)
constexpr int kAccCols = kBN;                // int32 columns of one accumulator
constexpr int kAccBufs = 2;
constexpr int kACols = kBK / 4;              // TMEM columns of one A slot (4 codes each)
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 4;
constexpr int kChunk = 32;                   // tokens per output block
constexpr int kOutBufBytes = kChunk * 32 * 4;            // 32 tokens x 32 rows x fp32
constexpr int kOutBytes = kEpiWarps * 2 * kOutBufBytes;  // two blocks per epilogue warp
constexpr int kTokBytes = kEpiWarps * kBN * 8;           // per-warp {scale, code sum} table
constexpr int kFirstEpiWarp = 6;
constexpr int kGemmThreads = 32 * (kFirstEpiWarp + kEpiWarps);   // 10 warps
static_assert(kAccBufs * kAccCols + kStages * kACols <= kTmemCols, "tensor memory budget");
static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
static_assert(kBN % kChunk == 0, "whole output blocks per tile");

struct __align__(8) GemmBarriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t afull[kStages];
    uint64_t acc_full[kAccBufs];
    uint64_t acc_empty[kAccBufs];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(GemmBarriers) <= 1024, "barrier block");
constexpr int kSmemBytes = kStages * kStageBytes + kOutBytes + kTokBytes + 1024 /* barriers */ +
                           1024 /* alignment slack */;

// ----------------------------------------------------------------- PTX ---
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
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

// mbarrier.try_wait with a suspend-time hint: a thread whose phase is not
// complete sleeps (up to 1 ms) until it completes rather than spinning.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, const DeviceCtx &ctx,
                                              volatile int *abort_flag) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > ctx.wait_ns) {
            atomicOr(ctx.err, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
    }
}


// TMA tensor store of one box from shared memory, tracked by bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::
                     "l"(reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// At most one committed store group may still be reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Every committed store group has completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
               const __grid_constant__ CUtensorMap map_y, const float *__restrict__ gamma_ptr,
               int d_out, int d_in, const float *__restrict__ beta,
               const int32_t *__restrict__ rowsum, int T, int32_t *__restrict__ acc_out,
               DeviceCtx ctx) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *out_stage = smem + kStages * kStageBytes;
    uint8_t *tok_stage = out_stage + kOutBytes;
    GemmBarriers *bars = reinterpret_cast<GemmBarriers *>(tok_stage + kTokBytes);
    const uint32_t smem_base = smem_u32(smem);
    auto stage_x = [&](int s) { return smem_base + s * kStageBytes; };
    auto stage_w = [&](int s) { return smem_base + s * kStageBytes + kBTile; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tiles = (d_out + kBM - 1) / kBM;
    const int num_tiles = m_tiles * ((T + kBN - 1) / kBN);
    const int num_k = d_in / kBK;
    volatile int *abort_flag = &bars->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
            mbar_init(smem_u32(&bars->afull[s]), 4);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(smem_u32(&bars->acc_full[b]), 1);
            mbar_init(smem_u32(&bars->acc_empty[b]), kEpiWarps);
        }
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort_flag = 0;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_y)) : "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    const uint32_t tmem_a = tmem_base + kAccBufs * kAccCols;
    // Everything above overlaps the previous kernel under a programmatic
    // launch; the codes, scales and gamma are read only after this point.
    pdl_wait_primary();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ---
        if (lane == 0) {
            int s = 0, step = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile % m_tiles) * kBM, n0 = (tile / m_tiles) * kBN;
                for (int kt = 0; kt < num_k; ++kt) {
                    if (step >= kStages &&
                        !wait_or_abort(smem_u32(&bars->empty[s]), ph ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&bars->full[s]);
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    tma_load_2d(stage_x(s), &map_x, kt * kBK, n0, fb);
                    tma_load_2d(stage_x(s) + kBHalf, &map_x, kt * kBK + 128, n0, fb);
                    tma_load_3d(stage_w(s), &map_w, 0, kt, m0 / 16, fb);
                    ++step;
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                }
            }
            // Drain: every copy issued must land before the CTA may exit.
            for (int q = step > kStages ? step - kStages : 0; q < step; ++q)
                mbar_wait_bounded(smem_u32(&bars->full[q % kStages]),
                                  (uint32_t)(q / kStages) & 1u, ctx);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, kBN);
            int s = 0, i = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++i) {
                const int buf = i & 1, use = i >> 1;
                if (use > 0 && !wait_or_abort(smem_u32(&bars->acc_empty[buf]),
                                              (uint32_t)(use - 1) & 1u, ctx, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t tmem_acc = tmem_base + buf * kAccCols;
                for (int kt = 0; kt < num_k; ++kt) {
                    // `afull` completes only after every expander thread has seen
                    // `full` (the stage's copies landed) and written its A slot,
                    // so one wait orders both operands before the MMAs.
                    if (!wait_or_abort(smem_u32(&bars->afull[s]), ph, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    #pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk) {
                        const uint64_t bdesc =
                            smem_desc_sw128(stage_x(s) + (kk >> 2) * kBHalf + (kk & 3) * 32);
                        tc_mma_i8_ts(tmem_acc, tmem_a + s * kACols + kk * 8, bdesc, idesc,
                                     (kt > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&bars->empty[s]));
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                }
                if (ok) tc_commit(smem_u32(&bars->acc_full[buf]));
            }
            // Completion of everything issued above, before tensor memory is freed.
            tc_commit(smem_u32(&bars->drain));
            mbar_wait_bounded(smem_u32(&bars->drain), 0, ctx);
        }
        __syncwarp();
    } else if (warp < kFirstEpiWarp) {
        // ---------------------------------------------------- expander ---
        // Row m's sixteen words sit contiguously (64 bytes) in the stage; word
        // kw holds columns 16 kw .. 16 kw + 15, with column 16 kw + 4 s + j in
        // bits 8 j + 2 s, so (word >> 2 s) & 0x03030303 is the four codes of
        // columns 16 kw + 4 s + 0..3 -- exactly TMEM column 4 kw + s of the
        // K-major A operand (four int8 codes per 32-bit column).
        const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
        const int m = quarter * 32 + lane;      // weight row within the tile
        const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
        int s = 0, step = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int kt = 0; kt < num_k; ++kt) {
                ok = wait_or_abort(smem_u32(&bars->full[s]), ph, ctx, abort_flag);
                uint32_t w[16];
                if (ok) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        smem + s * kStageBytes + kBTile + m * 64);
                    #pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 v = src[q];
                        w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
                    }
                    // The A slot is free once the MMAs of its previous use completed.
                    if (step >= kStages)
                        ok = wait_or_abort(smem_u32(&bars->empty[s]), ph ^ 1u, ctx, abort_flag);
                }
                // The warp stays converged: tcgen05.st is a warp-wide instruction.
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                #pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t a[32];
                    #pragma unroll
                    for (int j = 0; j < 8; ++j)
                        #pragma unroll
                        for (int sl = 0; sl < 4; ++sl)
                            a[4 * j + sl] = (w[8 * h + j] >> (2 * sl)) & 0x03030303u;
                    tmem_st_32x32b_x32(tmem_a + lane_field + s * kACols + 32 * h, a);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->afull[s]));
                ++step;
                if (++s == kStages) { s = 0; ph ^= 1u; }
            }
        }
    } else {
        // ---------------------------------------------------- epilogue ---
        const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
        const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
        const int ep = warp - kFirstEpiWarp;
        uint8_t *my_out = out_stage + ep * 2 * kOutBufBytes;
        float2 *tok = reinterpret_cast<float2 *>(tok_stage + ep * kBN * 8);
        const float4 *tok4 = reinterpret_cast<const float4 *>(tok);
        const float gamma = *gamma_ptr;
        int ob = 0, i = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
            const int m0 = (tile % m_tiles) * kBM, n0 = (tile / m_tiles) * kBN;
            const int buf = i & 1, use = i >> 1;
            const bool ok = wait_or_abort(smem_u32(&bars->acc_full[buf]), (uint32_t)use & 1u, ctx,
                                          abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int r0 = m0 + quarter * 32;   // first output row of this warp
            const int o = r0 + lane;
            // Output blocks of 32 tokens that exist (warp-uniform).
            int nblk = r0 < d_out ? (T - n0 + kChunk - 1) / kChunk : 0;
            if (nblk > kBN / kChunk) nblk = kBN / kChunk;
            // The whole accumulator row of this lane, in four loads.
            uint32_t v[kBN / kChunk][kChunk];
            #pragma unroll
            for (int c = 0; c < kBN / kChunk; ++c)
                if (c < nblk)
                    tmem_ld_32x32b_x32(tmem_base + lane_field + buf * kAccCols + c * kChunk, v[c]);
            // Token table of this tile: lane j fills tokens j, j + 32, j + 64, j + 96
            // with {gamma beta / 127, code sum}; read back as broadcasts.
            __syncwarp();
            #pragma unroll
            for (int q = 0; q < kBN / 32; ++q) {
                const int t = n0 + q * 32 + lane;
                float sc = 0.0f;
                int rs = 0;
                if (t < T) {
                    sc = __fdiv_rn(__fmul_rn(gamma, beta[t]), 127.0f);
                    rs = rowsum[t];
                }
                tok[q * 32 + lane] = make_float2(sc, __int_as_float(rs));
            }
            tmem_wait_ld();
            // Accumulator now in registers: the MMA may refill it.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty[buf]));
            #pragma unroll
            for (int c = 0; c < kBN / kChunk; ++c) {
                if (c < nblk) {
                    const int t0 = n0 + c * kChunk;
                    // The block staged two blocks ago has been read by its store.
                    if (lane == 0) bulk_wait_read_1();
                    __syncwarp();
                    uint8_t *stg = my_out + ob * kOutBufBytes;
                    #pragma unroll
                    for (int j2 = 0; j2 < kChunk / 2; ++j2) {
                        const float4 tp = tok4[(c * kChunk) / 2 + j2];
                        #pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int j = 2 * j2 + h;
                            const float sc = h ? tp.z : tp.x;
                            const int rs = __float_as_int(h ? tp.w : tp.y);
                            const int a = (int)v[c][j] - rs;
                            const float y = __fmul_rn((float)a, sc);
                            if (OUT_BF16)
                                reinterpret_cast<__nv_bfloat16 *>(stg)[j * 32 + lane] =
                                    __float2bfloat16_rn(y);
                            else
                                reinterpret_cast<float *>(stg)[j * 32 + lane] = y;
                            if (acc_out && o < d_out && t0 + j < T)
                                acc_out[(size_t)(t0 + j) * d_out + o] = a;
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        // Rows past d_out and tokens past T are clipped by the copy.
                        tma_store_2d(&map_y, smem_u32(stg), r0, t0);
                        bulk_commit_group();
                    }
                    ob ^= 1;
                }
            }
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
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
    const bool bf = out_dtype == BITLINEAR_OUT_BF16;

    CUtensorMap map_x, map_w, map_y;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)d_in};
        const cuuint32_t box[2] = {128, kBN};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(Xq), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    {
        // Packed words as a 3-D array [row tile][k tile][256 words of one tile].
        const cuuint64_t kb = (cuuint64_t)(d_in / 256);
        const cuuint64_t dims[3] = {256, kb, (cuuint64_t)(d_out / 16)};
        const cuuint64_t strides[2] = {1024, kb * 1024};
        const cuuint32_t box[3] = {256, 1, kBM / 16};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (encode(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t *>(packed), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    {
        // Output [T][d_out], written in 32-row x 32-token boxes.
        const cuuint64_t esize = bf ? 2 : 4;
        const cuuint64_t dims[2] = {(cuuint64_t)d_out, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)d_out * esize};
        const cuuint32_t box[2] = {32, kChunk};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&map_y, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   2, Y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    auto kern = bf ? gemm_tc_kernel<true> : gemm_tc_kernel<false>;
    if (ensure_dynamic_smem((const void *)kern, kSmemBytes) != cudaSuccess)
        return BITLINEAR_ERR_CUDA;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles = ((d_out + kBM - 1) / kBM) * ((T + kBN - 1) / kBN);
    const int grid = (int)(tiles < sms ? tiles : sms);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, map_x, map_w, map_y, gamma, (int)d_out,
                                       (int)d_in, beta, rowsum, (int)T, acc_out, ctx);
    return e == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

}  // namespace bl
