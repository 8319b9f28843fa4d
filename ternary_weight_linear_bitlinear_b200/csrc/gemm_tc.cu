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
// the tokens as B (N = 256 tokens per tile).  The kernel is persistent: one
// CTA per SM walks the output tiles, and four roles run concurrently, each
// 128-column step passing through two rings of shared memory:
//   * warp 0 (one lane) TMA-loads the token tile X~[n0..n0+256)[k..k+128)
//     (128-byte swizzled, K-major) into the token ring, signalling `full`,
//     and, five steps ahead, the packed 2-bit codes of the 128 weight rows
//     (4 KiB) into a separate packed ring, signalling `pfull`;
//   * warps 2..5 (one thread per weight row) read their row's eight packed
//     words from the packed ring, expand them into 128 int8 codes and store
//     those into the weight ring in the same 128-byte swizzled K-major
//     layout the TMA gives the tokens, then signal `afull` (and `pempty`);
//   * warp 1 (one lane) waits for both operands of a step, issues four
//     tcgen05.mma.kind::i8 (K = 32 each) with both operands read from shared
//     memory into one of two TMEM accumulators, and commits to `empty`
//     (token stage free) and `aempty` (weight slot free); after a tile's
//     last step it commits to `acc_full`;
//   * warps 6..9 read a finished accumulator (tcgen05.ld), subtract each
//     token's code sum, apply gamma beta / 127, stage 32-row x 8-token
//     blocks in shared memory and write them with TMA tensor stores, then
//     hand the accumulator back (`acc_empty`) -- while the MMA already fills
//     the other accumulator with the next tile.
// Each expanded weight code feeds 256 tokens of MMA work, so the expansion
// is a small share of the issue slots.  A step's critical loop is: MMA
// completion frees a token stage -> its next TMA (~1200 cycles under load)
// -> the MMA issue, which four token stages cover.  The expansion runs off
// that loop: its packed words arrive steps early in their own ring (the
// expanders never wait for a token stage), and three weight slots let it
// run ahead of the MMA.  (Loading the packed words with per-thread global
// loads instead was slower: the proxy fence each expander thread needs
// before signalling `afull` also waits for its loads in flight.)  Tensor
// memory holds only the two 256-column accumulators (512 columns).  Waiting
// threads sleep in mbarrier.try_wait.  Every wait is bounded (see common.cuh); on expiry the
// CTA stops issuing, waits for its own copies, MMAs and stores in flight,
// frees its tensor memory and returns with the device error word set.
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>

#include "bitlinear.h"
#include "common.cuh"
#include "tc_common.cuh"

namespace bl {

constexpr int kBM = 128;          // weight rows per tile (MMA M = TMEM lanes)
constexpr int kBN = 256;          // tokens per tile (MMA N)
constexpr int kBK = 128;          // reduction columns per step (bytes)
constexpr int kStages = 4;        // token ring
constexpr int kASlots = 3;        // weight ring
constexpr int kPSlots = 8;        // packed ring
constexpr int kPAhead = 5;        // steps the packed loads run ahead of the token loads
constexpr int kBTile = kBN * kBK;            // 32 KiB token tile
constexpr int kStageBytes = kBTile;          // a multiple of 1024
constexpr int kPTile = kBM * kBK / 4;        // 4 KiB packed codes of a step
constexpr int kATile = kBM * kBK;            // 16 KiB expanded weight codes
constexpr int kAccCols = kBN;                // int32 columns of one accumulator
constexpr int kAccBufs = 2;
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 4;
constexpr int kChunk = 8;                    // tokens per output block
constexpr int kOutBufBytes = kChunk * 32 * 4;            // 8 tokens x 32 rows x fp32
constexpr int kOutBytes = kEpiWarps * 2 * kOutBufBytes;  // two blocks per epilogue warp
constexpr int kTokBytes = kBN * 8;                       // {scale, code sum} of the tile's tokens
constexpr int kFirstEpiWarp = 6;
constexpr int kGemmThreads = 32 * (kFirstEpiWarp + kEpiWarps);   // 10 warps
static_assert(kAccBufs * kAccCols <= kTmemCols, "tensor memory budget");
static_assert(kStageBytes % 1024 == 0 && kATile % 1024 == 0,
              "ring entries keep the 1024-byte swizzle alignment");
static_assert(kBN % 32 == 0 && 32 % kChunk == 0, "whole output blocks per tile");

struct __align__(8) GemmBarriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t afull[kASlots];
    uint64_t aempty[kASlots];
    uint64_t pfull[kPSlots];
    uint64_t pempty[kPSlots];
    uint64_t acc_full[kAccBufs];
    uint64_t acc_empty[kAccBufs];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int epi_ok[4];      // per epilogue warp: its wait for the accumulator succeeded
};
static_assert(sizeof(GemmBarriers) <= 1024, "barrier block");
constexpr int kSmemBytes = kStages * kStageBytes + kASlots * kATile + kPSlots * kPTile +
                           kOutBytes + kTokBytes +
                           1024 /* barriers */ + 1024 /* alignment slack */;

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
    uint8_t *a_ring = smem + kStages * kStageBytes;
    uint8_t *p_ring = a_ring + kASlots * kATile;
    uint8_t *out_stage = p_ring + kPSlots * kPTile;
    uint8_t *tok_stage = out_stage + kOutBytes;
    GemmBarriers *bars = reinterpret_cast<GemmBarriers *>(tok_stage + kTokBytes);
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t a_base = smem_u32(a_ring);
    auto stage_x = [&](int s) { return smem_base + s * kStageBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tiles = (d_out + kBM - 1) / kBM;
    const int num_tiles = m_tiles * ((T + kBN - 1) / kBN);
    const int num_k = d_in / kBK;
    volatile int *abort_flag = &bars->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        for (int s = 0; s < kASlots; ++s) {
            mbar_init(smem_u32(&bars->afull[s]), 4);
            mbar_init(smem_u32(&bars->aempty[s]), 1);
        }
        for (int s = 0; s < kPSlots; ++s) {
            mbar_init(smem_u32(&bars->pfull[s]), 1);
            mbar_init(smem_u32(&bars->pempty[s]), 4);
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
    // Everything above overlaps the previous kernel under a programmatic
    // launch; the codes, scales and gamma are read only after this point.
    pdl_wait_primary();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ---
        // Steps are numbered over this CTA's tiles in order; step g is
        // (tile blockIdx.x + (g / num_k) gridDim.x, kt = g mod num_k).  The
        // packed codes of step g are issued with the tokens of g - kPAhead.
        if (lane == 0) {
            const int my_tiles = blockIdx.x < num_tiles
                                     ? (num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1
                                     : 0;
            const int total = my_tiles * num_k;
            auto issue_packed = [&](int g) {
                const int tile = (int)blockIdx.x + (g / num_k) * (int)gridDim.x;
                const int kt = g - (g / num_k) * num_k;
                const int m0 = (tile % m_tiles) * kBM;
                const uint32_t pb = smem_u32(&bars->pfull[g % kPSlots]);
                mbar_arrive_expect_tx(pb, kPTile);
                tma_load_4d(smem_u32(p_ring + (g % kPSlots) * kPTile), &map_w, (kt & 1) * 8, 0,
                            kt >> 1, m0 / 16, pb);
            };
            int p_issued = 0;
            for (; p_issued < kPAhead && p_issued < total; ++p_issued) issue_packed(p_issued);
            int s = 0, step = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int n0 = (tile / m_tiles) * kBN;
                for (int kt = 0; kt < num_k; ++kt) {
                    if (step >= kStages &&
                        !wait_or_abort(smem_u32(&bars->empty[s]), ph ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&bars->full[s]);
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    tma_load_2d(stage_x(s), &map_x, kt * kBK, n0, fb);
                    ++step;
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                    if (p_issued < total) {
                        // The packed slot was last used by step p_issued - kPSlots.
                        if (p_issued >= kPSlots &&
                            !wait_or_abort(smem_u32(&bars->pempty[p_issued % kPSlots]),
                                           (uint32_t)(p_issued / kPSlots - 1) & 1u, ctx,
                                           abort_flag)) {
                            ok = false;
                            break;
                        }
                        issue_packed(p_issued++);
                    }
                }
            }
            // Drain: every copy issued must land before the CTA may exit.
            for (int q = step > kStages ? step - kStages : 0; q < step; ++q)
                mbar_wait_bounded(smem_u32(&bars->full[q % kStages]),
                                  (uint32_t)(q / kStages) & 1u, ctx);
            for (int q = p_issued > kPSlots ? p_issued - kPSlots : 0; q < p_issued; ++q)
                mbar_wait_bounded(smem_u32(&bars->pfull[q % kPSlots]),
                                  (uint32_t)(q / kPSlots) & 1u, ctx);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, kBN);
            int s = 0, sa = 0, i = 0;
            uint32_t ph = 0, pha = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++i) {
                const int buf = i & 1, use = i >> 1;
                if (use > 0 && !wait_or_abort(smem_u32(&bars->acc_empty[buf]),
                                              (uint32_t)(use - 1) & 1u, ctx, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t tmem_acc = tmem_base + buf * kAccCols;
                for (int kt = 0; kt < num_k; ++kt) {
                    // Both operands of the step: the expanded weight codes and
                    // the token tile.
                    if (!wait_or_abort(smem_u32(&bars->afull[sa]), pha, ctx, abort_flag) ||
                        !wait_or_abort(smem_u32(&bars->full[s]), ph, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    #pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)
                        tc_mma_i8_ss(tmem_acc, smem_desc_sw128(a_base + sa * kATile + kk * 32),
                                     smem_desc_sw128(stage_x(s) + kk * 32), idesc,
                                     (kt > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(smem_u32(&bars->empty[s]));
                    tc_commit(smem_u32(&bars->aempty[sa]));
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                    if (++sa == kASlots) { sa = 0; pha ^= 1u; }
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
        // Row m's eight words of a step sit contiguously (32 bytes) in the
        // packed slot; word j holds columns 16 j .. 16 j + 15 of the step,
        // with column 16 j + 4 s + b in bits 8 b + 2 s, so (word >> 2 s) &
        // 0x03030303 is the four codes of columns 16 j + 4 s + 0..3: word j
        // expands to the 16-byte chunk j of the row, which the 128-byte
        // swizzle places at chunk j ^ (m mod 8) of the row's 128 bytes.
        const int m = (warp & 3) * 32 + lane;   // weight row within the tile
        uint8_t *arow = a_ring + m * kBK;
        int sa = 0, sp = 0, step = 0;
        uint32_t pha = 0, php = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int kt = 0; kt < num_k; ++kt) {
                ok = wait_or_abort(smem_u32(&bars->pfull[sp]), php, ctx, abort_flag);
                uint32_t w[8];
                if (ok) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(p_ring + sp * kPTile + m * 32);
                    const uint4 lo = src[0], hi = src[1];
                    w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
                    w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
                    // The weight slot is free once the MMAs of its previous use completed.
                    if (step >= kASlots)
                        ok = wait_or_abort(smem_u32(&bars->aempty[sa]), pha ^ 1u, ctx, abort_flag);
                }
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                uint8_t *dst = arow + sa * kATile;
                #pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 c = make_uint4(w[j] & 0x03030303u, (w[j] >> 2) & 0x03030303u,
                                               (w[j] >> 4) & 0x03030303u, (w[j] >> 6) & 0x03030303u);
                    *reinterpret_cast<uint4 *>(dst + ((j ^ (m & 7)) << 4)) = c;
                }
                // The tensor cores read the codes through the async proxy.
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&bars->afull[sa]));
                    mbar_arrive(smem_u32(&bars->pempty[sp]));   // packed words consumed
                }
                ++step;
                if (++sa == kASlots) { sa = 0; pha ^= 1u; }
                if (++sp == kPSlots) { sp = 0; php ^= 1u; }
            }
        }
    } else {
        // ---------------------------------------------------- epilogue ---
        const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
        const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
        const int ep = warp - kFirstEpiWarp;
        uint8_t *my_out = out_stage + ep * 2 * kOutBufBytes;
        float2 *tok = reinterpret_cast<float2 *>(tok_stage);
        const float4 *tok4 = reinterpret_cast<const float4 *>(tok);
        // Barrier over the four epilogue warps (they share the token table).
        auto epi_barrier = [] { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); };
        const float gamma = *gamma_ptr;
        int ob = 0, i = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
            const int m0 = (tile % m_tiles) * kBM, n0 = (tile / m_tiles) * kBN;
            const int buf = i & 1, use = i >> 1;
            const bool ok = wait_or_abort(smem_u32(&bars->acc_full[buf]), (uint32_t)use & 1u, ctx,
                                          abort_flag);
            // The four warps share a barrier, so they leave together: each
            // posts its result, and after the barrier all read the same four.
            const bool warp_ok = __all_sync(0xffffffffu, ok);
            if (lane == 0) bars->epi_ok[ep] = warp_ok ? 1 : 0;
            epi_barrier();
            const volatile int *eok = bars->epi_ok;
            if (!(eok[0] && eok[1] && eok[2] && eok[3])) break;
            tc_fence_after();
            const int r0 = m0 + quarter * 32;   // first output row of this warp
            const int o = r0 + lane;
            // Token table of this tile, {gamma beta / 127, code sum}, written by
            // the four warps together (64 tokens each) and read back as
            // broadcasts; the barrier above kept it until every warp was done
            // with the previous tile's.
            #pragma unroll
            for (int q = 0; q < kBN / (32 * kEpiWarps); ++q) {
                const int tl = (q * kEpiWarps + ep) * 32 + lane;
                const int t = n0 + tl;
                float sc = 0.0f;
                int rs = 0;
                if (t < T) {
                    sc = __fdiv_rn(__fmul_rn(gamma, beta[t]), 127.0f);
                    rs = rowsum[t];
                }
                tok[tl] = make_float2(sc, __int_as_float(rs));
            }
            epi_barrier();
            #pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                const int tc0 = n0 + c * 32;
                if (tc0 >= T || r0 >= d_out) break;   // uniform: nothing of this block exists
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_field + buf * kAccCols + c * 32, v);
                tmem_wait_ld();
                #pragma unroll
                for (int h = 0; h < 32 / kChunk; ++h) {
                    const int t0 = tc0 + h * kChunk;
                    if (t0 < T) {   // uniform
                        // The block staged two blocks ago has been read by its store.
                        if (lane == 0) bulk_wait_read_1();
                        __syncwarp();
                        uint8_t *stg = my_out + ob * kOutBufBytes;
                        #pragma unroll
                        for (int j2 = 0; j2 < kChunk / 2; ++j2) {
                            const float4 tp = tok4[(c * 32 + h * kChunk) / 2 + j2];
                            #pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int j = 2 * j2 + e;
                                const float sc = e ? tp.z : tp.x;
                                const int rs = __float_as_int(e ? tp.w : tp.y);
                                const int a = (int)v[h * kChunk + j] - rs;
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
            // Accumulator drained: the MMA may refill it.
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
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------ host ---

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
        const cuuint32_t box[2] = {kBK, kBN};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(Xq), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    {
        // Packed words as a 4-D array [row tile][k tile][row in tile][word]; a
        // step takes words 8 (kt & 1) .. +7 of tile kt / 2 for 8 row tiles.
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
    {
        // Output [T][d_out], written in 32-row x 16-token boxes.
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
