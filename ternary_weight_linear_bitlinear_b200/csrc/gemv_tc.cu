// gemv_tc.cu -- decode-time ternary x int8 product (1..16 tokens) on the
// 5th-generation tensor cores (tcgen05, sm_100a).
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 2,
// "The Linear Transformation and Rescaling" (Y = (X~ W~^T) beta gamma /
// (Q_b - 1), int32 accumulation), and section 4, "Memory Bandwidth and
// Latency Bounds" (a decode step costs the weight bytes over the memory
// bandwidth).  Section 6 unpacks 2-bit codes into masks for a SIMD add; here
// the unpacked codes feed the int8 tensor-core MMA.
//
// One MMA is M = 128 weight rows x N = 16 token slots x K = 32 columns
// (tcgen05.mma.cta_group::1.kind::i8, tokens past T are zero rows of the
// token operand).  The weight operand A lives in tensor memory: writer warps
// turn the 2-bit codes of their rows into u8 codes c = W~ + 1 in registers
// and store them with tcgen05.st, so the codes never pass through shared
// memory a second time.  In the packed layout word kw of a row holds columns
// 16 kw + 4 s + j at bits 8 j + 2 s, so (word >> 2 s) & 0x03030303 is the
// four codes of columns 16 kw + 4 s + 0..3: the tensor-memory column 4 kw + s
// of the row (four K elements per 32-bit column), in the natural column
// order of the token codes.  The accumulator, sum c x, becomes W~ X~ by
// subtracting the token's code sum.
//
// Roles (448 threads): warps 0..7 write A (warp w owns tensor-memory lanes
// 32 (w mod 4) .. +31, i.e. rows 32 (w mod 4) .. +31 of the block, and the
// columns of chunks 2 (w / 4) and 2 (w / 4) + 1 of each k-tile); warps 8..11
// drain the accumulators (the same lanes); warp 12 issues the TMA copies of a
// ring of shared-memory stages (packed weights with the 64-byte swizzle, so
// that the writers' row reads are conflict-free, and the token codes with
// the 128-byte swizzle the MMA's K-major operand descriptor expects); warp 13
// allocates tensor memory and one of its threads issues the MMAs.
//
// Work: units of (128-row block, k-tile), group-major, cut into one share per
// CTA -- whole blocks, or with a split workspace equal shares whose shared
// blocks meet in the workspace as in the warp-MMA decode kernel (the same
// self-describing 64-bit words; see gemv.cu, "Balanced split").
//
// Every wait is bounded; on expiry the CTA stops, the error word is set, the
// producer waits (bounded) for the copies it issued and the MMA thread for
// the MMAs it issued before tensor memory is freed.
#include <cstddef>
#include <cstdint>

#include <cuda_bf16.h>

#include "bitlinear.h"
#include "common.cuh"
#include "decode_common.cuh"
#include "tc_common.cuh"

namespace bl {
namespace dtc {

constexpr int kRows = 128;                 // M: weight rows per block (tensor-memory lanes)
constexpr int kN = 16;                     // N: token slots
constexpr int kRowTiles = kRows / 16;      // packed 16-row tiles per block
constexpr int kWTile = 1024;               // packed bytes of one 16 x 256 tile
constexpr int kXTile = kN * 256;           // token codes of one k-tile (two 128-column boxes)
constexpr int kMaxStages = 4;
constexpr int kWriterWarps = 8;            // two per tensor-memory lane quarter
constexpr int kEpiWarp0 = 8;               // warps 8..11
constexpr int kProducerWarp = 12, kMmaWarp = 13;
constexpr int kThreads = 14 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr int kACols = 64;                 // A of one k-tile: 256 int8 = 64 columns
constexpr int kABufs = 4;
constexpr int kAccCols = kN;               // one int32 accumulator per token slot
constexpr int kAccBufs = 2;
constexpr int kAccBase = kABufs * kACols;  // columns [A0 | A1 | acc0 | acc1]
static_assert(kAccBase + kAccBufs * kAccCols <= (int)kTmemCols, "tensor memory plan");

// The split workspace word (the same layout as gemv.cu).
constexpr int kSplitKShift = 45;
constexpr int kSplitPartsShift = 36;
constexpr unsigned long long kSplitSumMask = (1ull << kSplitPartsShift) - 1;
constexpr long long kSplitBias = 1ll << 25;

struct Args {
    const float *gamma;
    int d_out, d_in, KB, T;
    const float *beta;
    const int32_t *rowsum;
    void *Y;
    int32_t *acc_out;
    unsigned long long *split_ws;   // null: whole blocks per CTA
    int static_weights;
    int ks;                         // k-tiles per stage
    int stages;
};

__device__ __forceinline__ unsigned long long split_word(int k, int v) {
    return ((unsigned long long)k << kSplitKShift) + (1ull << kSplitPartsShift) +
           (unsigned long long)(v + kSplitBias);
}
__device__ __forceinline__ int split_k(unsigned long long w) { return (int)(w >> kSplitKShift); }
__device__ __forceinline__ int split_sum(unsigned long long w) {
    const long long parts = (long long)((w >> kSplitPartsShift) & 511u);
    return (int)((long long)(w & kSplitSumMask) - parts * kSplitBias);
}

// D(tmem) (+)= A(tmem) * B(smem descriptor), kind::i8, one CTA.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
        "%10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15])
        : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 q;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(q.x), "=r"(q.y), "=r"(q.z), "=r"(q.w)
                 : "r"(addr));
    return q;
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

struct Shared {
    uint64_t full[kMaxStages], empty[kMaxStages];
    uint64_t a_full[kABufs], a_free[kABufs];
    uint64_t acc_full[kAccBufs], acc_free[kAccBufs];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    float yscale[kN];     // gamma beta_t / 127 of token t
    int rowsum[kN];
};

template <bool OUT_BF16, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap map_w,
                 const __grid_constant__ CUtensorMap map_x, const Args a, DeviceCtx ctx) {
    extern __shared__ __align__(1024) uint8_t dsm_raw[];
    __shared__ Shared sh;
    // The stages start on a 1024-byte boundary (the swizzled copies' rule);
    // the launch adds 1 KiB of slack.
    const uint32_t dsm = (smem_u32(dsm_raw) + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = a.KB, T = a.T;
    const int n_rt = a.d_out >> 4;
    const int n_mb = (a.d_out + kRows - 1) / kRows;
    const int ks = a.ks, stages = a.stages;
    const int stage_bytes = ks * (kRowTiles * kWTile + kXTile);
    // Stage st: [row tile][ks tiles of 1 KiB], then [ks k-tiles of two
    // 2 KiB token boxes].
    auto stage_w = [&](int st) { return dsm + (uint32_t)(st * stage_bytes); };
    auto stage_x = [&](int st) {
        return dsm + (uint32_t)(st * stage_bytes + ks * kRowTiles * kWTile);
    };
    volatile int *abort_flag = &sh.abort_flag;

    // This CTA's units (block, k-tile), as in gemv.cu.
    const int P = gridDim.x, c = blockIdx.x;
    int u0, u1;
    if (SPLIT) {
        const int U = n_mb * KB, q = U / P, rem = U - q * P;
        u0 = q * c + (c < rem ? c : rem);
        u1 = u0 + q + (c < rem ? 1 : 0);
    } else {
        const int q = n_mb / P, rem = n_mb - q * P;
        const int g0 = q * c + (c < rem ? c : rem);
        u0 = g0 * KB;
        u1 = (g0 + q + (c < rem ? 1 : 0)) * KB;
    }
    const int b_first = u0 / KB;
    const int nseg = u1 > u0 ? (u1 - 1) / KB - b_first + 1 : 0;
    auto seg_kb0 = [&](int sg) {
        const int b = u0 - (b_first + sg) * KB;
        return b > 0 ? b : 0;
    };
    auto seg_kb1 = [&](int sg) {
        const int e = u1 - (b_first + sg) * KB;
        return e < KB ? e : KB;
    };
    auto unit_kb = [&](int sg, int kb) { return seg_kb1(sg) - kb < ks ? seg_kb1(sg) - kb : ks; };
    auto next_unit = [&](int &sg, int &kb) {
        kb += ks;
        if (kb >= seg_kb1(sg)) {
            ++sg;
            kb = sg < nseg ? seg_kb0(sg) : 0;
        }
    };
    int units = 0;
    for (int sg = 0; sg < nseg; ++sg) units += (seg_kb1(sg) - seg_kb0(sg) + ks - 1) / ks;

    if (threadIdx.x == 0) {
        for (int st = 0; st < stages; ++st) {
            mbar_init(smem_u32(&sh.full[st]), 1);
            mbar_init(smem_u32(&sh.empty[st]), 1);
        }
        for (int b = 0; b < kABufs; ++b) {
            mbar_init(smem_u32(&sh.a_full[b]), kWriterWarps);
            mbar_init(smem_u32(&sh.a_free[b]), 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(smem_u32(&sh.acc_full[b]), 1);
            mbar_init(smem_u32(&sh.acc_free[b]), 4);
        }
        mbar_init(smem_u32(&sh.drain), 1);
        sh.abort_flag = 0;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    }
    if (warp == kMmaWarp) tmem_alloc(smem_u32(&sh.tmem_base), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sh.tmem_base;

    if (warp == kProducerWarp) {
        // --------------------------------------------------------- producer ---
        if (lane == 0) {
            // One box per stage for the weights (ks k-tiles of the block's
            // eight row tiles) and one for the token codes (2 ks atoms of 128
            // columns); the boxes are always whole: tiles past the block's
            // k-range or past d_out arrive too (zeros past the tensor) and are
            // not used.
            (void)unit_kb;
            auto arm = [&](int st) {
                mbar_arrive_expect_tx(smem_u32(&sh.full[st]),
                                      (uint32_t)(ks * (kRowTiles * kWTile + kXTile)));
            };
            auto issue_w = [&](int sg, int kb, int st) {
                tma_load_3d(stage_w(st), &map_w, 0, kb * 16, (b_first + sg) * kRowTiles,
                            smem_u32(&sh.full[st]));
            };
            auto issue_x = [&](int sg, int kb, int st) {
                (void)sg;
                tma_load_3d(stage_x(st), &map_x, 0, 0, kb * 2, smem_u32(&sh.full[st]));
            };
            // With static weights the first unit's weights are requested
            // before the dependency wait (the token codes only after it).
            const int first = units < 1 ? units : 1;
            if (a.static_weights && first) {
                arm(0);
                issue_w(0, seg_kb0(0), 0);
            }
            pdl_wait_primary();
            pdl_launch_dependents();
            int sg = 0, kb = nseg > 0 ? seg_kb0(0) : 0, st = 0, round = 0, issued = 0;
            for (int u = 0; u < units; ++u) {
                if (round > 0) {
                    if (!dec_wait(smem_u32(&sh.empty[st]), (uint32_t)(round - 1) & 1u, ctx,
                                  abort_flag))
                        break;
                }
                if (!(a.static_weights && u < first)) {
                    arm(st);
                    issue_w(sg, kb, st);
                }
                issue_x(sg, kb, st);
                ++issued;
                next_unit(sg, kb);
                if (++st == stages) { st = 0; ++round; }
            }
            // Every copy issued lands before the CTA may exit.
            for (int u = issued > stages ? issued - stages : 0; u < issued; ++u)
                mbar_wait_bounded(smem_u32(&sh.full[u % stages]), (uint32_t)(u / stages) & 1u,
                                  ctx);
        } else {
            pdl_wait_primary();
            pdl_launch_dependents();
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------ MMA issuer ---
        pdl_wait_primary();
        pdl_launch_dependents();
        if (lane == 0) {
            // A: unsigned 8-bit codes from tensor memory; B: signed 8-bit token
            // codes, K-major; D: s32.  M = 128, N = 16.
            constexpr uint32_t idesc = (2u << 4)                        // D s32
                                       | (0u << 7)                      // A unsigned 8-bit
                                       | (1u << 10)                     // B signed 8-bit
                                       | ((uint32_t)(kN >> 3) << 17)    // N / 8
                                       | ((uint32_t)(kRows >> 4) << 24);// M / 16
            int st = 0, ka = 0, sg = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (; sg < nseg && ok; ++sg) {
                const int ab = sg & 1, use = sg >> 1;
                if (use > 0 && !dec_wait(smem_u32(&sh.acc_free[ab]), (uint32_t)(use - 1) & 1u,
                                         ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(kAccBase + ab * kAccCols);
                const int kb0 = seg_kb0(sg), kb1 = seg_kb1(sg);
                for (int kb = kb0; kb < kb1 && ok; kb += ks) {
                    const int nkb = kb1 - kb < ks ? kb1 - kb : ks;
                    if (!dec_wait(smem_u32(&sh.full[st]), ph, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    for (int kk = 0; kk < nkb; ++kk, ++ka) {
                        const int abuf = ka % kABufs;
                        if (!dec_wait(smem_u32(&sh.a_full[abuf]), (uint32_t)(ka / kABufs) & 1u,
                                      ctx, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t xs = stage_x(st) + (uint32_t)(kk * kXTile);
                        #pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const uint64_t bdesc =
                                smem_desc_sw128(xs + (uint32_t)((j >> 2) * (kXTile / 2))) +
                                (uint64_t)(2 * (j & 3));
                            mma_i8_ts(d_tmem, tmem_base + (uint32_t)(abuf * kACols + 8 * j),
                                      bdesc, idesc, (kb > kb0 || kk > 0 || j > 0) ? 1u : 0u);
                        }
                        tc_commit(smem_u32(&sh.a_free[abuf]));
                    }
                    if (!ok) break;
                    tc_commit(smem_u32(&sh.empty[st]));
                    if (++st == stages) { st = 0; ph ^= 1u; }
                }
                if (ok) tc_commit(smem_u32(&sh.acc_full[ab]));
            }
            tc_commit(smem_u32(&sh.drain));
            mbar_wait_bounded(smem_u32(&sh.drain), 0, ctx);
        }
        __syncwarp();
    } else if (warp < kWriterWarps) {
        // ---------------------------------------------------------- writers ---
        pdl_wait_primary();
        pdl_launch_dependents();
        const int m = (warp & 3) * 32 + lane;         // row of the block = tensor-memory lane
        const int rl = m >> 4, r = m & 15;            // row tile of the block, row of the tile
        const int ch0 = 2 * (warp >> 2);              // this warp's two 16-byte chunks of a row
        const uint32_t lane_field = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t sw = (uint32_t)((r >> 1) & 3); // the 64-byte swizzle of this row
        int st = 0, ka = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int sg = 0; sg < nseg && ok; ++sg) {
            const int mb = b_first + sg;
            const bool live = mb * kRowTiles + rl < n_rt;
            const int kb0 = seg_kb0(sg), kb1 = seg_kb1(sg);
            for (int kb = kb0; kb < kb1 && ok; kb += ks) {
                const int nkb = kb1 - kb < ks ? kb1 - kb : ks;
                ok = dec_wait(smem_u32(&sh.full[st]), ph, ctx, abort_flag);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                for (int kk = 0; kk < nkb; ++kk, ++ka) {
                    const int abuf = ka % kABufs;
                    if (ka >= kABufs) {
                        ok = dec_wait(smem_u32(&sh.a_free[abuf]),
                                      (uint32_t)(ka / kABufs - 1) & 1u, ctx, abort_flag);
                        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    }
                    tc_fence_after();
                    // Both chunks' loads first; every lane stores (tcgen05.st
                    // is warp-wide), rows past d_out -- a warp's second half
                    // may be -- zero codes.
                    const uint32_t row_s =
                        stage_w(st) + (uint32_t)((rl * ks + kk) * kWTile + r * 64);
                    uint32_t w8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                    if (live) {
                        #pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t ch = (uint32_t)(ch0 + h);
                            const uint4 q = ld_shared_v4(row_s + ((ch ^ sw) << 4));
                            w8[4 * h + 0] = q.x;
                            w8[4 * h + 1] = q.y;
                            w8[4 * h + 2] = q.z;
                            w8[4 * h + 3] = q.w;
                        }
                    }
                    __syncwarp();
                    #pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // words kw = 4 ch + i -> columns 4 kw + s = 16 ch + 4 i + s
                        uint32_t v[16];
                        #pragma unroll
                        for (int i = 0; i < 4; ++i)
                            #pragma unroll
                            for (int s = 0; s < 4; ++s)
                                v[4 * i + s] = (w8[4 * h + i] >> (2 * s)) & 0x03030303u;
                        tmem_st_x16(tmem_base + lane_field +
                                        (uint32_t)(abuf * kACols + 16 * (ch0 + h)),
                                    v);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&sh.a_full[abuf]));
                }
                if (++st == stages) { st = 0; ph ^= 1u; }
            }
        }
    } else {
        // --------------------------------------------------------- epilogue ---
        pdl_wait_primary();
        pdl_launch_dependents();
        const int q4 = warp - kEpiWarp0;
        const int m = q4 * 32 + lane;
        const uint32_t lane_field = (uint32_t)(q4 * 32) << 16;
        if (q4 == 0 && lane < T) {
            sh.yscale[lane] = __fdiv_rn(__fmul_rn(__ldg(a.gamma), __ldg(a.beta + lane)), 127.0f);
            sh.rowsum[lane] = __ldg(a.rowsum + lane);
        }
        asm volatile("bar.sync 3, 128;" ::: "memory");   // the four epilogue warps
        auto emit = [&](int mb, int t, int v) {
            const int o = mb * kRows + m;
            const int accv = v - sh.rowsum[t];
            const size_t yi = (size_t)t * a.d_out + o;
            if (a.acc_out) a.acc_out[yi] = accv;
            const float y = __fmul_rn((float)accv, sh.yscale[t]);
            if (OUT_BF16)
                reinterpret_cast<__nv_bfloat16 *>(a.Y)[yi] = __float2bfloat16_rn(y);
            else
                reinterpret_cast<float *>(a.Y)[yi] = y;
        };
        // Split: the words of the last segment and of a shared first
        // segment, loaded when the last segment is next.
        const bool first_shared = SPLIT && nseg > 1 && seg_kb0(0) > 0;
        unsigned long long pre_w[SPLIT ? kN : 1], first_w[SPLIT ? kN : 1];
        auto words = [&](int mb) { return a.split_ws + ((size_t)mb * T) * kRows + m; };
        for (int sg = 0; sg < nseg; ++sg) {
            const int mb = b_first + sg;
            const int kb0 = seg_kb0(sg), kb1 = seg_kb1(sg);
            const bool part = SPLIT && (kb0 > 0 || kb1 < KB);
            const bool last_part = part && sg == nseg - 1;
            const bool row_ok = mb * kRows + m < a.d_out;
            const int my_k = kb1 - kb0;
            if constexpr (SPLIT) {
                if (sg == nseg - 1) {
                    #pragma unroll
                    for (int t = 0; t < kN; ++t) {
                        const bool in = t < T && row_ok;
                        pre_w[t] = last_part && in ? ld_relaxed_gpu_u64(words(mb) + t * kRows)
                                                   : 0ull;
                        first_w[t] = first_shared && in
                                         ? ld_relaxed_gpu_u64(words(b_first) + t * kRows)
                                         : 0ull;
                    }
                }
            }
            const int ab = sg & 1;
            bool ok = dec_wait(smem_u32(&sh.acc_full[ab]), (uint32_t)(sg >> 1) & 1u, ctx,
                               abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            uint32_t v[16];
            tmem_ld_x16(tmem_base + lane_field + (uint32_t)(kAccBase + ab * kAccCols), v);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.acc_free[ab]));
            if (!row_ok) continue;
            #pragma unroll
            for (int t = 0; t < kN; ++t) {
                if (t >= T) break;
                const int vt = (int)v[t];
                if (!part) {
                    emit(mb, t, vt);
                } else if constexpr (SPLIT) {
                    unsigned long long *w = words(mb) + t * kRows;
                    if (last_part) {
                        unsigned long long wd = pre_w[t];
                        if (split_k(wd) + my_k != KB) wd = atomicAdd(w, split_word(my_k, vt));
                        if (split_k(wd) + my_k == KB) {
                            emit(mb, t, vt + split_sum(wd));
                            *w = 0ull;
                        }
                    } else {
                        atomicAdd(w, split_word(my_k, vt));   // checked at the end
                    }
                }
            }
        }
        if constexpr (SPLIT) {
            if (first_shared && b_first * kRows + m < a.d_out) {
                #pragma unroll
                for (int t = 0; t < kN; ++t) {
                    if (t >= T) break;
                    if (split_k(first_w[t]) == KB) {
                        emit(b_first, t, split_sum(first_w[t]));
                        *(words(b_first) + t * kRows) = 0ull;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace dtc

// Stage plan: ks k-tiles per stage, four stages, one CTA (and all tensor
// memory) per SM.
static void decode_tc_plan(int KB, int *ks, int *stages, size_t *smem) {
    int k = 4;
    if (k > KB) k = KB;
    *ks = k;
    *stages = 4;
    *smem = (size_t)(*stages) * k * (dtc::kRowTiles * dtc::kWTile + dtc::kXTile) + 1024;
}

bool decode_tc_supported(int64_t T, int64_t d_in) { return T >= 1 && T <= 16 && d_in % 256 == 0; }

int decode_split_mode();

bitlinear_status prepare_decode_tc(const uint32_t *packed, const float *gamma, int64_t d_out,
                                   int64_t d_in, const int8_t *Xq, const float *beta,
                                   const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                   int32_t *acc_out, bool static_weights, void *ws,
                                   LaunchRec *rec) {
    using namespace dtc;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    PFN_encodeTiled encode = get_encode_fn();
    if (!encode) return BITLINEAR_ERR_CUDA;
    DeviceCtx ctx;
    bitlinear_status st = get_ctx(&ctx);
    if (st != BITLINEAR_OK) return st;
    const int KB = (int)(d_in / 256);
    const int64_t n_rt = d_out / 16;
    CUtensorMap map_w, map_x;
    int ks = 0, stages = 0;
    size_t smem = 0;
    decode_tc_plan(KB, &ks, &stages, &smem);
    {
        // Packed tiles as [row tile][k-tile row = 16 kb + r][64 bytes]; a box
        // is ks k-tiles of eight row tiles, each row tile's tiles contiguous
        // in shared memory, the 64-byte swizzle on.
        const cuuint64_t dims[3] = {64, (cuuint64_t)KB * 16, (cuuint64_t)n_rt};
        const cuuint64_t strides[2] = {64, (cuuint64_t)KB * 1024};
        const cuuint32_t box[3] = {64, (cuuint32_t)(16 * ks), (cuuint32_t)kRowTiles};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (encode(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint32_t *>(packed), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    {
        // Token codes [T][d_in] as [atom of 128 columns][token][128 bytes]; a
        // box is 2 ks atoms of 16 token rows (rows past T read as zero), each
        // atom 2 KiB with the 128-byte swizzle.
        const cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)(d_in / 128)};
        const cuuint64_t strides[2] = {(cuuint64_t)d_in, 128};
        const cuuint32_t box[3] = {128, (cuuint32_t)kN, (cuuint32_t)(2 * ks)};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (encode(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t *>(Xq), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    Args args = {};
    args.gamma = gamma;
    args.d_out = (int)d_out;
    args.d_in = (int)d_in;
    args.KB = KB;
    args.T = (int)T;
    args.beta = beta;
    args.rowsum = rowsum;
    args.Y = Y;
    args.acc_out = acc_out;
    args.static_weights = static_weights ? 1 : 0;
    args.ks = ks;
    args.stages = stages;
    const bool bf = out_dtype == BITLINEAR_OUT_BF16;
    // Split (one equal share of the (block, k-tile) units per resident CTA)
    // when the blocks do not divide over the resident CTAs (one per SM).
    const int n_mb = (int)((d_out + kRows - 1) / kRows);
    const int mode = decode_split_mode();
    const bool split = ws && mode != BITLINEAR_SPLIT_NEVER &&
                       (mode == BITLINEAR_SPLIT_ALWAYS || n_mb % sms != 0);
    const void *kern;
    if (split)
        kern = bf ? (const void *)decode_tc_kernel<true, true>
                  : (const void *)decode_tc_kernel<false, true>;
    else
        kern = bf ? (const void *)decode_tc_kernel<true, false>
                  : (const void *)decode_tc_kernel<false, false>;
    if (ensure_dynamic_smem(kern, smem) != cudaSuccess) return BITLINEAR_ERR_CUDA;
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) !=
            cudaSuccess || per_sm < 1)
        per_sm = 1;
    if (per_sm > 1) per_sm = 1;   // tensor memory: all 512 columns per CTA
    int grid;
    if (split) {
        args.split_ws = static_cast<unsigned long long *>(ws);
        grid = sms * per_sm;
    } else {
        grid = n_mb < sms * per_sm ? n_mb : sms * per_sm;
    }
    *rec = LaunchRec();
    rec->func = kern;
    rec->grid = dim3((unsigned)grid);
    rec->block = dim3(kThreads);
    rec->smem = smem;
    rec->pdl = true;
    rec->push(map_w);
    rec->push(map_x);
    rec->push(args);
    rec->push(ctx);
    return BITLINEAR_OK;
}

}  // namespace bl
