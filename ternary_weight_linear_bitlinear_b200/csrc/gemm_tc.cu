// gemm_tc.cu -- prefill ternary x int8 product on the 5th-generation tensor
// cores, CTA pairs (tcgen05 cta_group::2, sm_100a).
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 2,
// "The Linear Transformation and Rescaling": Y = (X~ W~^T) beta gamma /
// (Q_b - 1) with int32 accumulation.  With more than 16 tokens the product is
// a dense contraction and runs as an int8 MMA,
//
//   D[t][o] = sum_k X~[t][k] * C[o][k]     (C = W~ + 1 in {0,1,2}, s8 x u8)
//
// rescaled by gamma beta_t / 127 after subtracting each token's code sum
// S_t = sum_k X~[t][k].
//
// Two CTAs on two SMs (a cluster pair) compute a 256-token x 256-row output
// tile with tcgen05.mma.cta_group::2: one instruction does M = 256 x N = 256
// x K = 32, twice the work of a single-CTA M = 128 instruction, and each CTA
// supplies half of each operand -- its 128 tokens (A, signed) and its
// 128 weight rows (B, unsigned codes) -- and receives its 128 tokens x 256
// rows of the accumulator.  CTA r (cluster rank r) loads tokens n0 + 128 r ..
// and expands weight rows m0 + 128 r ...
//
// Each pipeline stage holds both operands of one 128-column step in each CTA.
// Roles in each CTA:
//   * warp 0 (one lane): TMA of its token half into the stage (`full`) and
//     of its rows' packed codes into the packed ring (`pfull`);
//   * warp 14 (one lane): relays each landed token half to the leader's
//     `ready` (so every copy completes on a barrier of the CTA that issued
//     it, and each CTA can wait for its own copies);
//   * warps 2..5 and 10..13 (two groups taking alternate steps): expand the
//     packed codes into the stage in the 128-byte swizzled K-major layout,
//     then arrive on the leader's `ready`;
//   * warp 1 of the leader: per step one wait on `ready` (both CTAs' token
//     halves and weight codes), four MMAs and one commit, multicast to both
//     CTAs, to `freed`; at a tile's end a commit to `acc_full`;
//   * warps 6..9: drain their CTA's accumulator half (tcgen05.ld): a lane is
//     a token, so each thread writes its token's outputs for 256 consecutive
//     rows as 16-byte vectors straight to Y, then arrives on the leader's
//     `acc_empty`.
// What sets the speed (measured): the single MMA-issuing thread.  Its
// operands are ready thousands of cycles early, but each of its barrier
// checks, MMA issues and commits takes tens to a hundred cycles, and any
// instruction-heavy warp on its SM sub-partition slows it further -- with an
// epilogue that looked up a token table and stored 2-byte values to shared
// memory for every output, the kernel ran 100 us on the 2048 x 4096 -> 11008
// prefill; with this one, 76 us (an empty epilogue: 61 us).  Hence one
// barrier check and one commit per step, and an epilogue of about four
// instructions per output.  Cross-CTA arrivals use the default release
// semantics; asking for cluster scope made each arrival cost about 1100
// cycles.  Every wait is bounded; on expiry a CTA stops issuing, waits for
// its own copies and for the pair's MMAs, and leaves through the final
// cluster barrier with the device error word set.  No load uses cluster
// multicast; only the MMA commits are multicast.
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>

#include "bitlinear.h"
#include "common.cuh"
#include "tc_common.cuh"

namespace bl {

namespace pair {

constexpr int kBM = 128;          // weight rows per CTA (MMA N = 256 per pair)
constexpr int kBN = 256;          // tokens per pair tile (MMA M), 128 loaded by each CTA
constexpr int kBNHalf = kBN / 2;
constexpr int kBK = 128;          // reduction columns per step (bytes)
// A stage holds both operands of one 128-column step: this CTA's 16 KiB token
// half (A) and its 16 KiB of expanded weight codes (B).  One barrier per
// stage says both CTAs' operands are in place and one multicast commit frees
// it, so the MMA issuer makes a single check and a single commit per step.
constexpr int kStages = 5;
// A packed slot holds this CTA's eight 16 x 256 packed tiles of one 256-column
// k tile -- two steps -- fetched as eight contiguous 1 KiB pieces.  The unit
// of steps 2u, 2u + 1 is loaded with the tokens of step 2u - kPAhead, so it
// lands about kPAhead steps before the expanders may start on it (they start
// on step g when the stage's previous step g - kStages is freed, which is
// also when its tokens are requested).  With 2 kPSlots >= kPAhead + kStages + 1
// its slot was released before the producer reaches it.
constexpr int kPSlots = 6;        // packed ring (units of two steps)
constexpr int kPAhead = 6;        // steps the packed loads run ahead of the token loads
constexpr int kBTile = kBNHalf * kBK;        // 16 KiB: this CTA's token half
constexpr int kATile = kBM * kBK;            // 16 KiB: this CTA's expanded weight codes
constexpr int kStage = kBTile + kATile;
constexpr int kPUnit = kBM * 2 * kBK / 4;    // 8 KiB packed codes of two steps
constexpr int kAccCols = kBN;
constexpr int kAccBufs = 2;
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 4;
constexpr int kFirstEpiWarp = 6;
constexpr int kFirstExp2Warp = kFirstEpiWarp + kEpiWarps;    // second expander group
constexpr int kRelayWarp = kFirstExp2Warp + 4;
constexpr int kThreads = 32 * (kRelayWarp + 1);              // 15 warps
// Arrivals that complete a stage's `ready` phase: the two CTAs' relays and
// the four warps of one expander group in each CTA.
constexpr int kReadyCount = 2 + 2 * 4;
static_assert(kAccBufs * kAccCols <= kTmemCols, "tensor memory budget");
static_assert(kBTile % 1024 == 0 && kATile % 1024 == 0, "1024-byte swizzle alignment");
static_assert(2 * kPSlots >= kPAhead + kStages + 1, "packed ring depth");

struct __align__(8) Barriers {
    uint64_t full[kStages];       // both: this CTA's token half landed (TMA bytes)
    uint64_t ready[kStages];      // leader: both CTAs' operands of the stage are in place
    uint64_t freed[kStages];      // both: the MMAs of the stage completed (multicast commit)
    uint64_t pfull[kPSlots];      // own packed ring
    uint64_t pempty[kPSlots];
    uint64_t acc_full[kAccBufs];  // both: multicast commit
    uint64_t acc_empty[kAccBufs]; // leader: 4 warps x 2 CTAs drained their halves
    uint64_t drain;               // both: multicast commit after the last MMA
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Barriers) <= 1024, "barrier block");
// Epilogue staging for the tensor-map store of Y: per epilogue warp 2 KiB, one
// box of 32 tokens x 64 bytes (32 bf16 or 16 fp32 outputs, 64-byte swizzle).
// Small enough that a quantiser CTA still fits beside this CTA on its SM, so
// that under a programmatic launch this CTA's prologue overlaps the
// quantiser (measured: 4 KiB per warp lost that overlap).
constexpr int kStageY = 2048;
constexpr int kSmemBytes = kStages * kStage + kPSlots * kPUnit + 1024 /* barriers */ +
                           kEpiWarps * kStageY + 1024 /* alignment slack */;
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

// ------------------------------------------------------------- cluster ---
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The shared::cluster address of `addr` (a shared::cta address) in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// Arrival on a barrier of the peer CTA, with the instruction's default
// semantics (release).  Asking for cluster scope explicitly made the arriving
// thread wait about 1100 cycles per arrival (measured); this form costs about
// 100.  The signalled data are shared-memory operands that only the pair's
// tensor cores read, after the leader's acquire and tcgen05 fence.
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Wait with cluster-scope acquire (for barriers a peer CTA arrives on).
__device__ __forceinline__ bool try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ bool wait_cluster_or_abort(uint32_t bar, uint32_t parity,
                                                      const DeviceCtx &ctx,
                                                      volatile int *abort_flag) {
    if (try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > ctx.wait_ns) {
            atomicOr(ctx.err, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
    }
}

// -------------------------------------------------------- pair tcgen05 ---
__device__ __forceinline__ void mma_i8_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on the barrier at this offset in both CTAs once the MMAs issued so
// far complete.
__device__ __forceinline__ void commit_pair_both(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar), "h"((uint16_t)3)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

}  // namespace pair

template <bool OUT_BF16>
__global__ void __launch_bounds__(pair::kThreads, 1)
gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                    const __grid_constant__ CUtensorMap map_y,
                    const float *__restrict__ gamma_ptr, int d_out, int d_in,
                    const float *__restrict__ beta, const int32_t *__restrict__ rowsum, int T,
                    void *__restrict__ Y, int32_t *__restrict__ acc_out, DeviceCtx ctx) {
    using namespace pair;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *p_ring = smem + kStages * kStage;
    Barriers *bars = reinterpret_cast<Barriers *>(p_ring + kPSlots * kPUnit);
    uint8_t *y_stage = p_ring + kPSlots * kPUnit + 1024;   // 1024-byte aligned
    const uint32_t smem_base = smem_u32(smem);
    auto stage_x = [&](int s) { return smem_base + s * kStage; };   // token half; codes at + kBTile

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair_id = (int)(blockIdx.x >> 1), num_pairs = (int)(gridDim.x >> 1);
    const int m_tiles = (d_out + 2 * kBM - 1) / (2 * kBM);
    const int num_tiles = m_tiles * ((T + kBN - 1) / kBN);
    const int num_k = d_in / kBK;
    const int my_tiles = pair_id < num_tiles ? (num_tiles - 1 - pair_id) / num_pairs + 1 : 0;
    const int total = my_tiles * num_k;   // steps; num_k is even, so units never straddle tiles
    const int total_units = total / 2;
    volatile int *abort_flag = &bars->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->ready[s]), kReadyCount);
            mbar_init(smem_u32(&bars->freed[s]), 1);
        }
        for (int s = 0; s < kPSlots; ++s) {
            mbar_init(smem_u32(&bars->pfull[s]), 1);
            mbar_init(smem_u32(&bars->pempty[s]), 2 * 4);   // both expander groups
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(smem_u32(&bars->acc_full[b]), 1);
            mbar_init(smem_u32(&bars->acc_empty[b]), 2 * kEpiWarps);
        }
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort_flag = 0;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
    }
    // The pair's tensor memory is allocated by warp 1 of both CTAs together.
    if (warp == 1) tmem_alloc_pair(smem_u32(&bars->tmem_base), kTmemCols);
    // Both CTAs' barriers and tensor memory exist before either CTA signals
    // the other or issues an MMA.
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    // Leader barriers that this CTA signals: local in the leader, through the
    // cluster window in the follower.
    auto signal_leader = [&](const uint64_t *b) {
        if (leader) mbar_arrive(smem_u32(b));
        else arrive_remote(map_to_rank(smem_u32(b), 0));
    };
    pdl_wait_primary();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ---
        if (lane == 0) {
            auto issue_unit = [&](int u) {
                const int g = 2 * u;
                const int tile = pair_id + (g / num_k) * num_pairs;
                const int kt = g - (g / num_k) * num_k;
                const int m0 = (tile % m_tiles) * 2 * kBM + (int)rank * kBM;
                const uint32_t pb = smem_u32(&bars->pfull[u % kPSlots]);
                mbar_arrive_expect_tx(pb, kPUnit);
                tma_load_3d(smem_u32(p_ring + (u % kPSlots) * kPUnit), &map_w, 0, kt >> 1, m0 / 16,
                            pb);
            };
            // Issue every unit whose first step is at most `last_step`; a slot
            // is reused once the expanders released unit u - kPSlots.
            int u_issued = 0;
            auto issue_units_through = [&](int last_step) {
                while (u_issued < total_units && 2 * u_issued <= last_step) {
                    if (u_issued >= kPSlots &&
                        !wait_or_abort(smem_u32(&bars->pempty[u_issued % kPSlots]),
                                       (uint32_t)(u_issued / kPSlots - 1) & 1u, ctx, abort_flag))
                        return false;
                    issue_unit(u_issued++);
                }
                return true;
            };
            bool ok = issue_units_through(kPAhead - 1);
            int step = 0;
            for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
                const int n0 = (tile / m_tiles) * kBN + (int)rank * kBNHalf;
                for (int kt = 0; kt < num_k; ++kt) {
                    const int s = step % kStages;
                    // The stage's previous step was consumed by the pair's MMAs.
                    if (step >= kStages &&
                        !wait_or_abort(smem_u32(&bars->freed[s]),
                                       (uint32_t)(step / kStages - 1) & 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&bars->full[s]);
                    mbar_arrive_expect_tx(fb, kBTile);
                    tma_load_2d(stage_x(s), &map_x, kt * kBK, n0, fb);
                    ++step;
                    if (!issue_units_through(step - 1 + kPAhead)) {
                        ok = false;
                        break;
                    }
                }
            }
            // Drain: every copy this CTA issued lands before it may exit.
            for (int q = step > kStages ? step - kStages : 0; q < step; ++q)
                mbar_wait_bounded(smem_u32(&bars->full[q % kStages]),
                                  (uint32_t)(q / kStages) & 1u, ctx);
            for (int q = u_issued > kPSlots ? u_issued - kPSlots : 0; q < u_issued; ++q)
                mbar_wait_bounded(smem_u32(&bars->pfull[q % kPSlots]),
                                  (uint32_t)(q / kPSlots) & 1u, ctx);
        }
    } else if (warp == kRelayWarp) {
        // ------------------------------------------------------- relay ---
        // This CTA's token half of step g landed: count it on the leader's
        // `ready`.  The step's previous use of the stage was consumed by an
        // MMA issued after its `ready` phase completed, so arrivals never run
        // a phase ahead.
        if (lane == 0) {
            for (int g = 0; g < total; ++g) {
                const int s = g % kStages;
                if (!wait_or_abort(smem_u32(&bars->full[s]), (uint32_t)(g / kStages) & 1u, ctx,
                                   abort_flag))
                    break;
                signal_leader(&bars->ready[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------ MMA issuer (leader) ---
        if (lane == 0 && leader) {
            // The tokens are the A operand (M = 256 tokens of the pair, signed)
            // and the weight codes B (N = 256 rows, unsigned), so that a
            // tensor-memory lane holds one token's outputs for 256
            // consecutive rows -- contiguous in Y -- for the epilogue.
            constexpr uint32_t idesc = (2u << 4)            // D s32
                                       | (1u << 7)          // A signed 8-bit (tokens)
                                       | (0u << 10)         // B unsigned 8-bit (codes)
                                       | ((uint32_t)((2 * kBM) >> 3) << 17)      // N / 8
                                       | ((uint32_t)((2 * kBNHalf) >> 4) << 24); // M / 16
            // Descriptors of stage 0; a stage is kStage >> 4 descriptor units
            // further and a 32-column slice 2 units.
            const uint64_t xdesc0 = smem_desc_sw128(stage_x(0));
            const uint64_t wdesc0 = smem_desc_sw128(stage_x(0) + kBTile);
            const uint32_t ready0 = smem_u32(&bars->ready[0]);
            const uint32_t freed0 = smem_u32(&bars->freed[0]);
            int s = 0, i = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs, ++i) {
                const int buf = i & 1, use = i >> 1;
                if (use > 0 && !wait_cluster_or_abort(smem_u32(&bars->acc_empty[buf]),
                                                      (uint32_t)(use - 1) & 1u, ctx, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t tmem_acc = tmem_base + buf * kAccCols;
                for (int kt = 0; kt < num_k; ++kt) {
                    if (!wait_cluster_or_abort(ready0 + 8 * s, ph, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t off = (uint64_t)(s * (kStage >> 4));
                    #pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)
                        mma_i8_ss_pair(tmem_acc, xdesc0 + off + 2 * kk, wdesc0 + off + 2 * kk,
                                       idesc, (kt > 0 || kk > 0) ? 1u : 0u);
                    commit_pair_both(freed0 + 8 * s);
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                }
                if (ok) commit_pair_both(smem_u32(&bars->acc_full[buf]));
            }
            // Completion of everything issued, in both CTAs, before either
            // frees tensor memory or exits.
            commit_pair_both(smem_u32(&bars->drain));
        }
        if (lane == 0) mbar_wait_bounded(smem_u32(&bars->drain), 0, ctx);
        __syncwarp();
    } else if (warp < kFirstEpiWarp || warp >= kFirstExp2Warp) {
        // ---------------------------------------------------- expander ---
        // Two groups of four warps take alternate steps (group grp the steps
        // g = grp mod 2), so each warp's serial chain per step -- waits,
        // stores, proxy fence, arrival -- has two steps' time.  Thread m
        // (weight row m of the CTA) reads its row's eight packed words of the
        // step; word j holds columns 16 j .. 16 j + 15 of the step, column
        // 16 j + 4 s + b in bits 8 b + 2 s, so (word >> 2 s) & 0x03030303 is
        // the four codes of columns 16 j + 4 s + 0..3: word j expands to the
        // 16-byte chunk j of the row, which the 128-byte swizzle places at
        // chunk j ^ (m mod 8) of the row's 128 bytes.  In the packed slot,
        // row m's sixteen words of the unit sit at 1024 (m / 16) +
        // 64 (m mod 16); step g takes the half at + 32 (g mod 2).  The two
        // 16-byte halves are read in an order that alternates with m / 2,
        // which halves the bank conflicts of the 64-byte row stride.
        const int grp = warp >= kFirstExp2Warp ? 1 : 0;
        const int m = (warp & 3) * 32 + lane;
        uint8_t *arow = smem + kBTile + m * kBK;
        const int prow = (m >> 4) * 1024 + (m & 15) * 64 + grp * 32;
        const int flip = (m >> 1) & 1;
        bool ok = true;
        for (int g = grp; g < total && ok; g += 2) {
            const int s = g % kStages, u = g >> 1, sp = u % kPSlots;
            ok = wait_or_abort(smem_u32(&bars->pfull[sp]), (uint32_t)(u / kPSlots) & 1u, ctx,
                               abort_flag);
            uint32_t w[8];
            if (ok) {
                const uint4 *src = reinterpret_cast<const uint4 *>(p_ring + sp * kPUnit + prow);
                const uint4 x0 = src[flip], x1 = src[flip ^ 1];
                const uint4 lo = flip ? x1 : x0, hi = flip ? x0 : x1;
                w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
                w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
                // The stage is free once the MMAs of its previous step completed.
                if (g >= kStages)
                    ok = wait_or_abort(smem_u32(&bars->freed[s]),
                                       (uint32_t)(g / kStages - 1) & 1u, ctx, abort_flag);
            }
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            uint8_t *dst = arow + s * kStage;
            #pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 c = make_uint4(w[j] & 0x03030303u, (w[j] >> 2) & 0x03030303u,
                                           (w[j] >> 4) & 0x03030303u, (w[j] >> 6) & 0x03030303u);
                *reinterpret_cast<uint4 *>(dst + ((j ^ (m & 7)) << 4)) = c;
            }
            // The tensor cores (issued by the leader) read the codes through
            // the async proxy.
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                signal_leader(&bars->ready[s]);
                mbar_arrive(smem_u32(&bars->pempty[sp]));   // this group's half of the unit read
            }
        }
    } else {
        // ---------------------------------------------------- epilogue ---
        // Tensor-memory lane 32 (warp mod 4) + l of this CTA's accumulator
        // is its token n0 + 32 (warp mod 4) + l, and column j is weight row
        // m0 + j of the pair tile.  Each thread so holds its token's outputs
        // for 256 consecutive rows, contiguous in Y[t][.]: it subtracts the
        // token's code sum, scales by gamma beta / 127 and writes 16-byte
        // vectors straight to global memory.  (With rows in the lanes, each
        // output needed a table lookup and a 2-byte shared-memory store; that
        // epilogue's instruction stream slowed the MMA issuer sharing its
        // SM sub-partition by half -- measured.)
        const int quarter = warp & 3;
        const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
        const float gamma = *gamma_ptr;
        // Without acc_out, each 32-row chunk of the warp's 32 tokens goes
        // through shared memory (row = token, swizzled so the lanes' 16-byte
        // writes do not conflict) and out with one tensor-map store, which
        // writes whole lines and clips tokens past T and rows past d_out.
        const bool staged = acc_out == nullptr;
        const uint32_t ystage = smem_u32(y_stage) + (uint32_t)(quarter * kStageY);
        int i = 0;
        for (int tile = pair_id; tile < num_tiles; tile += num_pairs, ++i) {
            const int m0 = (tile % m_tiles) * 2 * kBM;
            const int t = (tile / m_tiles) * kBN + (int)rank * kBNHalf + quarter * 32 + lane;
            const int buf = i & 1, use = i >> 1;
            const bool ok = wait_or_abort(smem_u32(&bars->acc_full[buf]), (uint32_t)use & 1u, ctx,
                                          abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const bool live = t < T;
            const float sc = live ? __fdiv_rn(__fmul_rn(gamma, beta[t]), 127.0f) : 0.0f;
            const int rs = live ? rowsum[t] : 0;
            #pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                const int o0 = m0 + c * 32;
                if (o0 >= d_out) break;   // uniform: rows past the matrix
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_field + buf * kAccCols + c * 32, v);
                tmem_wait_ld();
                if (staged) {
                    float y[32];
                    #pragma unroll
                    for (int e = 0; e < 32; ++e) y[e] = __fmul_rn((float)((int)v[e] - rs), sc);
                    // bf16: one box of the 32 outputs; fp32: two boxes of 16.
                    constexpr int kBoxes = OUT_BF16 ? 1 : 2;
                    #pragma unroll
                    for (int h = 0; h < kBoxes; ++h) {
                        if (lane == 0) bulk_wait_read_0();   // the buffer's last store has read it
                        __syncwarp();
                        // row = lane, 64 bytes: chunk k at k ^ ((lane >> 1) & 3)
                        #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            uint32_t pw[4];
                            if (OUT_BF16) {
                                #pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const __nv_bfloat162 hh = __floats2bfloat162_rn(
                                        y[8 * k + 2 * e], y[8 * k + 2 * e + 1]);
                                    pw[e] = *reinterpret_cast<const uint32_t *>(&hh);
                                }
                            } else {
                                #pragma unroll
                                for (int e = 0; e < 4; ++e) pw[e] = __float_as_uint(y[16 * h + 4 * k + e]);
                            }
                            const uint32_t at = ystage + (uint32_t)lane * 64u +
                                                (((uint32_t)k ^ (((uint32_t)lane >> 1) & 3u)) << 4);
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(at),
                                         "r"(pw[0]), "r"(pw[1]), "r"(pw[2]), "r"(pw[3])
                                         : "memory");
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&map_y, ystage, o0 + 16 * h, t - lane);
                            bulk_commit_group();
                        }
                    }
                    continue;
                }
                if (!live) continue;
                #pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int o = o0 + q * 8;
                    if (o >= d_out) break;   // d_out is a multiple of 16: whole vectors
                    int a[8];
                    float y[8];
                    #pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        a[e] = (int)v[q * 8 + e] - rs;
                        y[e] = __fmul_rn((float)a[e], sc);
                    }
                    const size_t base = (size_t)t * d_out + o;
                    if (OUT_BF16) {
                        uint4 pk;
                        uint32_t *pw = reinterpret_cast<uint32_t *>(&pk);
                        #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * e], y[2 * e + 1]);
                            pw[e] = *reinterpret_cast<const uint32_t *>(&h);
                        }
                        *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(Y) + base) = pk;
                    } else {
                        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(Y) + base);
                        dst[0] = make_float4(y[0], y[1], y[2], y[3]);
                        dst[1] = make_float4(y[4], y[5], y[6], y[7]);
                    }
                    if (acc_out) {
                        int4 *dst = reinterpret_cast<int4 *>(acc_out + base);
                        dst[0] = make_int4(a[0], a[1], a[2], a[3]);
                        dst[1] = make_int4(a[4], a[5], a[6], a[7]);
                    }
                }
            }
            // This CTA's half of the accumulator is drained.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) signal_leader(&bars->acc_empty[buf]);
        }
        // Every staged store has completed before the CTA may exit.
        if (staged && lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    // Neither CTA frees tensor memory or exits while the other may still
    // signal it.
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------ host ---

// Launches the CTA-pair kernel: 2 x min(pair tiles, SMs / 2) CTAs in clusters
// of two, one pair per two SMs.  A pair tile spans as many SMs as two 128-row
// single-CTA tiles would, so every problem uses the pair form.
// The prefill GEMM's launch (both tensor maps encoded) as a launch record.
bitlinear_status prepare_gemm_tc_pair(const uint32_t *packed, const float *gamma, int64_t d_out,
                                      int64_t d_in, const int8_t *Xq, const float *beta,
                                      const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                      int32_t *acc_out, LaunchRec *rec) {
    using namespace pair;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t pair_tiles = ((d_out + 2 * kBM - 1) / (2 * kBM)) * ((T + kBN - 1) / kBN);
    PFN_encodeTiled encode = get_encode_fn();
    if (!encode) return BITLINEAR_ERR_CUDA;
    DeviceCtx ctx;
    bitlinear_status st = get_ctx(&ctx);
    if (st != BITLINEAR_OK) return st;
    const bool bf = out_dtype == BITLINEAR_OUT_BF16;

    CUtensorMap map_x, map_w;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)d_in};
        const cuuint32_t box[2] = {kBK, kBNHalf};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(Xq), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    {
        // Packed words as [row tile][k tile][256 words]; a unit is the k tile's
        // 1 KiB of each of the CTA's eight row tiles.
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
    CUtensorMap map_y;
    {
        // Y [T][d_out]; boxes of 32 tokens x 64 bytes (32 bf16 or 16 fp32
        // outputs), the 64-byte swizzle of the epilogue's staging.
        const cuuint64_t esz = bf ? 2 : 4;
        const cuuint64_t dims[2] = {(cuuint64_t)d_out, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)d_out * esz};
        const cuuint32_t box[2] = {bf ? 32u : 16u, 32};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&map_y, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   2, Y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BITLINEAR_ERR_CUDA;
    }
    auto kern = bf ? gemm_tc_pair_kernel<true> : gemm_tc_pair_kernel<false>;
    if (ensure_dynamic_smem((const void *)kern, kSmemBytes) != cudaSuccess)
        return BITLINEAR_ERR_CUDA;
    const int64_t max_pairs = sms / 2 > 0 ? sms / 2 : 1;
    const int64_t pairs = pair_tiles < max_pairs ? pair_tiles : max_pairs;

    *rec = LaunchRec();
    rec->func = (const void *)kern;
    rec->grid = dim3((unsigned)(2 * pairs));
    rec->block = dim3(kThreads);
    rec->smem = kSmemBytes;
    rec->cluster_x = 2;
    rec->pdl = true;
    rec->push(map_x);
    rec->push(map_w);
    rec->push(map_y);
    rec->push(gamma);
    rec->push((int)d_out);
    rec->push((int)d_in);
    rec->push(beta);
    rec->push(rowsum);
    rec->push((int)T);
    rec->push(Y);
    rec->push(acc_out);
    rec->push(ctx);
    return BITLINEAR_OK;
}

bitlinear_status launch_gemm_tc_pair(const uint32_t *packed, const float *gamma, int64_t d_out,
                                     int64_t d_in, const int8_t *Xq, const float *beta,
                                     const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                     int32_t *acc_out, cudaStream_t stream) {
    LaunchRec rec;
    bitlinear_status st = prepare_gemm_tc_pair(packed, gamma, d_out, d_in, Xq, beta, rowsum, T,
                                               Y, out_dtype, acc_out, &rec);
    if (st != BITLINEAR_OK) return st;
    return rec.launch(stream) == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

}  // namespace bl
