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
// Work decomposition.  Row tiles (16 rows of W~) are taken R at a time
// ("groups"); a persistent CTA owns a contiguous run of groups, so it streams
// its packed weights in address order.  The CTA is warp-specialised: one
// producer warp issues bulk asynchronous copies (the TMA engine) of whole
// K-slabs -- for each row tile of a group, `ks` consecutive 1 KiB packed
// tiles, one contiguous copy -- into a ring of shared-memory stages, plus the
// matching activation codes unless they were quantised in shared memory; four
// consumer warps take the k-blocks of a stage in turn (warp w: blocks w,
// w+4, ...) and release the stage through an "empty" barrier.
//
// MMA fragments straight from the packed layout.  In a 1 KiB tile lane l
// reads bytes 16l.. of rows 0..7 and of rows 8..15 (conflict-free), so lane
// (g = l/4, q = l%4) holds words 4q..4q+3 of rows g and g+8, i.e. the A
// fragments of m16n8k32 MMAs under a permutation of the reduction index that
// the activation fragments follow too:
//   MMA (p, s), p in {0,1}, s in {0..3}:
//     a0/a2 = word 4q+2p / 4q+2p+1 of row g  masked to slot s,
//     a1/a3 = the same words of row g+8,
//     b0/b1 = activation bytes 64q+32p+4s.. and 64q+32p+16+4s.. of token g.
// Masking slot s without shifting leaves the codes scaled by 4^s (at most
// 2*64 = 128, a valid u8), so each slot has its own accumulator and the four
// are combined exactly as acc0 + acc1/4 + acc2/16 + acc3/64.  Codes are
// c = W~ + 1; the epilogue subtracts the activation row sum.
//
// FUSED variant: the consumer warps first quantise the bf16 activations
// themselves (the routine of quant_common.cuh, same order as the stand-alone
// quantiser) into shared memory, so a whole decode BitLinear forward is one
// kernel.
//
// Dependent launch: every variant is launched as a programmatic dependent of
// the previous kernel in the stream.  Nothing produced earlier is read before
// griddepcontrol.wait, except the packed weights and gamma when the caller
// declared them static (not written by work still in flight): then the
// weight stream of this layer overlaps the tail of the previous one.
//
// BASE-3 variant (section 4 of the same page, "Memory Bandwidth and Latency
// Bounds": five ternary values per byte, 1.6 bits per weight).  Tiles of 16
// rows x 160 columns (512 bytes); lane (g, q) reads 8 bytes of rows g and
// g+8 (bytes 8 lane.. and 256 + 8 lane.., conflict-free) = two 20-column
// groups = columns 40q .. 40q+39 of the tile.  A byte b is expanded with
// packed half-precision arithmetic, exact for every b < 243: the halves
// v = 1024 + b (bit pattern 0x6400 | b) give the quotient by 3 as
// v' = RN(v * fp16(1/3) + 682.5) = 1024 + floor(b / 3) and the digit as
// e = v - 3 v' = d - 2048, whose low byte is -d as an int8.  Four bytes of a
// group thus yield, digit by digit, the s8 values -c of four consecutive
// columns -- an A-operand register of an s8 MMA whose activation fragment is
// eight consecutive code bytes.  The accumulator is -sum c x.
//
// 1-BIT variant (the W1 of the W1A4 regime on "The End of Matrix
// Multiplications: Welcome to Addition"; binary alphabet of [MF] section 1):
// tiles of 16 rows x 512 columns (1 KiB), word kw of a row holding columns
// 32 kw .. 32 kw + 31 with the bit c = (W~ + 1) / 2 of column 32 kw + 4 s + j
// at bit 8 j + s.  The lane reads the same 16-byte pieces as in the 2-bit
// tile; word & (0x01010101 << s) is four codes of four consecutive columns
// scaled by 2^s (one accumulator per slot, combined exactly), or, with two
// token groups, (word >> s) & 0x01010101 into a single accumulator.  The sum
// is sum c x, and W~ X~ = 2 sum c x - S.  The rescale divides by Q_b - 1 of
// the activation codes (127, or 7 for 4-bit codes).
//
// Balanced split.  Without a workspace a CTA owns a run of whole groups, so
// when the groups do not divide evenly over the resident CTAs (896 groups on
// 296 CTAs: three or four each) the kernel ends with the CTAs that own one
// more.  With a split workspace the (group, k-tile) units, group-major, are
// cut into equal contiguous shares, one per resident CTA; a CTA's first and
// last groups may then be shared with its neighbours ("segments" of
// k-tiles).  A shared group's int32 partial sums meet in the workspace:
// integer addition is exact, so the result does not depend on the split.
// Each output has one 64-bit workspace word that describes itself: the sum of
// the k-tile counts of the segments added so far (bits 45..63), their number
// (bits 36..44) and the sum of their partial sums each biased by 2^25 (bits
// 0..35; |partial| < 2 * 128 * 65536 < 2^25).  A segment adds
// (k << 45) + (1 << 36) + (v + 2^25) with one atomic; whoever completes the
// count to the group's k-tiles writes the output and zeroes the word.  No
// counter, no fence, no waiting: a word is never seen half-updated.  A CTA's
// first segment (shared with its left neighbour, which reaches that group
// last) adds early and checks the returned word only at the CTA's end; its
// last segment loads its words when it starts (the right neighbour has
// usually added its part by then) and finalises from them without a round
// trip, falling back to the atomic when they are not complete.

// Every mbarrier wait is bounded; on expiry the CTA stops consuming, the
// producer waits (bounded) for the copies it issued, and the error word is
// set.
#include <atomic>
#include <cstddef>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "bitlinear.h"
#include "common.cuh"
#include "decode_common.cuh"
#include "quant_common.cuh"

namespace bl {

constexpr int kDecWarps = 4;                          // consumer warps
constexpr int kDecThreads = (kDecWarps + 1) * 32;      // + one producer warp
constexpr int kDecMaxStages = 4;
static_assert(kDecWarps * 32 == kQuantThreads, "fused quantiser runs on the consumer warps");

struct DecodeArgs {
    const uint8_t *packed;   // 2-bit tiles (1 KiB) or base-3 tiles (512 B)
    const float *gamma;
    int d_out;
    int d_in;
    int kb_total;            // k-tiles per row: d_in / 256, ceil(d_in / 160) (base 3), ceil(d_in / 512) (1 bit)
    float qmax;              // Q_b - 1 of the activation codes: 127, or 7 for 4-bit codes
    int T;
    // product-only inputs (written by the stand-alone quantiser)
    const int8_t *Xq;
    const float *beta;
    const int32_t *rowsum;
    // fused inputs and the intermediates CTA 0 writes back
    const uint16_t *X;
    const float *gain;
    const float *inv_rms_in; // supplied per-token reciprocal RMS, or null
    int rmsnorm;
    float eps;
    float norm_eps;
    double inv_k;            // 1 / d_in
    int8_t *Xq_out;
    float *beta_out;
    int32_t *rowsum_out;
    // outputs
    void *Y;
    int32_t *acc_out;
    int static_weights;
    // Split workspace (see "Balanced split" above), or null: then every CTA
    // owns whole groups.  One 64-bit word per output, T * 16R per group; zero
    // before the launch, zero after it.
    unsigned long long *split_ws;
};

// The split workspace word's fields.
constexpr int kSplitKShift = 45;
constexpr int kSplitPartsShift = 36;
constexpr unsigned long long kSplitSumMask = (1ull << kSplitPartsShift) - 1;
constexpr long long kSplitBias = 1ll << 25;

__device__ __forceinline__ unsigned long long split_word(int k, int v) {
    return ((unsigned long long)k << kSplitKShift) + (1ull << kSplitPartsShift) +
           (unsigned long long)(v + kSplitBias);
}
__device__ __forceinline__ int split_k(unsigned long long w) { return (int)(w >> kSplitKShift); }
__device__ __forceinline__ int split_sum(unsigned long long w) {
    const long long parts = (long long)((w >> kSplitPartsShift) & 511u);
    return (int)((long long)(w & kSplitSumMask) - parts * kSplitBias);
}

struct DecodePlan {
    int ks;            // k-blocks per slab
    int nslab;         // slabs per row tile
    int stages;        // ring depth
    int stage_bytes;   // R * ks KiB of weights + T * ks * 256 B of codes (unfused)
    int xs_bytes;      // fused: T * K codes, rounded up to 128
};

__device__ __forceinline__ __half2 h2_bits(uint32_t u) {
    return *reinterpret_cast<const __half2 *>(&u);
}
__device__ __forceinline__ uint32_t h2_u32(__half2 h) {
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Four base-3 bytes (one 20-column group) -> d[i] = the int8 values -c of
// columns 4i .. 4i+3 of the group (byte j -> column 4i + j), i = 0..4.
__device__ __forceinline__ void base3_neg_codes(uint32_t w, uint32_t *d) {
    const __half2 third = h2_bits(0x35553555u);    // fp16(1/3) = 0.33325195
    const __half2 bias = h2_bits(0x61556155u);     // 682.5
    const __half2 minus3 = h2_bits(0xC200C200u);   // -3
    const __half2 m3072 = h2_bits(0xEA00EA00u);    // -3072
    __half2 ve = h2_bits(__byte_perm(w, 0x64646464u, 0x4240));   // 1024 + b0, 1024 + b2
    __half2 vo = h2_bits(__byte_perm(w, 0x64646464u, 0x4341));   // 1024 + b1, 1024 + b3
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 qe = __hfma2(ve, third, bias);   // 1024 + floor(v / 3)
        const __half2 qo = __hfma2(vo, third, bias);
        const uint32_t ee = h2_u32(__hfma2(qe, minus3, ve));   // digit - 2048
        const uint32_t eo = h2_u32(__hfma2(qo, minus3, vo));
        d[i] = __byte_perm(ee, eo, 0x6240);
        ve = qe;
        vo = qo;
    }
    d[4] = __byte_perm(h2_u32(__hadd2(ve, m3072)), h2_u32(__hadd2(vo, m3072)), 0x6240);
}

__device__ __forceinline__ void consumer_barrier() {
    asm volatile("bar.sync 2, %0;" ::"n"(kDecWarps * 32) : "memory");
}

// Resident CTAs per SM the register budget must allow: the one-tile-per-group
// variants run many small CTAs per SM, and a programmatic dependent's CTAs
// only overlap this grid's tail when both fit on the SM together.
template <int NT, int R, int FMT>
constexpr int dec_min_blocks() { return NT == 1 && R == 1 && FMT != kFmt1Bit ? 6 : 1; }

// SPLIT: the balanced split (a.split_ws non-null); otherwise whole groups.
template <int NT, int R, bool FUSED, bool OUT_BF16, int FMT, bool SPLIT>
__global__ void __launch_bounds__(kDecThreads, dec_min_blocks<NT, R, FMT>())
decode_kernel(const __grid_constant__ DecodeArgs a, DecodePlan plan, DeviceCtx ctx) {
    constexpr int TMAX = NT * 8;
    constexpr bool B3 = FMT == kFmtBase3;
    constexpr bool W1 = FMT == kFmt1Bit;
    constexpr int kTileBytes = B3 ? 512 : 1024;
    constexpr int kTileCols = B3 ? 160 : (W1 ? 512 : 256);
    // Accumulators per (row tile, token group): one per 2-bit slot, one per
    // 1-bit slot with a single token group, else one.
    constexpr bool kW1Shift = W1 && NT > 1;
    constexpr int kSlots = B3 ? 1 : (W1 ? (kW1Shift ? 1 : 8) : 4);
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ __align__(8) uint64_t full_bar[kDecMaxStages];
    __shared__ __align__(8) uint64_t empty_bar[kDecMaxStages];
    __shared__ __align__(8) uint64_t x_bar;   // fused: bf16 activations staged
    __shared__ QuantShared<FUSED ? TMAX : 1> qs;
    __shared__ int4 red[kDecWarps][R][NT][32];
    __shared__ float s_yscale[TMAX];
    __shared__ int s_rowsum[TMAX];
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = a.kb_total, K = a.d_in, T = a.T;
    const int n_rt = a.d_out >> 4;
    const int n_groups = (n_rt + R - 1) / R;
    const int ks = plan.ks, stages = plan.stages;
    const int stage_bytes = plan.stage_bytes;
    // This CTA's share of the (group, k-tile) units, group-major: a run of
    // whole groups, or with a split workspace an equal share of the units
    // (the first U mod P CTAs one unit more).  32-bit: U < 2^27.
    const int P = gridDim.x, c = blockIdx.x;
    int u0, u1;
    if (SPLIT) {
        const int U = n_groups * KB, q = U / P, rem = U - q * P;
        u0 = q * c + (c < rem ? c : rem);
        u1 = u0 + q + (c < rem ? 1 : 0);
    } else {
        const int q = n_groups / P, rem = n_groups - q * P;
        const int g0 = q * c + (c < rem ? c : rem);
        u0 = g0 * KB;
        u1 = (g0 + q + (c < rem ? 1 : 0)) * KB;
    }
    const int g_first = u0 / KB;
    const int nseg = u1 > u0 ? (u1 - 1) / KB - g_first + 1 : 0;
    // Segment s: k-tiles [seg_kb0(s), seg_kb1(s)) of group g_first + s.
    auto seg_kb0 = [&](int sg) {
        const int b = u0 - (g_first + sg) * KB;
        return b > 0 ? b : 0;
    };
    auto seg_kb1 = [&](int sg) {
        const int e = u1 - (g_first + sg) * KB;
        return e < KB ? e : KB;
    };
    // Ring units: slabs of up to ks k-tiles of one segment, in order.
    int units = 0;
    for (int sg = 0; sg < nseg; ++sg) units += (seg_kb1(sg) - seg_kb0(sg) + ks - 1) / ks;
    // Dynamic shared memory: [bf16 X (fused)] [codes (fused)] [stages].
    const int xb_bytes = FUSED ? ((T * K * 2 + 127) & ~127) : 0;
    uint16_t *xb = reinterpret_cast<uint16_t *>(dsm);
    int8_t *xs = reinterpret_cast<int8_t *>(dsm + xb_bytes);
    uint8_t *ring = dsm + xb_bytes + plan.xs_bytes;
    const uint32_t ring_s = smem_u32(ring);
    volatile int *abort_flag = &s_abort;

    if (threadIdx.x == 0) {
        for (int st = 0; st < stages; ++st) {
            mbar_init(smem_u32(&full_bar[st]), 1);
            mbar_init(smem_u32(&empty_bar[st]), kDecWarps);
        }
        mbar_init(smem_u32(&x_bar), 1);
        s_abort = 0;
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == kDecWarps) {
        // ------------------------------------------------------ producer ---
        if (lane == 0) {
            // Unit (sg, kb): k-tiles kb .. kb + nkb - 1 of segment sg.
            auto unit_kb = [&](int sg, int kb) { return seg_kb1(sg) - kb < ks ? seg_kb1(sg) - kb : ks; };
            auto next_unit = [&](int &sg, int &kb) {
                kb += ks;
                if (kb >= seg_kb1(sg)) {
                    ++sg;
                    kb = sg < nseg ? seg_kb0(sg) : 0;
                }
            };
            // Activation columns of a unit (the last base-3 tile may overhang d_in).
            auto unit_cols = [&](int sg, int kb) {
                const int c = unit_kb(sg, kb) * kTileCols, left = K - kb * kTileCols;
                return c < left ? c : left;
            };
            auto issue_w = [&](int sg, int kb, int st) {
                const uint32_t bar = smem_u32(&full_bar[st]);
                const int rt = (g_first + sg) * R;
                const int nkb = unit_kb(sg, kb);
                int nrow = 0;
                #pragma unroll
                for (int r = 0; r < R; ++r) nrow += rt + r < n_rt ? 1 : 0;
                const uint32_t xbytes = FUSED ? 0u : (uint32_t)(T * unit_cols(sg, kb));
                mbar_arrive_expect_tx(bar, (uint32_t)(nrow * nkb * kTileBytes) + xbytes);
                for (int r = 0; r < nrow; ++r)
                    bulk_g2s(ring_s + st * stage_bytes + r * ks * kTileBytes,
                             a.packed + ((size_t)(rt + r) * KB + (size_t)kb) * kTileBytes,
                             (uint32_t)(nkb * kTileBytes), bar);
            };
            auto issue_x = [&](int sg, int kb, int st) {
                if (FUSED) return;
                const uint32_t bar = smem_u32(&full_bar[st]);
                for (int t = 0; t < T; ++t)
                    bulk_g2s(ring_s + st * stage_bytes + R * ks * kTileBytes + t * ks * kTileCols,
                             a.Xq + (size_t)t * K + (size_t)kb * kTileCols,
                             (uint32_t)unit_cols(sg, kb), bar);
            };
            // With static weights the first unit's weights are requested
            // before the dependency wait.  Only the first: a CTA's whole ring
            // requested at once (by every CTA) arrives later as a whole, and
            // the copies issued after the wait (activations) queue behind it.
            const int first = units < 1 ? units : 1;
            if (a.static_weights) {
                int sg = 0, kb = nseg > 0 ? seg_kb0(0) : 0;
                for (int u = 0; u < first; ++u) {
                    issue_w(sg, kb, u);
                    next_unit(sg, kb);
                }
            }
            pdl_wait_primary();
            pdl_launch_dependents();
            if (FUSED) {
                // One bulk copy of the bf16 activations for the quantiser.
                const uint32_t xbar = smem_u32(&x_bar);
                mbar_arrive_expect_tx(xbar, (uint32_t)(T * K * 2));
                bulk_g2s(smem_u32(xb), a.X, (uint32_t)(T * K * 2), xbar);
            }
            int sg = 0, kb = nseg > 0 ? seg_kb0(0) : 0, st = 0, round = 0, issued = 0;
            for (int u = 0; u < units; ++u) {
                if (round > 0) {
                    // Stage st was last used by unit u - stages: wait for its
                    // release (completion number round - 1 of its barrier).
                    if (!dec_wait(smem_u32(&empty_bar[st]), (uint32_t)(round - 1) & 1u, ctx,
                                  abort_flag))
                        break;
                    issue_w(sg, kb, st);
                } else if (!a.static_weights || u >= first) {
                    issue_w(sg, kb, st);
                }
                issue_x(sg, kb, st);
                ++issued;
                next_unit(sg, kb);
                if (++st == stages) { st = 0; ++round; }
            }
            // Every copy issued must land before the CTA may exit.
            for (int u = issued > stages ? issued - stages : 0; u < issued; ++u)
                mbar_wait_bounded(smem_u32(&full_bar[u % stages]), (uint32_t)(u / stages) & 1u,
                                  ctx);
            if (FUSED) mbar_wait_bounded(smem_u32(&x_bar), 0, ctx);
        } else {
            pdl_wait_primary();
            pdl_launch_dependents();
        }
        return;
    }

    // ------------------------------------------------------- consumers ---
    // gamma belongs to the weights: with static weights it is read before the
    // dependency wait, hiding its latency.
    float gamma = 0.0f;
    if (a.static_weights) gamma = __ldg(a.gamma);
    pdl_wait_primary();
    pdl_launch_dependents();
    if (!a.static_weights) gamma = __ldg(a.gamma);
    const int g = lane >> 2, q = lane & 3;
    float in_beta = 0.0f;   // product only: beta[t] and rowsum[t] of token t = threadIdx.x
    int in_rowsum = 0;
    bool fast_quant = false;   // fused, no gain: codes made per warp, rowsum in the epilogue
    if constexpr (FUSED) {
        bool xok = dec_wait(smem_u32(&x_bar), 0, ctx, abort_flag);
        (void)xok;   // on expiry the codes are garbage and the error word is set
        if (a.gain == nullptr) {
            // Statistics in the canonical order, one barrier, then every
            // thread finalises them itself; each warp makes the codes of the
            // k-blocks it multiplies (kb = warp mod 4), so no barrier sits
            // between the codes and the MMAs.
            fast_quant = true;
            const bool rmsnorm = a.rmsnorm != 0;
            token_partials_smem<TMAX>(xb, T, K, rmsnorm && !a.inv_rms_in, qs);
            consumer_barrier();
            int sums[TMAX];
            #pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                sums[t] = 0;
                if (t < T) {
                    const TokenScale ts =
                        token_finalize<TMAX>(t, rmsnorm, a.eps, a.norm_eps, a.inv_k, a.qmax,
                                             a.inv_rms_in, qs);
                    if (threadIdx.x == 0) {
                        s_yscale[t] = __fdiv_rn(__fmul_rn(gamma, ts.beta), a.qmax);
                        if (blockIdx.x == 0 && a.beta_out) a.beta_out[t] = ts.beta;
                    }
                    const uint4 *xrow = reinterpret_cast<const uint4 *>(xb + (size_t)t * K);
                    uint2 *qrow = reinterpret_cast<uint2 *>(xs + (size_t)t * K);
                    for (int kb = warp; kb < (K >> 8); kb += kDecWarps) {
                        const int v = kb * 32 + lane;
                        qrow[v] = codes8(xrow[v], rmsnorm, ts.inv_rms, ts.scale, &sums[t]);
                    }
                }
            }
            #pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t < T) {
                    const int sum = warp_sum_i32(sums[t]);
                    if (lane == 0) qs.sum[warp][t] = sum;
                }
            }
            __syncwarp();
            // Base-3 and 1-bit tiles do not line up with the quantiser's
            // 256-column blocks: every warp needs every code.
            if constexpr (FMT != kFmt2Bit) consumer_barrier();
        } else {
            token_stats<TMAX, true>(xb, T, K, a.gain, a.rmsnorm != 0, a.eps, a.norm_eps,
                                    a.inv_k, a.qmax, a.inv_rms_in, qs);
            token_codes<TMAX, true>(xb, T, K, a.gain, a.rmsnorm != 0, xs, qs);
            if (threadIdx.x < T) {
                const int t = threadIdx.x;
                s_yscale[t] = __fdiv_rn(__fmul_rn(gamma, qs.beta[t]), a.qmax);
                s_rowsum[t] = qs.rowsum[t];
                if (blockIdx.x == 0) {
                    if (a.beta_out) a.beta_out[t] = qs.beta[t];
                    if (a.rowsum_out) a.rowsum_out[t] = qs.rowsum[t];
                }
            }
            if (blockIdx.x == 0 && a.Xq_out) {
                const uint4 *src = reinterpret_cast<const uint4 *>(xs);
                uint4 *dst = reinterpret_cast<uint4 *>(a.Xq_out);
                for (int v = threadIdx.x; v < (T * K) >> 4; v += kDecWarps * 32) dst[v] = src[v];
            }
            consumer_barrier();
        }
    } else if (threadIdx.x < T) {
        // Needed first by the first epilogue: loaded now, stored to shared
        // memory after the first segment's MMAs, so that the load's latency
        // (behind this CTA's weight stream) overlaps them.
        in_beta = a.beta[threadIdx.x];
        in_rowsum = a.rowsum[threadIdx.x];
    }

    // Fused: the CTAs hand back the intermediates once every warp's codes
    // are complete.  Every CTA holds the same codes, so they are written in
    // slices spread over the grid, and no single CTA lengthens it.
    auto hand_back = [&]() {
        if (blockIdx.x == 0 && threadIdx.x < T && a.rowsum_out) {
            int sum = 0;
            #pragma unroll
            for (int w = 0; w < kDecWarps; ++w) sum += qs.sum[w][threadIdx.x];
            a.rowsum_out[threadIdx.x] = sum;
        }
        if (a.Xq_out) {
            const uint4 *src = reinterpret_cast<const uint4 *>(xs);
            uint4 *dst = reinterpret_cast<uint4 *>(a.Xq_out);
            const int nv = (T * K) >> 4;
            for (int v = blockIdx.x * kDecWarps * 32 + threadIdx.x; v < nv;
                 v += gridDim.x * kDecWarps * 32)
                dst[v] = src[v];
        }
    };
    if (FUSED && fast_quant && nseg == 0) {   // a split share with no units
        consumer_barrier();
        hand_back();
    }

    bool ok = true;
    int st = 0;
    uint32_t fph = 0;
    constexpr int per_t = 16 * R;
    // Outputs of a segment per consumer thread: i = threadIdx.x + 128 j.
    constexpr int kEPT = (TMAX * per_t + kDecWarps * 32 - 1) / (kDecWarps * 32);
    // Output (token t, row tile r, row) of group grp from sum c x over all of K.
    auto emit = [&](int grp, int t, int r, int row, int v) {
        int rsum;
        if (FUSED && fast_quant) {
            rsum = 0;
            #pragma unroll
            for (int w = 0; w < kDecWarps; ++w) rsum += qs.sum[w][t];
        } else {
            rsum = s_rowsum[t];
        }
        // Offset codes: W~ = c - 1 (2-bit, base 3) or 2c - 1 (1 bit).
        const int accv = W1 ? 2 * v - rsum : v - rsum;
        const int o = (grp * R + r) * 16 + row;
        const size_t yi = (size_t)t * a.d_out + o;
        if (a.acc_out) a.acc_out[yi] = accv;
        const float y = __fmul_rn((float)accv, s_yscale[t]);
        if (OUT_BF16)
            reinterpret_cast<__nv_bfloat16 *>(a.Y)[yi] = __float2bfloat16_rn(y);
        else
            reinterpret_cast<float *>(a.Y)[yi] = y;
    };
    // Split: the words of the last segment and of a shared first segment,
    // loaded when the last segment starts.
    const bool first_shared = SPLIT && nseg > 1 && seg_kb0(0) > 0;
    unsigned long long pre_w[SPLIT ? kEPT : 1], first_w[SPLIT ? kEPT : 1];
    for (int sg = 0; sg < nseg; ++sg) {
        const int grp = g_first + sg;
        const int kb0 = seg_kb0(sg), kb1 = seg_kb1(sg);
        const bool part = SPLIT && (kb0 > 0 || kb1 < KB);   // shared with a neighbour
        const bool last_part = part && sg == nseg - 1;
        const int my_k = kb1 - kb0;
        unsigned long long *gws = SPLIT ? a.split_ws + (size_t)grp * T * per_t : nullptr;
        if constexpr (SPLIT) {
            if (sg == nseg - 1) {
                unsigned long long *gws0 = a.split_ws + (size_t)g_first * T * per_t;
                #pragma unroll
                for (int j = 0; j < kEPT; ++j) {
                    const int idx = threadIdx.x + kDecWarps * 32 * j;
                    const bool in = idx < T * per_t;
                    pre_w[j] = last_part && in ? ld_relaxed_gpu_u64(gws + idx) : 0ull;
                    first_w[j] = first_shared && in ? ld_relaxed_gpu_u64(gws0 + idx) : 0ull;
                }
            }
        }
        int acc[R][NT][kSlots][4];
        #pragma unroll
        for (int r = 0; r < R; ++r)
            #pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                #pragma unroll
                for (int s = 0; s < kSlots; ++s)
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) acc[r][nt][s][e] = 0;

        for (int kbs = kb0; kbs < kb1 && ok; kbs += ks) {
            ok = dec_wait(smem_u32(&full_bar[st]), fph, ctx, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            const uint8_t *stage = ring + st * stage_bytes;
            const int nkb = kb1 - kbs < ks ? kb1 - kbs : ks;
            // Warp w multiplies the k-tiles kb = w (mod 4) (those it quantised).
            const int kk0 = (warp - kbs) & (kDecWarps - 1);
            if constexpr (B3) {
                for (int kk = kk0; kk < nkb; kk += kDecWarps) {
                    // This lane's 40 columns of the tile: 40q .. 40q+39.
                    const int col0 = (kbs + kk) * 160 + 40 * q;
                    uint32_t dg[R][10], dh[R][10];   // rows g and g + 8
                    #pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint8_t *tile = stage + (r * ks + kk) * 512;
                        const uint2 lo = *reinterpret_cast<const uint2 *>(tile + lane * 8);
                        const uint2 hi = *reinterpret_cast<const uint2 *>(tile + 256 + lane * 8);
                        base3_neg_codes(lo.x, &dg[r][0]);
                        base3_neg_codes(lo.y, &dg[r][5]);
                        base3_neg_codes(hi.x, &dh[r][0]);
                        base3_neg_codes(hi.y, &dh[r][5]);
                    }
                    #pragma unroll
                    for (int m = 0; m < 5; ++m) {
                        const bool in_k = col0 + 8 * m < K;   // d_in is a multiple of 8
                        uint2 xr[NT];
                        #pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const int t = nt * 8 + g;
                            const uint8_t *xsrc =
                                FUSED ? reinterpret_cast<const uint8_t *>(xs) + (size_t)t * K +
                                            col0 + 8 * m
                                      : stage + R * ks * 512 + t * ks * 160 + kk * 160 + 40 * q +
                                            8 * m;
                            xr[nt] = make_uint2(0, 0);
                            if (t < T && in_k) xr[nt] = *reinterpret_cast<const uint2 *>(xsrc);
                        }
                        #pragma unroll
                        for (int r = 0; r < R; ++r)
                            #pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
                                mma_s8s8(acc[r][nt][0], dg[r][2 * m], dh[r][2 * m],
                                         dg[r][2 * m + 1], dh[r][2 * m + 1], xr[nt].x, xr[nt].y);
                    }
                }
            } else if constexpr (W1) {
                for (int kk = kk0; kk < nkb; kk += kDecWarps) {
                    // This lane's 128 columns of the tile: 128q .. 128q+127.
                    const int col0 = (kbs + kk) * 512 + 128 * q;
                    uint32_t w0[R][4], w1[R][4];   // words 4q..4q+3 of rows g and g + 8
                    #pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint8_t *tile = stage + (r * ks + kk) * 1024;
                        const uint4 lo = *reinterpret_cast<const uint4 *>(tile + lane * 16);
                        const uint4 hi = *reinterpret_cast<const uint4 *>(tile + 512 + lane * 16);
                        w0[r][0] = lo.x; w0[r][1] = lo.y; w0[r][2] = lo.z; w0[r][3] = lo.w;
                        w1[r][0] = hi.x; w1[r][1] = hi.y; w1[r][2] = hi.z; w1[r][3] = hi.w;
                    }
                    #pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        // Activation bytes of columns col0 + 64p .. +63 of each token.
                        uint32_t xr[NT][16];
                        #pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const int t = nt * 8 + g;
                            const uint8_t *xsrc =
                                FUSED ? reinterpret_cast<const uint8_t *>(xs) + (size_t)t * K +
                                            col0 + 64 * p
                                      : stage + R * ks * 1024 + t * ks * 512 + kk * 512 +
                                            128 * q + 64 * p;
                            #pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                uint4 x = make_uint4(0, 0, 0, 0);
                                if (t < T && col0 + 64 * p + 16 * v < K)   // d_in % 256 == 0
                                    x = *reinterpret_cast<const uint4 *>(xsrc + 16 * v);
                                xr[nt][4 * v + 0] = x.x;
                                xr[nt][4 * v + 1] = x.y;
                                xr[nt][4 * v + 2] = x.z;
                                xr[nt][4 * v + 3] = x.w;
                            }
                        }
                        #pragma unroll
                        for (int r = 0; r < R; ++r) {
                            #pragma unroll
                            for (int s = 0; s < 8; ++s) {
                                auto slot = [&](uint32_t w) {
                                    return kW1Shift ? (w >> s) & 0x01010101u
                                                    : w & (0x01010101u << s);
                                };
                                const uint32_t a0 = slot(w0[r][2 * p]), a2 = slot(w0[r][2 * p + 1]);
                                const uint32_t a1 = slot(w1[r][2 * p]), a3 = slot(w1[r][2 * p + 1]);
                                #pragma unroll
                                for (int nt = 0; nt < NT; ++nt)
                                    mma_u8s8(acc[r][nt][kW1Shift ? 0 : s], a0, a1, a2, a3,
                                             xr[nt][s], xr[nt][8 + s]);
                            }
                        }
                    }
                }
            } else
            for (int kk = kk0; kk < nkb; kk += kDecWarps) {
                uint32_t w0[R][4], w1[R][4];
                #pragma unroll
                for (int r = 0; r < R; ++r) {
                    const uint8_t *tile = stage + (r * ks + kk) * 1024;
                    const uint4 lo = *reinterpret_cast<const uint4 *>(tile + lane * 16);
                    const uint4 hi = *reinterpret_cast<const uint4 *>(tile + 512 + lane * 16);
                    w0[r][0] = lo.x; w0[r][1] = lo.y; w0[r][2] = lo.z; w0[r][3] = lo.w;
                    w1[r][0] = hi.x; w1[r][1] = hi.y; w1[r][2] = hi.z; w1[r][3] = hi.w;
                }
                uint32_t xr[NT][16];
                #pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int t = nt * 8 + g;
                    const uint8_t *xsrc =
                        FUSED ? reinterpret_cast<const uint8_t *>(xs) + (size_t)t * K +
                                    (size_t)(kbs + kk) * 256 + 64 * q
                              : stage + R * ks * 1024 + (t * ks + kk) * 256 + 64 * q;
                    #pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 x = make_uint4(0, 0, 0, 0);
                        if (t < T) x = *reinterpret_cast<const uint4 *>(xsrc + 16 * v);
                        xr[nt][4 * v + 0] = x.x;
                        xr[nt][4 * v + 1] = x.y;
                        xr[nt][4 * v + 2] = x.z;
                        xr[nt][4 * v + 3] = x.w;
                    }
                }
                #pragma unroll
                for (int r = 0; r < R; ++r) {
                    #pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        #pragma unroll
                        for (int s = 0; s < 4; ++s) {
                            const uint32_t m = 0x03030303u << (2 * s);
                            const uint32_t a0 = w0[r][2 * p] & m, a2 = w0[r][2 * p + 1] & m;
                            const uint32_t a1 = w1[r][2 * p] & m, a3 = w1[r][2 * p + 1] & m;
                            #pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
                                mma_u8s8(acc[r][nt][s], a0, a1, a2, a3, xr[nt][8 * p + s],
                                         xr[nt][8 * p + 4 + s]);
                        }
                    }
                }
            }
            // This warp is done with the stage.
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
            if (++st == stages) { st = 0; fph ^= 1u; }
        }

        #pragma unroll
        for (int r = 0; r < R; ++r)
            #pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                int c[4];
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if constexpr (B3) {
                        c[e] = -acc[r][nt][0][e];
                    } else if constexpr (W1) {
                        // Slot s summed c 2^s x; every term is a multiple of 2^s.
                        c[e] = acc[r][nt][0][e];
                        #pragma unroll
                        for (int s2 = 1; s2 < kSlots; ++s2) c[e] += acc[r][nt][s2][e] >> s2;
                    } else {
                        c[e] = acc[r][nt][0][e] + (acc[r][nt][1 % kSlots][e] >> 2) +
                               (acc[r][nt][2 % kSlots][e] >> 4) + (acc[r][nt][3 % kSlots][e] >> 6);
                    }
                }
                red[warp][r][nt][lane] = make_int4(c[0], c[1], c[2], c[3]);
            }
        if (!FUSED && sg == 0 && threadIdx.x < T) {
            s_yscale[threadIdx.x] = __fdiv_rn(__fmul_rn(gamma, in_beta), a.qmax);
            s_rowsum[threadIdx.x] = in_rowsum;
        }
        consumer_barrier();
        // Every warp's codes are complete (fused, after a barrier).
        if (FUSED && fast_quant && sg == 0) hand_back();

        // Epilogue of this segment: output i -> (token t, row tile r, row),
        // rows fastest, so consecutive threads store consecutive outputs.
        // v is sum c x over this segment's k-tiles.
        #pragma unroll
        for (int j = 0; j < kEPT; ++j) {
            const int idx = threadIdx.x + kDecWarps * 32 * j;
            if (idx >= T * per_t) break;
            const int t = idx / per_t, rem = idx - t * per_t;
            const int r = rem >> 4, row = rem & 15;
            if (grp * R + r >= n_rt) continue;
            const int gg = row & 7, half = row >> 3;
            const int nt = t >> 3, tt = t & 7;
            const int src_lane = gg * 4 + (tt >> 1);
            const int reg = (tt & 1) + 2 * half;
            int v = 0;
            #pragma unroll
            for (int w = 0; w < kDecWarps; ++w) {
                const int *e = reinterpret_cast<const int *>(&red[w][r][nt][src_lane]);
                v += e[reg];
            }
            if (!part) {
                emit(grp, t, r, row, v);
            } else if constexpr (SPLIT) {
                if (last_part) {
                    unsigned long long wd = pre_w[j];
                    if (split_k(wd) + my_k != KB)
                        wd = atomicAdd(gws + idx, split_word(my_k, v));   // not all in yet
                    if (split_k(wd) + my_k == KB) {
                        emit(grp, t, r, row, v + split_sum(wd));
                        gws[idx] = 0ull;
                    }
                } else {
                    atomicAdd(gws + idx, split_word(my_k, v));   // checked at the end
                }
            }
        }
        consumer_barrier();
    }
    if constexpr (SPLIT) {
        // A shared first segment (not also the last) added its part with no
        // look at the result; its words, loaded after that addition, show
        // whether it completed them (then this CTA writes those outputs: a
        // neighbour whose own addition completed them first may write the
        // same values too, which is harmless).
        if (first_shared) {
            unsigned long long *gws0 = a.split_ws + (size_t)g_first * T * per_t;
            #pragma unroll
            for (int j = 0; j < kEPT; ++j) {
                const int idx = threadIdx.x + kDecWarps * 32 * j;
                if (idx >= T * per_t) break;
                const int t = idx / per_t, rem = idx - t * per_t;
                const int r = rem >> 4, row = rem & 15;
                if (g_first * R + r >= n_rt) continue;
                if (split_k(first_w[j]) == KB) {
                    emit(g_first, t, r, row, split_sum(first_w[j]));
                    gws0[idx] = 0ull;
                }
            }
        }
    }
}

// Compile-time tuning knobs (defaults are the measured choices).
#ifndef BL_FUSED_MAX_CODE_BYTES
#define BL_FUSED_MAX_CODE_BYTES 32768   // largest T * d_in quantised inside the GEMV CTA
#endif
#ifndef BL_DEC_WIDE_ROW_TILES
#define BL_DEC_WIDE_ROW_TILES (148 * 8) // from this many 16-row tiles on, 2 tiles per group
#endif
#ifndef BL_DEC_STAGE_BYTES
#define BL_DEC_STAGE_BYTES 49152        // target bytes per pipeline stage
#endif
#ifndef BL_DEC_RING_BYTES
#define BL_DEC_RING_BYTES 98304         // bytes of all stages of a CTA
#endif
#ifndef BL_DEC_CTA_FRACTION
#define BL_DEC_CTA_FRACTION 1           // persistent grid = resident CTAs / this
#endif
#ifndef BL_DEC_MIN_GROUPS
#define BL_DEC_MIN_GROUPS 1             // at least this many groups per CTA
#endif
constexpr int kFusedMaxCodeBytes = BL_FUSED_MAX_CODE_BYTES;
constexpr int kSmemPerSm = 228 * 1024;      // shared memory of an SM
constexpr int kDecSmemReserve = 8 * 1024;   // per CTA: static shared memory + the 1 KiB reserve

// When a call that has a split workspace splits its units (see "Balanced
// split"): BITLINEAR_SPLIT_AUTO, _ALWAYS or _NEVER.
static std::atomic<int> g_split_mode{BITLINEAR_SPLIT_AUTO};

int decode_split_mode() { return g_split_mode.load(); }

// Which decode product kernel T <= 16 calls on 2-bit weights use:
// BITLINEAR_DECODE_AUTO, _WARP_MMA (mma.sync) or _TCGEN05.
static std::atomic<int> g_decode_kernel{BITLINEAR_DECODE_AUTO};

int set_decode_kernel(int mode) {
    if (mode != BITLINEAR_DECODE_AUTO && mode != BITLINEAR_DECODE_WARP_MMA &&
        mode != BITLINEAR_DECODE_TCGEN05)
        return BITLINEAR_ERR_INVALID_ARG;
    g_decode_kernel.store(mode);
    return BITLINEAR_OK;
}

bool decode_use_tc(int64_t T, int64_t d_out, int64_t d_in) {
    const int mode = g_decode_kernel.load();
    if (mode == BITLINEAR_DECODE_TCGEN05) return true;
    if (mode == BITLINEAR_DECODE_WARP_MMA) return false;
    (void)T;
    (void)d_out;
    (void)d_in;
    return false;
}

int set_decode_split_mode(int mode) {
    if (mode != BITLINEAR_SPLIT_AUTO && mode != BITLINEAR_SPLIT_ALWAYS &&
        mode != BITLINEAR_SPLIT_NEVER)
        return BITLINEAR_ERR_INVALID_ARG;
    g_split_mode.store(mode);
    return BITLINEAR_OK;
}

template <int NT, int R, bool FUSED, bool OUT_BF16, int FMT>
static cudaError_t prepare_decode_t(DecodeArgs args, const DeviceCtx &ctx, LaunchRec *rec) {
    constexpr int kTileBytes = FMT == kFmtBase3 ? 512 : 1024;
    constexpr int kTileCols = FMT == kFmtBase3 ? 160 : (FMT == kFmt1Bit ? 512 : 256);
    const int n_rt = args.d_out / 16;
    const int n_groups = (n_rt + R - 1) / R;
    const int KB = args.kb_total, K = args.d_in;
    DecodePlan plan;
    plan.xs_bytes = FUSED ? ((args.T * K + 127) & ~127) : 0;
    const int xb_bytes = FUSED ? ((args.T * K * 2 + 127) & ~127) : 0;
    // bytes per k-tile column of a stage
    const int per_kb = R * kTileBytes + (FUSED ? 0 : args.T * kTileCols);
    plan.ks = BL_DEC_STAGE_BYTES / per_kb;
    if (plan.ks > KB) plan.ks = KB;
    // With several slabs keep ks a multiple of the warp count, so that warp w
    // multiplies exactly the k-blocks kb = w (mod 4) (those it quantised).
    if (plan.ks < KB) plan.ks = plan.ks >= kDecWarps ? plan.ks - plan.ks % kDecWarps : kDecWarps;
    if (plan.ks > KB) plan.ks = KB;
    // Keep two CTAs per SM (eight MMA warps) where two stages of at least
    // four k-tiles still fit beside the activations: one CTA of four MMA warps
    // cannot keep up with the weight stream.
    int ring_bytes = BL_DEC_RING_BYTES;
    const int two_per_sm = kSmemPerSm / 2 - kDecSmemReserve - xb_bytes - plan.xs_bytes;
    if (two_per_sm < ring_bytes && two_per_sm >= 2 * kDecWarps * per_kb) {
        ring_bytes = two_per_sm;
        while (plan.ks > kDecWarps && 2 * plan.ks * per_kb > ring_bytes) plan.ks -= kDecWarps;
    }
    plan.nslab = (KB + plan.ks - 1) / plan.ks;
    plan.stage_bytes = plan.ks * per_kb;
    plan.stages = ring_bytes / plan.stage_bytes;
    if (plan.stages > kDecMaxStages) plan.stages = kDecMaxStages;
    // No deeper than the units a CTA can get when up to 8 CTAs fit per SM.
    const int min_units = ((n_groups + 148 * 8 - 1) / (148 * 8)) * plan.nslab;
    if (plan.stages > min_units) plan.stages = min_units;
    if (plan.stages < 2) plan.stages = 2;
    const size_t smem =
        (size_t)xb_bytes + (size_t)plan.xs_bytes + (size_t)plan.stages * plan.stage_bytes;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // Resident CTAs per SM of a kernel variant with this shared memory.
    auto prep = [&](const void *k, int *per_sm) {
        cudaError_t e = ensure_dynamic_smem(k, smem);
        if (e != cudaSuccess) return e;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, k, kDecThreads, smem) !=
                cudaSuccess || *per_sm < 1)
            *per_sm = 1;
        return cudaSuccess;
    };
    // Split the units evenly (one share per resident CTA) when whole groups
    // would not divide over the resident CTAs and every CTA still gets two
    // groups' worth of units, so that a CTA's last segment usually finds its
    // neighbour's part already added.
    const int mode = g_split_mode.load();
    bool split = false;
    int per_sm = 1;
    const void *kern = (const void *)decode_kernel<NT, R, FUSED, OUT_BF16, FMT, true>;
    if (args.split_ws && mode != BITLINEAR_SPLIT_NEVER) {
        cudaError_t e = prep(kern, &per_sm);
        if (e != cudaSuccess) return e;
        const int resident = sms * per_sm / BL_DEC_CTA_FRACTION;
        split = mode == BITLINEAR_SPLIT_ALWAYS ||
                (n_groups >= 2 * resident && n_groups % resident != 0);
    }
    int grid;
    if (split) {
        grid = sms * per_sm / BL_DEC_CTA_FRACTION;
    } else {
        args.split_ws = nullptr;
        kern = (const void *)decode_kernel<NT, R, FUSED, OUT_BF16, FMT, false>;
        cudaError_t e = prep(kern, &per_sm);
        if (e != cudaSuccess) return e;
        int max_ctas = sms * per_sm / BL_DEC_CTA_FRACTION;
        const int by_groups = (n_groups + BL_DEC_MIN_GROUPS - 1) / BL_DEC_MIN_GROUPS;
        if (max_ctas > by_groups) max_ctas = by_groups;
        if (max_ctas < sms) max_ctas = sms;
        grid = n_groups < max_ctas ? n_groups : max_ctas;
    }

    *rec = LaunchRec();
    rec->func = kern;
    rec->grid = dim3((unsigned)grid);
    rec->block = dim3(kDecThreads);
    rec->smem = smem;
    rec->pdl = true;
    rec->push(args);
    rec->push(plan);
    rec->push(ctx);
    return cudaSuccess;
}

template <bool FUSED, bool OUT_BF16, int FMT>
static cudaError_t prepare_decode_r(const DecodeArgs &args, const DeviceCtx &ctx,
                                    LaunchRec *rec) {
    // One row tile per group while that still leaves a few CTAs per SM;
    // larger matrices share each activation fragment over two row tiles.
    const int n_rt = args.d_out / 16;
    const bool wide = n_rt >= BL_DEC_WIDE_ROW_TILES;
    if (args.T <= 8)
        return wide ? prepare_decode_t<1, 2, FUSED, OUT_BF16, FMT>(args, ctx, rec)
                    : prepare_decode_t<1, 1, FUSED, OUT_BF16, FMT>(args, ctx, rec);
    if constexpr (FUSED) return cudaErrorInvalidValue;   // fused path is T <= 8 only
    return wide ? prepare_decode_t<2, 2, false, OUT_BF16, FMT>(args, ctx, rec)
                : prepare_decode_t<2, 1, false, OUT_BF16, FMT>(args, ctx, rec);
}

bool decode_can_fuse(int64_t T, int64_t d_in) {
    return T >= 1 && T <= 8 && T * d_in <= kFusedMaxCodeBytes;
}

template <int FMT>
static cudaError_t prepare_decode_f(const DecodeArgs &args, bool fused, bool bf,
                                    const DeviceCtx &ctx, LaunchRec *rec) {
    if (fused)
        return bf ? prepare_decode_r<true, true, FMT>(args, ctx, rec)
                  : prepare_decode_r<true, false, FMT>(args, ctx, rec);
    return bf ? prepare_decode_r<false, true, FMT>(args, ctx, rec)
              : prepare_decode_r<false, false, FMT>(args, ctx, rec);
}

// The decode kernel's launch for `args` (kernel choice, shared-memory plan,
// grid) as a launch record; its parameter 0 is the DecodeArgs, whose X field
// sits at decode_x_offset().
static bitlinear_status prepare_decode(DecodeArgs args, bool fused, int out_dtype, int fmt,
                                       LaunchRec *rec) {
    DeviceCtx ctx;
    bitlinear_status st = get_ctx(&ctx);
    if (st != BITLINEAR_OK) return st;
    const bool bf = out_dtype == BITLINEAR_OUT_BF16;
    cudaError_t e;
    if (fmt == kFmtBase3) {
        args.kb_total = (args.d_in + 159) / 160;
        e = prepare_decode_f<kFmtBase3>(args, fused, bf, ctx, rec);
    } else if (fmt == kFmt1Bit) {
        args.kb_total = (args.d_in + 511) / 512;
        e = prepare_decode_f<kFmt1Bit>(args, fused, bf, ctx, rec);
    } else {
        args.kb_total = args.d_in / 256;
        e = prepare_decode_f<kFmt2Bit>(args, fused, bf, ctx, rec);
    }
    return e == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

size_t decode_x_offset() { return offsetof(DecodeArgs, X); }

// Split workspace: one 64-bit word per token and row of 16 * (row tiles + 1)
// rows rounded up to a multiple of 128 (groups of two 16-row tiles may
// overhang d_out by one tile, the tensor-core kernel's 128-row blocks by up
// to 112 rows).
size_t decode_workspace_bytes(int64_t d_out, int64_t T) {
    if (T < 1 || T > 16 || d_out < 16) return 0;
    const size_t rows = ((size_t)16 * (size_t)(d_out / 16 + 1) + 127) & ~(size_t)127;
    const size_t bytes = 8 * rows * (size_t)T;
    return (bytes + 255) & ~(size_t)255;
}

static void set_split(DecodeArgs &a, void *ws) {
    if (!ws || a.T < 1 || a.T > 16) return;
    a.split_ws = static_cast<unsigned long long *>(ws);
}


bitlinear_status launch_decode(DecodeArgs args, bool fused, int out_dtype, int fmt,
                               cudaStream_t stream) {
    LaunchRec rec;
    bitlinear_status st = prepare_decode(args, fused, out_dtype, fmt, &rec);
    if (st != BITLINEAR_OK) return st;
    return rec.launch(stream) == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

static DecodeArgs gemv_args(const void *packed, const float *gamma, int64_t d_out,
                            int64_t d_in, const int8_t *Xq, const float *beta,
                            const int32_t *rowsum, int64_t T, void *Y, int32_t *acc_out,
                            bool static_weights, float qmax, void *ws) {
    DecodeArgs a = {};
    a.packed = static_cast<const uint8_t *>(packed);
    a.gamma = gamma;
    a.d_out = (int)d_out;
    a.d_in = (int)d_in;
    a.T = (int)T;
    a.Xq = Xq;
    a.beta = beta;
    a.rowsum = rowsum;
    a.Y = Y;
    a.acc_out = acc_out;
    a.static_weights = static_weights ? 1 : 0;
    a.qmax = qmax;
    set_split(a, ws);
    return a;
}

bitlinear_status launch_gemv(const void *packed, const float *gamma, int64_t d_out,
                             int64_t d_in, const int8_t *Xq, const float *beta,
                             const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                             int32_t *acc_out, bool static_weights, int fmt, float qmax,
                             void *ws, cudaStream_t stream) {
    return launch_decode(gemv_args(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y, acc_out,
                                   static_weights, qmax, ws),
                         false, out_dtype, fmt, stream);
}

bitlinear_status prepare_gemv(const void *packed, const float *gamma, int64_t d_out,
                              int64_t d_in, const int8_t *Xq, const float *beta,
                              const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                              int32_t *acc_out, bool static_weights, int fmt, float qmax,
                              void *ws, LaunchRec *rec) {
    return prepare_decode(gemv_args(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y, acc_out,
                                    static_weights, qmax, ws),
                          false, out_dtype, fmt, rec);
}

bitlinear_status prepare_linear_fused(const void *packed, const float *gamma, int64_t d_out,
                                      int64_t d_in, const uint16_t *X, int64_t T,
                                      const float *gain, bool rmsnorm, float eps,
                                      float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                      float *beta, int32_t *rowsum, void *Y, int out_dtype,
                                      bool static_weights, int fmt, float qmax, void *ws,
                                      LaunchRec *rec) {
    DecodeArgs a = {};
    a.inv_rms_in = inv_rms_in;
    a.packed = static_cast<const uint8_t *>(packed);
    a.gamma = gamma;
    a.d_out = (int)d_out;
    a.d_in = (int)d_in;
    a.T = (int)T;
    a.X = X;
    a.gain = gain;
    a.rmsnorm = rmsnorm ? 1 : 0;
    a.eps = eps;
    a.norm_eps = norm_eps;
    a.inv_k = 1.0 / (double)d_in;
    a.Xq_out = Xq;
    a.beta_out = beta;
    a.rowsum_out = rowsum;
    a.Y = Y;
    a.static_weights = static_weights ? 1 : 0;
    a.qmax = qmax;
    set_split(a, ws);
    return prepare_decode(a, true, out_dtype, fmt, rec);
}

bitlinear_status launch_linear_fused(const void *packed, const float *gamma, int64_t d_out,
                                     int64_t d_in, const uint16_t *X, int64_t T,
                                     const float *gain, bool rmsnorm, float eps, float norm_eps,
                                     const float *inv_rms_in, int8_t *Xq, float *beta,
                                     int32_t *rowsum, void *Y, int out_dtype,
                                     bool static_weights, int fmt, float qmax, void *ws,
                                     cudaStream_t stream) {
    LaunchRec rec;
    bitlinear_status st = prepare_linear_fused(packed, gamma, d_out, d_in, X, T, gain, rmsnorm,
                                               eps, norm_eps, inv_rms_in, Xq, beta, rowsum, Y,
                                               out_dtype, static_weights, fmt, qmax, ws, &rec);
    if (st != BITLINEAR_OK) return st;
    return rec.launch(stream) == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

}  // namespace bl
