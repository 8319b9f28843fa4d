/*
 * bitlinear.h -- C ABI of the B200 (sm_100a) BitNet b1.58 BitLinear library.
 *
 * The operation (cited as [MF]: "BitNet b1.58: Mathematical Foundations of
 * 1.58-Bit Ternary Quantization, Absmean Scaling, and Multiplication-Free LLM
 * Architectures", section 2 "Mathematical Formulation of the BitLinear b1.58
 * Layer", and section 6 "Implementation Considerations and Inference
 * Engines"):
 *
 *   gamma   = mean |W|                                   (absmean, per tensor)
 *   W~      = RoundClip(W / (gamma + eps), -1, 1)          in {-1, 0, +1}
 *   n       = RMSNorm(x) = x * r,  r = 1/sqrt(mean(x^2)+e) (optional, per token)
 *   beta_t  = max_k |n_tk|                                 (absmax, per token)
 *   X~      = RoundClip(n * 127 / (beta + eps), -127, 127) int8
 *   Y       = (X~ W~^T) * beta * gamma / 127               int32 accumulate
 *   RoundClip(z, a, b) = max(a, min(b, floor(z + 0.5)))
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers on the current CUDA device,
 *     owned by the caller; the library allocates nothing and keeps no
 *     pointer after the call returns (plans, below, are the exception: they
 *     keep the pointers they were given and own a small workspace).
 *   - All work is enqueued on `stream` (0 = legacy default stream); no entry
 *     point synchronises except bitlinear_device_error and
 *     bitlinear_get_last_device_error, and bitlinear_linear_plan_create,
 *     which waits for the zero fill of the plan's own workspace.
 *   - Per device the library remembers the address of its device error word
 *     and the shared-memory limits it has raised.  A device reset
 *     (cudaDeviceReset) in the process invalidates them: after one, the
 *     library must not be used on that device again (plans made before it
 *     included).  bitlinear_pack_weights_noalloc alone looks its address up
 *     again.
 *   - Shapes: d_out (output features, N) is a positive multiple of 16,
 *     d_in (input features, K) a positive multiple of 256 and at most 65536,
 *     T (tokens) is 0 .. 1048576.  T = 0 is a no-op that returns
 *     BITLINEAR_OK and enqueues nothing.
 *   - Alignment: W, X, Xq, packed and Y must be 16-byte aligned; gamma, beta,
 *     rowsum, rms and gain 4-byte aligned.
 *   - Errors: arguments are validated on the host before anything is
 *     enqueued; a failed validation returns a status and enqueues nothing.
 *     A failed launch returns BITLINEAR_ERR_CUDA.  A kernel that gives up a
 *     bounded wait records BITLINEAR_ERR_TIMEOUT in a device error word read
 *     by bitlinear_device_error.  No entry point aborts, traps or throws.
 *   - There is no CPU fallback: without an sm_100 device every compute call
 *     returns BITLINEAR_ERR_DEVICE.
 *
 * Packed ternary weight layout (this library's own format; [MF] section 6
 * names "packed 2-bit" ternary registers without fixing an order): the
 * d_out x d_in matrix W~ is cut into tiles of 16 rows x 256 columns stored
 * tile-row-major (tile (rb, kb) at index rb * (d_in/256) + kb, 1 KiB each);
 * inside a tile the 16 rows follow one another, each as 16 little-endian
 * uint32 words; word kw of a row holds columns 16*kw .. 16*kw+15, and the
 * 2-bit code c = W~ + 1 (0, 1 or 2; 3 never occurs) of column 16*kw + 4*s + j
 * sits at bits 8*j + 2*s.  Thus (word >> 2s) & 0x03030303 is four int8 codes
 * of four consecutive columns.  Size: d_out * d_in / 4 bytes.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BITLINEAR_OK = 0,
    BITLINEAR_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, bad eps */
    BITLINEAR_ERR_MISALIGNED = 2,        /* pointer alignment rule broken    */
    BITLINEAR_ERR_UNSUPPORTED_SHAPE = 3, /* shape outside the rules above    */
    BITLINEAR_ERR_CUDA = 4,              /* a CUDA runtime call failed       */
    BITLINEAR_ERR_TIMEOUT = 5,           /* a device-side bounded wait expired */
    BITLINEAR_ERR_DEVICE = 6             /* no usable sm_100 device          */
} bitlinear_status;

/* Output element types of bitlinear_forward. */
#define BITLINEAR_OUT_F32 0
#define BITLINEAR_OUT_BF16 1

/* Flags of bitlinear_quant_act and bitlinear_linear. */
#define BITLINEAR_RMSNORM 1u
/* bitlinear_linear only: the caller guarantees that no work still in flight
 * on the stream writes `packed` or `gamma`, so the product kernel may start
 * reading them before earlier work completes (decode layers with fixed
 * weights: the next layer's weight stream overlaps the current layer). */
#define BITLINEAR_STATIC_WEIGHTS 2u
/* bitlinear_quant_act and bitlinear_linear: one beta for the whole X -- the
 * largest absmax over all tokens ([MF] section 2 prints beta as the max over
 * all i, j and allows this scope) -- instead of one per token.  beta[t] then
 * holds that one value for every t.  Three launches (statistics, max,
 * codes); bitlinear_linear never fuses the quantiser into the product in
 * this mode. */
#define BITLINEAR_PER_TENSOR_ABSMAX 4u

/* Flag of bitlinear_quant_act and bitlinear_linear_w1: 4-bit activation codes,
 * the A4 of the W1A4 regime ("The End of Matrix Multiplications: Welcome to
 * Addition", Technical Details).  [MF] section 2 defines Q_b = 2^(k-1) for
 * k-bit activations; with k = 4 the multiplier and the clip bound are
 * Q_b - 1 = 7, codes in [-7, 7] (still stored one per int8). */
#define BITLINEAR_ACT_4BIT 8u

/* Library ABI version (this header: 3). */
int bitlinear_version(void);

/* Static description of a status code.  Never NULL. */
const char *bitlinear_status_string(int status);

/* Number of uint32 words of a packed d_out x d_in matrix (d_out*d_in/16),
 * or 0 when the shape breaks the rules above. */
size_t bitlinear_packed_words(int64_t d_out, int64_t d_in);

/* The same size in bytes (4 x bitlinear_packed_words: 0.25 byte per weight,
 * [MF] section 6's 2-bit code); 0 when the shape breaks the rules above. */
size_t bitlinear_packed_bytes(int64_t d_out, int64_t d_in);

/* Bytes of device scratch bitlinear_pack_weights needs when it computes gamma
 * itself (gamma_in == NULL); 0 when the shape breaks the rules above. */
size_t bitlinear_pack_workspace_bytes(int64_t d_out, int64_t d_in);

/*
 * bitlinear_pack_weights -- absmean ternarisation and 2-bit packing
 * ([MF] section 2, "Weight Quantization: Absmean Scaling").
 *
 *   W          fp32 [d_out][d_in], row-major, latent weights.
 *   eps        the epsilon of W / (gamma + eps); must be finite and >= 0.
 *   gamma_in   device fp32 scalar, or NULL.  When given it is used as gamma
 *              and no reduction runs; when NULL gamma = mean|W| is computed
 *              (sum of |W| in double over a fixed, deterministic two-stage
 *              reduction, divided by d_out*d_in and rounded once to fp32).
 *   workspace  device scratch of bitlinear_pack_workspace_bytes() bytes,
 *              8-byte aligned; needed only when gamma_in == NULL.
 *   packed     out: bitlinear_packed_words() uint32 words, layout above.
 *   gamma_out  out: device fp32 scalar, the gamma used (may equal gamma_in).
 * W / (gamma + eps) is one binary32 division; floor(z + 0.5) is then taken
 * exactly and clipped to [-1, 1].  NaN or infinite weights give unspecified
 * codes (never code 3).
 */
int bitlinear_pack_weights(const float *W, int64_t d_out, int64_t d_in, float eps,
                           const float *gamma_in, void *workspace,
                           size_t workspace_bytes, uint32_t *packed,
                           float *gamma_out, cudaStream_t stream);

/*
 * bitlinear_pack_weights_noalloc -- bitlinear_pack_weights with gamma
 * computed, for callers that cannot allocate device memory.  The pages have
 * no counterpart: this entry exists for callers such as code that packs
 * weights while a stream is being captured into a CUDA graph (where
 * cudaMalloc is not allowed), runtimes whose device memory is entirely
 * reserved up front by their own pool, or hosts with no device allocator
 * they may call -- none of which can supply the workspace that
 * bitlinear_pack_weights needs for its partial sums of |W|.
 *
 * Same arguments and results as bitlinear_pack_weights(W, d_out, d_in, eps,
 * NULL, workspace, ..., packed, gamma_out, stream); gamma is bit-identical.
 * The partial sums live instead in one fixed array inside the library of
 * 1184 doubles (9,472 bytes), held in the memory of every GPU that loads
 * the library until the process exits.  The reduction grid is capped at
 * 1184 blocks, so every shape the rules above accept fits; shapes they
 * reject return BITLINEAR_ERR_UNSUPPORTED_SHAPE as in bitlinear_pack_weights.
 * Calls no allocator (no cudaMalloc, cudaFree or allocating library
 * routine).  Every call made outside stream capture looks up the array's
 * device address (cudaGetSymbolAddress) with the current device, so a
 * device reset between calls is harmless; a call made during a capture uses
 * the address found by the last such call on that device, and fails with
 * BITLINEAR_ERR_CUDA if there was none: make one call on each device before
 * capturing, and again after any device reset.  All calls share the one
 * array, which keeps the last call's contents (every partial read is first
 * written by the same call, so nothing needs clearing): calls that overlap
 * on the GPU -- on different streams, or on different host threads -- race
 * and must be serialised by the caller.
 */
int bitlinear_pack_weights_noalloc(const float *W, int64_t d_out, int64_t d_in,
                                   float eps, uint32_t *packed, float *gamma_out,
                                   cudaStream_t stream);

/*
 * bitlinear_quant_act -- fused RMSNorm + per-token absmax int8 quantisation
 * ([MF] section 2, "Activation Quantization: Absmax Scaling"; beta taken per
 * token; Q_b - 1 = 127 is both multiplier and clip bound).
 *
 *   X          bf16 [T][d_in], row-major, as raw uint16 bit patterns.
 *   norm_gain  fp32 [d_in] RMSNorm gain, or NULL for all ones.
 *   flags      BITLINEAR_RMSNORM to normalise first, 0 to quantise X as is;
 *              BITLINEAR_PER_TENSOR_ABSMAX for one beta over all of X;
 *              BITLINEAR_ACT_4BIT for 4-bit codes (multiplier and clip 7
 *              instead of 127).
 *   eps        the epsilon of 127 / (beta + eps); finite, >= 0.
 *   norm_eps   the epsilon inside the RMS; finite, >= 0.  The reciprocal RMS
 *              r = 1 / sqrt(mean(x^2) + norm_eps): sum of squares in double in
 *              a fixed order, reciprocal square root refined in double to
 *              ~1e-13 relative, rounded to fp32 (within 1e-6 relative of the
 *              correctly rounded value; identical in every path of this
 *              library).
 *   inv_rms_in fp32 [T] per-token r to use instead of computing it, or NULL.
 *   Xq         out: int8 [T][d_in] activation codes in [-127, 127].
 *   beta       out: fp32 [T] per-token absmax of the (normalised) row.
 *   rowsum     out: int32 [T] sum of each row of Xq (consumed by forward).
 *   inv_rms_out out: fp32 [T] r used, or NULL.
 * n = x * r is one binary32 multiplication (times the gain, one more); the
 * scale 127 / (beta + eps) is one binary32 addition and one division,
 * applied with one multiplication; floor(v + 0.5) is then taken exactly.
 */
int bitlinear_quant_act(const uint16_t *X, int64_t T, int64_t d_in,
                        const float *norm_gain, uint32_t flags, float eps,
                        float norm_eps, const float *inv_rms_in, int8_t *Xq,
                        float *beta, int32_t *rowsum, float *inv_rms_out,
                        cudaStream_t stream);

/*
 * bitlinear_forward -- the multiplier-free ternary x int8 product with int32
 * accumulation and the fused rescale ([MF] section 2, "The Linear
 * Transformation and Rescaling"; section 6, scale-factor fusion):
 *
 *   acc[t][o] = sum_k W~[o][k] * Xq[t][k]                 exact int32
 *   Y[t][o]   = acc[t][o] * (gamma * beta[t] / 127)        one fp32 multiply
 *
 * with gamma * beta[t] / 127 formed as one binary32 multiplication and one
 * division.  The kernels multiply the offset codes c = W~ + 1 and subtract
 * rowsum[t]; the result is the same exact integer.
 *
 *   packed     packed ternary weights (layout above), d_out x d_in.
 *   gamma      device fp32 scalar.
 *   Xq, beta, rowsum   as written by bitlinear_quant_act for these T rows.
 *   Y          out: [T][d_out] row-major, fp32 or bf16 (round to nearest even)
 *              per out_dtype.
 *   acc_out    out: int32 [T][d_out] raw accumulators, or NULL.
 * T <= 16 runs the decode GEMV (register-decoded ternary weights, warp-level
 * int8 tensor-core MMA); T > 16 runs the prefill GEMM (TMA-staged packed
 * tiles expanded in shared memory, tcgen05 int8 MMA on clusters of two CTAs,
 * TMEM accumulators).  The prefill GEMM launches clusters of two CTAs of
 * about 215 KiB of shared memory each, one pair per two SMs.
 *
 * workspace, workspace_bytes: optional (NULL, 0) split workspace of the
 * decode product (T <= 16), caller-owned: at least
 * bitlinear_decode_workspace_bytes(d_out, T) bytes (else
 * BITLINEAR_ERR_INVALID_ARG), 16-byte aligned, zero-filled before its first
 * use.  Every call that runs to completion leaves it zero again, so one
 * workspace serves any sequence of calls on one stream; calls that may
 * overlap on the GPU need workspaces of their own.  With it, a matrix whose
 * 16-row tiles do not divide evenly over the resident CTAs has its
 * (rows, k-tile) units split evenly instead, the CTAs sharing a row tile
 * adding exact int32 partial sums (the results are the same integers).
 * Ignored for T > 16.
 */
int bitlinear_forward(const uint32_t *packed, const float *gamma, int64_t d_out,
                      int64_t d_in, const int8_t *Xq, const float *beta,
                      const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                      int32_t *acc_out, void *workspace, size_t workspace_bytes,
                      cudaStream_t stream);

/* Bytes of the split workspace of a decode product with d_out outputs and T
 * tokens (1 <= T <= 16), or 0 for other T or an unsupported d_out:
 * 8 * T * R with R = 16 * (d_out / 16 + 1) rounded up to a multiple of 128,
 * the total rounded up to a multiple of 256. */
size_t bitlinear_decode_workspace_bytes(int64_t d_out, int64_t T);

/* When decode calls given a split workspace split their units (process-wide;
 * calls and plans made afterwards follow it): BITLINEAR_SPLIT_AUTO (default:
 * when the 16-row tiles do not divide evenly over the resident CTAs and each
 * CTA gets at least two tiles' worth), BITLINEAR_SPLIT_ALWAYS (every decode
 * call with a workspace, whatever its size: for tests), BITLINEAR_SPLIT_NEVER.
 * The results are the same integers in every mode.  Returns
 * BITLINEAR_ERR_INVALID_ARG for another value. */
#define BITLINEAR_SPLIT_AUTO 0
#define BITLINEAR_SPLIT_ALWAYS 1
#define BITLINEAR_SPLIT_NEVER 2
int bitlinear_set_decode_split(int mode);

/* Which product kernel decode calls (T <= 16) on 2-bit weights use
 * (process-wide; calls and plans made afterwards follow it):
 * BITLINEAR_DECODE_AUTO (default: by shape and T), BITLINEAR_DECODE_WARP_MMA
 * (warp-level mma.sync on codes decoded in registers; the only one with the
 * one-kernel quantise-and-multiply path) or BITLINEAR_DECODE_TCGEN05 (codes
 * written to tensor memory, tcgen05.mma of 128 weight rows x 16 token slots;
 * bitlinear_linear then runs the quantiser first).  The results are the same
 * integers with every kernel.  Returns BITLINEAR_ERR_INVALID_ARG for another
 * value. */
#define BITLINEAR_DECODE_AUTO 0
#define BITLINEAR_DECODE_WARP_MMA 1
#define BITLINEAR_DECODE_TCGEN05 2
int bitlinear_set_decode_kernel(int mode);

/*
 * bitlinear_linear -- the whole BitLinear forward from bf16 activations:
 * bitlinear_quant_act followed by bitlinear_forward, with the same arguments,
 * meaning and results (bit for bit) as those two calls made back to back
 * ([MF] section 2, all three parts).  flags: BITLINEAR_RMSNORM,
 * BITLINEAR_STATIC_WEIGHTS, BITLINEAR_PER_TENSOR_ABSMAX.  inv_rms_in: fp32
 * [T] per-token reciprocal RMS to use instead of computing it, or NULL (as in
 * bitlinear_quant_act).  Xq, beta and rowsum are caller-owned intermediates
 * of T*d_in, T and T elements, written with the codes, absmax and row sums.
 * For T <= 8 with T*d_in <= 32768 one kernel quantises (in shared memory,
 * per CTA) and multiplies; otherwise the quantiser runs first and the
 * product kernel is its programmatic dependent.  Kernels are launched as
 * programmatic dependents of the work before them and read nothing earlier
 * work produces before their dependency wait, except the weights under
 * BITLINEAR_STATIC_WEIGHTS.  workspace, workspace_bytes: the optional split
 * workspace, as in bitlinear_forward.
 */
int bitlinear_linear(const uint32_t *packed, const float *gamma, int64_t d_out,
                     int64_t d_in, const uint16_t *X, int64_t T,
                     const float *norm_gain, uint32_t flags, float eps,
                     float norm_eps, const float *inv_rms_in, int8_t *Xq,
                     float *beta, int32_t *rowsum, void *Y, int out_dtype,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Plans: a bitlinear_linear call bound once.  For a serving loop that calls
 * the same layer again and again with new activations ([MF] section 6: the
 * per-call work -- here argument checks, kernel selection, launch shapes and,
 * for T > 16, the prefill GEMM's tensor-map descriptors -- is done once).
 *
 * bitlinear_linear_plan_create validates the arguments (every argument of
 * bitlinear_linear except X, inv_rms_in, which a plan does not take, and the
 * stream; same rules and errors), checks the device, prepares the launches
 * and returns a plan in *plan (NULL on error).  The plan is a small host
 * object owned by the caller; it keeps the pointers it was given, which must
 * stay valid while it is used, and, for 1 <= T <= 16, owns a split
 * workspace in device memory (bitlinear_decode_workspace_bytes(d_out, T)
 * bytes, used when its decode product splits its units, see
 * bitlinear_forward).  The workspace is zero-filled before plan_create
 * returns (it waits for that fill alone), so a first run on any stream finds
 * it ready; BITLINEAR_ERR_CUDA if it cannot be allocated or filled.  As it
 * allocates device memory, plan_create may not be called while a stream
 * capture is in progress.
 * flags: BITLINEAR_RMSNORM, BITLINEAR_STATIC_WEIGHTS,
 * BITLINEAR_PER_TENSOR_ABSMAX (2-bit weights only, as bitlinear_linear).
 *
 * bitlinear_linear_plan_run enqueues on `stream` exactly what
 * bitlinear_linear(..., X, ...) with the bound arguments would (the same
 * kernels and results, bit for bit).  X: bf16 [T][d_in], 16-byte aligned.
 * The device current at creation must be current; otherwise
 * BITLINEAR_ERR_DEVICE.  Runs of one plan may be enqueued on any streams;
 * runs that overlap on the GPU share the plan's output buffers and its
 * workspace, as two bitlinear_linear calls on the same buffers would, and
 * must not.  A run may be captured into a CUDA graph.
 *
 * bitlinear_plan_destroy frees the plan and its workspace (NULL is allowed);
 * no run of it may still be in flight.
 */
typedef struct bitlinear_plan bitlinear_plan;
int bitlinear_linear_plan_create(const uint32_t *packed, const float *gamma, int64_t d_out,
                                 int64_t d_in, int64_t T, const float *norm_gain,
                                 uint32_t flags, float eps, float norm_eps, int8_t *Xq,
                                 float *beta, int32_t *rowsum, void *Y, int out_dtype,
                                 bitlinear_plan **plan);
int bitlinear_linear_plan_run(const bitlinear_plan *plan, const uint16_t *X,
                              cudaStream_t stream);
void bitlinear_plan_destroy(bitlinear_plan *plan);

/*
 * Base-3 weight format ([MF] section 4, "Memory Bandwidth and Latency
 * Bounds": five ternary values fit in one byte, 3^5 = 243 < 256, so a weight
 * costs 1.6 bits instead of 2).  This library's own order: each row is padded
 * with W~ = 0 to Kp = 160 * ceil(d_in / 160) columns; the matrix is cut into
 * tiles of 16 rows x 160 columns (512 bytes) stored tile-row-major (tile
 * (rb, kb) at byte 512 * (rb * Kp/160 + kb)); inside a tile the 16 rows follow
 * one another as 32 bytes each; byte B of a tile row belongs to the
 * 20-column group g = B / 4 and, with j = B % 4, holds the codes
 * c_i = W~ + 1 of columns 20*g + 4*i + j (i = 0..4) as the base-3 number
 * c_0 + 3 c_1 + 9 c_2 + 27 c_3 + 81 c_4 (never above 242).  Four bytes of a
 * group thus give, digit by digit, the codes of four consecutive columns.
 * Size: d_out * Kp / 5 bytes.  Decode-only: the entry points below take
 * 1 <= T <= 16.
 */

/* Bytes of the base-3 format for d_out x d_in, or 0 if the shape is
 * unsupported (same shape rules as the 2-bit format). */
size_t bitlinear_base3_bytes(int64_t d_out, int64_t d_in);

/*
 * bitlinear_repack_base3 -- convert 2-bit packed weights (as written by
 * bitlinear_pack_weights) into the base-3 format, exactly.
 *   packed   in: 2-bit layout, d_out x d_in, 16-byte aligned.
 *   packed3  out: bitlinear_base3_bytes(d_out, d_in) bytes, 16-byte aligned.
 * gamma is unchanged and shared by both formats.
 */
int bitlinear_repack_base3(const uint32_t *packed, int64_t d_out, int64_t d_in,
                           uint8_t *packed3, cudaStream_t stream);

/*
 * bitlinear_forward_base3 -- bitlinear_forward on base-3 weights: the same
 * arguments, meaning and results (the int32 accumulators are the same exact
 * integers), for 1 <= T <= 16 (otherwise BITLINEAR_ERR_UNSUPPORTED_SHAPE;
 * T = 0 is a no-op).  The decode kernel expands each byte to its five codes
 * in registers and multiplies them on the warp-level int8 tensor-core MMA.
 */
int bitlinear_forward_base3(const uint8_t *packed3, const float *gamma, int64_t d_out,
                            int64_t d_in, const int8_t *Xq, const float *beta,
                            const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                            int32_t *acc_out, void *workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/*
 * bitlinear_linear_base3 -- bitlinear_linear on base-3 weights (same
 * arguments, flags and results), for 1 <= T <= 16.  BITLINEAR_PER_TENSOR_ABSMAX
 * runs the quantiser first, as in bitlinear_linear.
 */
int bitlinear_linear_base3(const uint8_t *packed3, const float *gamma, int64_t d_out,
                           int64_t d_in, const uint16_t *X, int64_t T,
                           const float *norm_gain, uint32_t flags, float eps,
                           float norm_eps, const float *inv_rms_in, int8_t *Xq,
                           float *beta, int32_t *rowsum, void *Y, int out_dtype,
                           void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * W1A4: binary weights with 4-bit activations, the regime "The End of Matrix
 * Multiplications: Welcome to Addition" names (Technical Details).  The pages
 * give no binarisation rule; this library takes the binary alphabet
 * {-1, +1} of [MF] section 1 as W~ = +1 where W >= 0 and -1 elsewhere, with
 * the same absmean gamma as scale (the least-squares scale of a sign code),
 * and the A4 codes of BITLINEAR_ACT_4BIT:
 *
 *   Y = (X~ W~^T) * beta * gamma / (Q_b - 1),  Q_b - 1 = 7 (4-bit) or 127
 *
 * 1-bit weight format (this library's own): rows padded with W~ = -1 to a
 * multiple of 512 columns; tiles of 16 rows x 512 columns (1 KiB) stored
 * tile-row-major (tile (rb, kb) at byte 1024 * (rb * ceil(d_in/512) + kb));
 * each tile row is 16 little-endian uint32 words; word kw covers columns
 * 32 kw .. 32 kw + 31 and the bit c = (W~ + 1) / 2 of column 32 kw + 4 s + j
 * sits at bit 8 j + s.  Size: d_out * ceil(d_in / 512) * 64 bytes (one bit
 * per weight).  Decode only: the product takes 1 <= T <= 16.
 */

/* Bytes of the 1-bit format for d_out x d_in, or 0 for an unsupported shape. */
size_t bitlinear_w1_packed_bytes(int64_t d_out, int64_t d_in);

/*
 * bitlinear_pack_weights_w1 -- binarise and pack fp32 latent weights.
 *   W, gamma_in, workspace, workspace_bytes, gamma_out: as in
 *   bitlinear_pack_weights (gamma = mean |W| unless gamma_in is given; it
 *   scales the outputs and does not enter the codes).
 *   packed1   out: bitlinear_w1_packed_bytes(d_out, d_in) bytes, 16-byte aligned.
 */
int bitlinear_pack_weights_w1(const float *W, int64_t d_out, int64_t d_in,
                              const float *gamma_in, void *workspace, size_t workspace_bytes,
                              uint32_t *packed1, float *gamma_out, cudaStream_t stream);

/*
 * bitlinear_forward_w1 -- the product on 1-bit weights with the fused
 * rescale: acc[t][o] = sum_k W~[o][k] Xq[t][k] exactly in int32 (the kernel
 * multiplies the bits c = (W~ + 1) / 2 and forms 2 sum c x - rowsum[t]),
 * Y = acc * (gamma * beta[t] / (2^(act_bits-1) - 1)).  act_bits is 4 or 8 and
 * must be the width the codes were made with (bitlinear_quant_act, with or
 * without BITLINEAR_ACT_4BIT).  1 <= T <= 16; other arguments as in
 * bitlinear_forward.
 */
int bitlinear_forward_w1(const uint32_t *packed1, const float *gamma, int64_t d_out,
                         int64_t d_in, const int8_t *Xq, const float *beta,
                         const int32_t *rowsum, int64_t T, int act_bits, void *Y, int out_dtype,
                         int32_t *acc_out, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/*
 * bitlinear_linear_w1 -- bitlinear_linear on 1-bit weights: quantise (with
 * BITLINEAR_ACT_4BIT: 4-bit codes, the W1A4 forward), then the product; one
 * kernel for T <= 8 with T * d_in <= 32768.  flags: BITLINEAR_RMSNORM,
 * BITLINEAR_STATIC_WEIGHTS, BITLINEAR_PER_TENSOR_ABSMAX, BITLINEAR_ACT_4BIT.
 * 1 <= T <= 16.
 */
int bitlinear_linear_w1(const uint32_t *packed1, const float *gamma, int64_t d_out,
                        int64_t d_in, const uint16_t *X, int64_t T, const float *norm_gain,
                        uint32_t flags, float eps, float norm_eps, const float *inv_rms_in,
                        int8_t *Xq, float *beta, int32_t *rowsum, void *Y, int out_dtype,
                        void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * bitlinear_dense_bf16_forward -- the dense bf16 linear layer Y = X W^T that
 * BitLinear replaces, kept as the context the measurements compare against
 * ([MF] section 2, "The Linear Transformation and Rescaling", without the
 * quantisers; section 4, "Memory Bandwidth and Latency Bounds": 2 bytes per
 * weight instead of 0.25).  Not a step of the method.
 *
 *   W          bf16 [d_out][d_in], row-major, 16-byte aligned.
 *   X          bf16 [T][d_in], row-major, 16-byte aligned.
 *   Y          out: [T][d_out] row-major, fp32 or bf16 (out_dtype), 16-byte
 *              aligned.
 *   Products and sums in fp32 (fused multiply-add, order unspecified), the
 *   result rounded to nearest even for bf16.  T <= 16 runs a streaming
 *   GEMV, larger T a tcgen05 GEMM.  Shape and error rules as above.
 */
int bitlinear_dense_bf16_forward(const uint16_t *W, int64_t d_out, int64_t d_in,
                                 const uint16_t *X, int64_t T, void *Y, int out_dtype,
                                 cudaStream_t stream);

/*
 * bitlinear_backward -- gradients of the BitLinear forward with the
 * straight-through estimator ([MF] section 3, "Training Dynamics and the
 * Straight-Through Estimator": the rounding is bypassed, so the layer acts
 * as Y = X^ (gamma W~)^T with X^ = X~ beta / 127, gamma and beta constant):
 *
 *   dX = gamma dY W~       [T][d_in]     gradient at X^ (the quantiser input)
 *   dW = gamma dY^T X^     [d_out][d_in] gradient at W~, passed to the latent
 *                                        weights
 *
 *   packed, gamma   the weights as bitlinear_pack_weights left them.
 *   Xq, beta        the forward's activation codes [T][d_in] and scales [T];
 *                   needed for dW only.
 *   dY              bf16 [T][d_out], row-major, 16-byte aligned.
 *   dX, dW          out: fp32 or bf16 (out_dtype), row-major, 16-byte aligned;
 *                   either may be NULL (not computed), not both.
 *   workspace       device scratch of bitlinear_backward_workspace_bytes()
 *                   bytes, 256-byte aligned, owned by the caller (W~ and
 *                   X^ in bf16; the tensor-core GEMMs read them and dY in
 *                   their row-major layouts, without transposes).
 * X^ enters the dW product as bf16 of fl32(q * fl32(beta / 127)); products
 * and sums in fp32, gamma applied once to the fp32 sum.  Shapes: d_out a
 * multiple of 256 and at most 65536, d_in as above, 0 <= T <= 65536 (T = 0
 * zeroes dW).  Errors as above; a short workspace is BITLINEAR_ERR_INVALID_ARG.
 */
size_t bitlinear_backward_workspace_bytes(int64_t d_out, int64_t d_in, int64_t T,
                                          int want_dx, int want_dw);
int bitlinear_backward(const uint32_t *packed, const float *gamma, int64_t d_out,
                       int64_t d_in, const int8_t *Xq, const float *beta, int64_t T,
                       const uint16_t *dY, void *dX, void *dW, int out_dtype,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * bitlinear_device_error -- synchronises `stream`, then reads the device
 * error word that kernels set when a bounded wait gives up.  Returns
 * BITLINEAR_OK when the word is clear, BITLINEAR_ERR_TIMEOUT when a wait
 * expired, BITLINEAR_ERR_CUDA when the synchronisation itself failed.  With
 * clear != 0 the word is reset to zero afterwards.
 */
int bitlinear_device_error(cudaStream_t stream, int clear);

/* bitlinear_device_error(stream, 1): synchronise, report, then clear the
 * device error word. */
int bitlinear_get_last_device_error(cudaStream_t stream);

/*
 * bitlinear_set_wait_limit_ns -- the time after which a kernel's bounded wait
 * on an mbarrier gives up (default 2e9 ns).  Applies to launches made after
 * the call on the current device.  limit_ns must be in [1e3, 6e10].
 */
int bitlinear_set_wait_limit_ns(uint64_t limit_ns);

/*
 * bitlinear_wait_probe -- launches one CTA that waits, through the same
 * bounded-wait routine the GEMM uses, on an mbarrier that nothing ever
 * arrives on.  After limit_ns the wait gives up and the kernel records
 * BITLINEAR_ERR_TIMEOUT in the device error word and returns.  Exists so the
 * timeout path can be tested without stalling any real pipeline.
 */
int bitlinear_wait_probe(uint64_t limit_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
