// abi.cu -- the library's C entry points: validation, kernel selection,
// device error word, bounded-wait configuration.
#include <cmath>
#include <cstdint>
#include <mutex>
#include <new>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {

bitlinear_status launch_quant_act(const uint16_t *X, int64_t T, int64_t d_in,
                                  const float *norm_gain, uint32_t flags, float eps,
                                  float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                  float *beta, int32_t *rowsum, float *inv_rms_out, bool pdl,
                                  cudaStream_t stream);
bitlinear_status launch_gemv(const void *packed, const float *gamma, int64_t d_out,
                             int64_t d_in, const int8_t *Xq, const float *beta,
                             const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                             int32_t *acc_out, bool static_weights, int fmt, float qmax,
                             void *ws, cudaStream_t stream);
bool decode_can_fuse(int64_t T, int64_t d_in);
size_t decode_workspace_bytes(int64_t d_out, int64_t T);
int set_decode_split_mode(int mode);
int set_decode_kernel(int mode);
bool decode_use_tc(int64_t T, int64_t d_out, int64_t d_in);
bitlinear_status prepare_decode_tc(const uint32_t *packed, const float *gamma, int64_t d_out,
                                   int64_t d_in, const int8_t *Xq, const float *beta,
                                   const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                   int32_t *acc_out, bool static_weights, void *ws,
                                   LaunchRec *rec);
bitlinear_status launch_linear_fused(const void *packed, const float *gamma, int64_t d_out,
                                     int64_t d_in, const uint16_t *X, int64_t T,
                                     const float *gain, bool rmsnorm, float eps, float norm_eps,
                                     const float *inv_rms_in, int8_t *Xq, float *beta,
                                     int32_t *rowsum, void *Y, int out_dtype,
                                     bool static_weights, int fmt, float qmax, void *ws,
                                     cudaStream_t stream);
bitlinear_status prepare_gemv(const void *packed, const float *gamma, int64_t d_out,
                              int64_t d_in, const int8_t *Xq, const float *beta,
                              const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                              int32_t *acc_out, bool static_weights, int fmt, float qmax,
                              void *ws, LaunchRec *rec);
bitlinear_status prepare_linear_fused(const void *packed, const float *gamma, int64_t d_out,
                                      int64_t d_in, const uint16_t *X, int64_t T,
                                      const float *gain, bool rmsnorm, float eps,
                                      float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                      float *beta, int32_t *rowsum, void *Y, int out_dtype,
                                      bool static_weights, int fmt, float qmax, void *ws,
                                      LaunchRec *rec);
size_t decode_x_offset();
bitlinear_status prepare_quant_act(const uint16_t *X, int64_t T, int64_t d_in,
                                   const float *norm_gain, uint32_t flags, float eps,
                                   float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                   float *beta, int32_t *rowsum, float *inv_rms_out, bool pdl,
                                   LaunchRec *rec);
bitlinear_status prepare_gemm_tc_pair(const uint32_t *packed, const float *gamma, int64_t d_out,
                                      int64_t d_in, const int8_t *Xq, const float *beta,
                                      const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                      int32_t *acc_out, LaunchRec *rec);
bitlinear_status launch_gemm_tc_pair(const uint32_t *packed, const float *gamma, int64_t d_out,
                                     int64_t d_in, const int8_t *Xq, const float *beta,
                                     const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                     int32_t *acc_out, cudaStream_t stream);
bitlinear_status launch_dense_bf16(const uint16_t *W, int64_t d_out, int64_t d_in,
                                   const uint16_t *X, int64_t T, void *Y, int out_dtype,
                                   const float *alpha, cudaStream_t stream);

// Device error word: set by kernels whose bounded waits expire.
__device__ uint32_t g_error_word;

__global__ void wait_probe_kernel(DeviceCtx ctx) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        mbar_init_fence();
        // Nothing ever arrives: the wait must give up after ctx.wait_ns.
        mbar_wait_bounded(smem_u32(&bar), 0, ctx);
    }
}

namespace {
constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
std::mutex g_mu;
uint32_t *g_err_ptr[kMaxDevices];
uint64_t g_wait_ns[kMaxDevices];
int g_dev_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 unusable
}  // namespace

bitlinear_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return BITLINEAR_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_dev_ok[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return BITLINEAR_ERR_DEVICE;
        g_dev_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    return g_dev_ok[dev] == 1 ? BITLINEAR_OK : BITLINEAR_ERR_DEVICE;
}

bitlinear_status get_ctx(DeviceCtx *ctx) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return BITLINEAR_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return BITLINEAR_ERR_CUDA;
        g_err_ptr[dev] = static_cast<uint32_t *>(p);
    }
    ctx->err = g_err_ptr[dev];
    ctx->wait_ns = g_wait_ns[dev] ? g_wait_ns[dev] : kDefaultWaitNs;
    return BITLINEAR_OK;
}

cudaError_t ensure_dynamic_smem(const void *kernel, size_t bytes) {
    struct Entry { const void *kernel; int dev; size_t bytes; };
    static Entry entries[256];
    static int n_entries = 0;
    if (bytes <= 16 * 1024) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < n_entries; ++i)
        if (entries[i].kernel == kernel && entries[i].dev == dev && entries[i].bytes >= bytes)
            return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    for (int i = 0; i < n_entries; ++i)
        if (entries[i].kernel == kernel && entries[i].dev == dev) {
            entries[i].bytes = bytes;
            return cudaSuccess;
        }
    if (n_entries < 256) entries[n_entries++] = {kernel, dev, bytes};
    return cudaSuccess;
}

static bitlinear_status validate_forward(const void *packed, const float *gamma,
                                         int64_t d_out, int64_t d_in, int64_t T, void *Y,
                                         int out_dtype, int32_t *acc_out) {
    if (T < 0 || T > (1 << 20)) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (d_out <= 0 || d_out % 16 || d_out > (1 << 22)) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (d_in <= 0 || d_in % 256 || d_in > 65536) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (out_dtype != BITLINEAR_OUT_F32 && out_dtype != BITLINEAR_OUT_BF16)
        return BITLINEAR_ERR_INVALID_ARG;
    if (T == 0) return BITLINEAR_OK;  // empty problem: nothing to check or enqueue
    if (!packed || !gamma || !Y) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(gamma, 4) || !aligned(Y, 16) ||
        (acc_out && !aligned(acc_out, 16)))
        return BITLINEAR_ERR_MISALIGNED;
    return BITLINEAR_OK;
}

static bitlinear_status dispatch_forward(const void *packed, const float *gamma,
                                         int64_t d_out, int64_t d_in, const int8_t *Xq,
                                         const float *beta, const int32_t *rowsum, int64_t T,
                                         void *Y, int out_dtype, int32_t *acc_out,
                                         bool static_weights, int fmt, float qmax, void *ws,
                                         cudaStream_t stream) {
    if (T <= 16 && fmt == kFmt2Bit && qmax == 127.0f && decode_use_tc(T, d_out, d_in)) {
        LaunchRec rec;
        bitlinear_status st = prepare_decode_tc(static_cast<const uint32_t *>(packed), gamma,
                                                d_out, d_in, Xq, beta, rowsum, T, Y, out_dtype,
                                                acc_out, static_weights, ws, &rec);
        if (st != BITLINEAR_OK) return st;
        return rec.launch(stream) == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
    }
    if (T <= 16 || fmt != kFmt2Bit)
        return launch_gemv(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y, out_dtype,
                           acc_out, static_weights, fmt, qmax, ws, stream);
    return launch_gemm_tc_pair(static_cast<const uint32_t *>(packed), gamma, d_out, d_in, Xq,
                               beta, rowsum, T, Y, out_dtype, acc_out, stream);
}

// The optional split workspace of the decode product: large enough for
// (d_out, T) and 16-byte aligned.
static bitlinear_status validate_workspace(int64_t d_out, int64_t T, const void *ws,
                                           size_t ws_bytes) {
    if (!ws) return BITLINEAR_OK;
    if (ws_bytes < decode_workspace_bytes(d_out, T)) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(ws, 16)) return BITLINEAR_ERR_MISALIGNED;
    return BITLINEAR_OK;
}

static bitlinear_status forward_common(const void *packed, const float *gamma, int64_t d_out,
                                       int64_t d_in, const int8_t *Xq, const float *beta,
                                       const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                       int32_t *acc_out, int fmt, float qmax, void *ws,
                                       size_t ws_bytes, cudaStream_t stream) {
    bitlinear_status st = validate_forward(packed, gamma, d_out, d_in, T, Y, out_dtype, acc_out);
    if (st != BITLINEAR_OK) return st;
    st = validate_workspace(d_out, T, ws, ws_bytes);
    if (st != BITLINEAR_OK) return st;
    if (fmt != kFmt2Bit && T > 16) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return BITLINEAR_OK;
    if (!Xq || !beta || !rowsum) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(Xq, 16) || !aligned(beta, 4) || !aligned(rowsum, 4))
        return BITLINEAR_ERR_MISALIGNED;
    st = check_device();
    if (st != BITLINEAR_OK) return st;
    return dispatch_forward(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y, out_dtype,
                            acc_out, false, fmt, qmax, ws, stream);
}

// Argument checks of bitlinear_linear (and of a plan for it), X excluded:
// everything but the device.
static bitlinear_status validate_linear(const void *packed, const float *gamma, int64_t d_out,
                                        int64_t d_in, int64_t T, const float *norm_gain,
                                        uint32_t flags, float eps, float norm_eps,
                                        const float *inv_rms_in, int8_t *Xq, float *beta,
                                        int32_t *rowsum, void *Y, int out_dtype, int fmt) {
    bitlinear_status st = validate_forward(packed, gamma, d_out, d_in, T, Y, out_dtype, nullptr);
    if (st != BITLINEAR_OK) return st;
    if (fmt != kFmt2Bit && T > 16) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    uint32_t allowed = BITLINEAR_RMSNORM | BITLINEAR_STATIC_WEIGHTS | BITLINEAR_PER_TENSOR_ABSMAX;
    if (fmt == kFmt1Bit) allowed |= BITLINEAR_ACT_4BIT;   // the A4 of W1A4
    if (flags & ~allowed) return BITLINEAR_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !std::isfinite(eps) || !(norm_eps >= 0.0f) || !std::isfinite(norm_eps))
        return BITLINEAR_ERR_INVALID_ARG;
    if (T == 0) return BITLINEAR_OK;
    if (!Xq || !beta || !rowsum) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(Xq, 16) || !aligned(beta, 4) || !aligned(rowsum, 4) ||
        (norm_gain && !aligned(norm_gain, 4)) || (inv_rms_in && !aligned(inv_rms_in, 4)))
        return BITLINEAR_ERR_MISALIGNED;
    return BITLINEAR_OK;
}

static bitlinear_status linear_common(const void *packed, const float *gamma, int64_t d_out,
                                      int64_t d_in, const uint16_t *X, int64_t T,
                                      const float *norm_gain, uint32_t flags, float eps,
                                      float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                      float *beta, int32_t *rowsum, void *Y, int out_dtype,
                                      int fmt, void *ws, size_t ws_bytes, cudaStream_t stream) {
    bitlinear_status st = validate_linear(packed, gamma, d_out, d_in, T, norm_gain, flags, eps,
                                          norm_eps, inv_rms_in, Xq, beta, rowsum, Y, out_dtype,
                                          fmt);
    if (st != BITLINEAR_OK) return st;
    st = validate_workspace(d_out, T, ws, ws_bytes);
    if (st != BITLINEAR_OK || T == 0) return st;
    if (!X) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(X, 16)) return BITLINEAR_ERR_MISALIGNED;
    const float qmax = (flags & BITLINEAR_ACT_4BIT) ? 7.0f : 127.0f;
    st = check_device();
    if (st != BITLINEAR_OK) return st;
    const bool static_weights = (flags & BITLINEAR_STATIC_WEIGHTS) != 0;
    const bool rmsnorm = (flags & BITLINEAR_RMSNORM) != 0;
    const bool per_tensor = (flags & BITLINEAR_PER_TENSOR_ABSMAX) != 0;
    if (!per_tensor && decode_can_fuse(T, d_in) &&
        !(fmt == kFmt2Bit && decode_use_tc(T, d_out, d_in)))
        return launch_linear_fused(packed, gamma, d_out, d_in, X, T, norm_gain, rmsnorm, eps,
                                   norm_eps, inv_rms_in, Xq, beta, rowsum, Y, out_dtype,
                                   static_weights, fmt, qmax, ws, stream);
    // Quantiser, then the product as its programmatic dependent: with static
    // weights the product streams them while the codes are still being made.
    st = launch_quant_act(X, T, d_in, norm_gain,
                          flags & (BITLINEAR_RMSNORM | BITLINEAR_PER_TENSOR_ABSMAX |
                                   BITLINEAR_ACT_4BIT),
                          eps, norm_eps, inv_rms_in, Xq, beta, rowsum, nullptr, true, stream);
    if (st != BITLINEAR_OK) return st;
    return dispatch_forward(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y, out_dtype,
                            nullptr, static_weights, fmt, qmax, ws, stream);
}

}  // namespace bl

// A bound bitlinear_linear call: the validated arguments and the prepared
// launches, with the activations left to fill in at each run.
struct bitlinear_plan {
    int device = -1;
    int64_t T = 0;
    int steps = 0;            // 0: nothing to run (T = 0); -1: no prepared launches
    bl::LaunchRec rec[2];     // rec[0] takes X
    size_t x_field = 0;       // byte offset of X inside rec[0]'s parameter 0
    // the call's arguments, for plans run through bitlinear_linear itself
    const uint32_t *packed = nullptr;
    const float *gamma = nullptr;
    int64_t d_out = 0, d_in = 0;
    const float *norm_gain = nullptr;
    uint32_t flags = 0;
    float eps = 0.0f, norm_eps = 0.0f;
    int8_t *Xq = nullptr;
    float *beta = nullptr;
    int32_t *rowsum = nullptr;
    void *Y = nullptr;
    int out_dtype = 0;
    void *ws = nullptr;       // owned split workspace of the decode product, or null
    size_t ws_bytes = 0;
};

using namespace bl;

extern "C" int bitlinear_version(void) { return 3; }

extern "C" int bitlinear_set_decode_split(int mode) { return set_decode_split_mode(mode); }

extern "C" int bitlinear_set_decode_kernel(int mode) { return set_decode_kernel(mode); }

extern "C" size_t bitlinear_decode_workspace_bytes(int64_t d_out, int64_t T) {
    if (d_out <= 0 || d_out % 16 || d_out > (1 << 22)) return 0;
    return decode_workspace_bytes(d_out, T);
}

extern "C" const char *bitlinear_status_string(int status) {
    switch (status) {
        case BITLINEAR_OK: return "ok";
        case BITLINEAR_ERR_INVALID_ARG: return "invalid argument";
        case BITLINEAR_ERR_MISALIGNED: return "misaligned pointer";
        case BITLINEAR_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case BITLINEAR_ERR_CUDA: return "CUDA runtime error";
        case BITLINEAR_ERR_TIMEOUT: return "device-side bounded wait expired";
        case BITLINEAR_ERR_DEVICE: return "no usable sm_100 device";
        default: return "unknown status";
    }
}

extern "C" int bitlinear_forward(const uint32_t *packed, const float *gamma, int64_t d_out,
                                 int64_t d_in, const int8_t *Xq, const float *beta,
                                 const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                 int32_t *acc_out, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
    return forward_common(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y, out_dtype, acc_out,
                          kFmt2Bit, 127.0f, workspace, workspace_bytes, stream);
}

extern "C" int bitlinear_forward_base3(const uint8_t *packed3, const float *gamma, int64_t d_out,
                                       int64_t d_in, const int8_t *Xq, const float *beta,
                                       const int32_t *rowsum, int64_t T, void *Y, int out_dtype,
                                       int32_t *acc_out, void *workspace, size_t workspace_bytes,
                                       cudaStream_t stream) {
    return forward_common(packed3, gamma, d_out, d_in, Xq, beta, rowsum, T, Y, out_dtype,
                          acc_out, kFmtBase3, 127.0f, workspace, workspace_bytes, stream);
}

extern "C" int bitlinear_forward_w1(const uint32_t *packed1, const float *gamma, int64_t d_out,
                                    int64_t d_in, const int8_t *Xq, const float *beta,
                                    const int32_t *rowsum, int64_t T, int act_bits, void *Y,
                                    int out_dtype, int32_t *acc_out, void *workspace,
                                    size_t workspace_bytes, cudaStream_t stream) {
    if (act_bits != 4 && act_bits != 8) return BITLINEAR_ERR_INVALID_ARG;
    return forward_common(packed1, gamma, d_out, d_in, Xq, beta, rowsum, T, Y, out_dtype,
                          acc_out, kFmt1Bit, act_bits == 4 ? 7.0f : 127.0f, workspace,
                          workspace_bytes, stream);
}

extern "C" int bitlinear_linear(const uint32_t *packed, const float *gamma, int64_t d_out,
                                int64_t d_in, const uint16_t *X, int64_t T,
                                const float *norm_gain, uint32_t flags, float eps, float norm_eps,
                                const float *inv_rms_in, int8_t *Xq, float *beta,
                                int32_t *rowsum, void *Y, int out_dtype, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream) {
    return linear_common(packed, gamma, d_out, d_in, X, T, norm_gain, flags, eps, norm_eps,
                         inv_rms_in, Xq, beta, rowsum, Y, out_dtype, kFmt2Bit, workspace,
                         workspace_bytes, stream);
}

extern "C" int bitlinear_linear_base3(const uint8_t *packed3, const float *gamma, int64_t d_out,
                                      int64_t d_in, const uint16_t *X, int64_t T,
                                      const float *norm_gain, uint32_t flags, float eps,
                                      float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                      float *beta, int32_t *rowsum, void *Y, int out_dtype,
                                      void *workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
    return linear_common(packed3, gamma, d_out, d_in, X, T, norm_gain, flags, eps, norm_eps,
                         inv_rms_in, Xq, beta, rowsum, Y, out_dtype, kFmtBase3, workspace,
                         workspace_bytes, stream);
}

extern "C" int bitlinear_linear_w1(const uint32_t *packed1, const float *gamma, int64_t d_out,
                                   int64_t d_in, const uint16_t *X, int64_t T,
                                   const float *norm_gain, uint32_t flags, float eps,
                                   float norm_eps, const float *inv_rms_in, int8_t *Xq,
                                   float *beta, int32_t *rowsum, void *Y, int out_dtype,
                                   void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
    return linear_common(packed1, gamma, d_out, d_in, X, T, norm_gain, flags, eps, norm_eps,
                         inv_rms_in, Xq, beta, rowsum, Y, out_dtype, kFmt1Bit, workspace,
                         workspace_bytes, stream);
}

extern "C" int bitlinear_dense_bf16_forward(const uint16_t *W, int64_t d_out, int64_t d_in,
                                            const uint16_t *X, int64_t T, void *Y,
                                            int out_dtype, cudaStream_t stream) {
    if (T < 0 || T > (1 << 20)) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (d_out <= 0 || d_out % 16 || d_out > (1 << 22)) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (d_in <= 0 || d_in % 256 || d_in > 65536) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (out_dtype != BITLINEAR_OUT_F32 && out_dtype != BITLINEAR_OUT_BF16)
        return BITLINEAR_ERR_INVALID_ARG;
    if (T == 0) return BITLINEAR_OK;
    if (!W || !X || !Y) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(X, 16) || !aligned(Y, 16)) return BITLINEAR_ERR_MISALIGNED;
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;
    return launch_dense_bf16(W, d_out, d_in, X, T, Y, out_dtype, nullptr, stream);
}

extern "C" int bitlinear_device_error(cudaStream_t stream, int clear) {
    DeviceCtx ctx;
    bitlinear_status st = get_ctx(&ctx);
    if (st != BITLINEAR_OK) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return BITLINEAR_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, ctx.err, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess)
        return BITLINEAR_ERR_CUDA;
    if (clear && word) {
        const uint32_t zero = 0;
        if (cudaMemcpy(ctx.err, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
            return BITLINEAR_ERR_CUDA;
    }
    return (word & kErrTimeout) ? BITLINEAR_ERR_TIMEOUT : BITLINEAR_OK;
}

extern "C" int bitlinear_get_last_device_error(cudaStream_t stream) {
    return bitlinear_device_error(stream, 1);
}

extern "C" int bitlinear_set_wait_limit_ns(uint64_t limit_ns) {
    if (limit_ns < 1000ull || limit_ns > 60000000000ull) return BITLINEAR_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return BITLINEAR_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    g_wait_ns[dev] = limit_ns;
    return BITLINEAR_OK;
}

extern "C" int bitlinear_wait_probe(uint64_t limit_ns, cudaStream_t stream) {
    if (limit_ns < 1000ull || limit_ns > 60000000000ull) return BITLINEAR_ERR_INVALID_ARG;
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;
    DeviceCtx ctx;
    st = get_ctx(&ctx);
    if (st != BITLINEAR_OK) return st;
    ctx.wait_ns = limit_ns;
    wait_probe_kernel<<<1, 32, 0, stream>>>(ctx);
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

extern "C" int bitlinear_linear_plan_create(const uint32_t *packed, const float *gamma,
                                            int64_t d_out, int64_t d_in, int64_t T,
                                            const float *norm_gain, uint32_t flags, float eps,
                                            float norm_eps, int8_t *Xq, float *beta,
                                            int32_t *rowsum, void *Y, int out_dtype,
                                            bitlinear_plan **plan) {
    if (!plan) return BITLINEAR_ERR_INVALID_ARG;
    *plan = nullptr;
    bitlinear_status st = validate_linear(packed, gamma, d_out, d_in, T, norm_gain, flags, eps,
                                          norm_eps, nullptr, Xq, beta, rowsum, Y, out_dtype,
                                          kFmt2Bit);
    if (st != BITLINEAR_OK) return st;
    st = check_device();
    if (st != BITLINEAR_OK) return st;
    bitlinear_plan *p = new (std::nothrow) bitlinear_plan();
    if (!p) return BITLINEAR_ERR_INVALID_ARG;
    if (cudaGetDevice(&p->device) != cudaSuccess) {
        delete p;
        return BITLINEAR_ERR_DEVICE;
    }
    p->T = T;
    p->packed = packed;
    p->gamma = gamma;
    p->d_out = d_out;
    p->d_in = d_in;
    p->norm_gain = norm_gain;
    p->flags = flags;
    p->eps = eps;
    p->norm_eps = norm_eps;
    p->Xq = Xq;
    p->beta = beta;
    p->rowsum = rowsum;
    p->Y = Y;
    p->out_dtype = out_dtype;
    const bool static_weights = (flags & BITLINEAR_STATIC_WEIGHTS) != 0;
    const bool rmsnorm = (flags & BITLINEAR_RMSNORM) != 0;
    const bool per_tensor = (flags & BITLINEAR_PER_TENSOR_ABSMAX) != 0;
    // A decode plan owns a split workspace, used by its launches when they
    // split.  It is zeroed on a private stream and waited for here, so that a
    // first run on any stream (one that does not wait for the legacy default
    // stream included) finds it zero.
    if (T >= 1 && T <= 16) {
        p->ws_bytes = decode_workspace_bytes(d_out, T);
        if (cudaMalloc(&p->ws, p->ws_bytes) != cudaSuccess) {
            cudaGetLastError();
            delete p;
            return BITLINEAR_ERR_CUDA;
        }
        cudaStream_t zs = nullptr;
        bool zeroed = cudaStreamCreateWithFlags(&zs, cudaStreamNonBlocking) == cudaSuccess;
        if (zeroed)
            zeroed = cudaMemsetAsync(p->ws, 0, p->ws_bytes, zs) == cudaSuccess &&
                     cudaStreamSynchronize(zs) == cudaSuccess;
        if (zs) cudaStreamDestroy(zs);
        if (!zeroed) {
            cudaGetLastError();
            cudaFree(p->ws);
            delete p;
            return BITLINEAR_ERR_CUDA;
        }
    }
    if (T == 0) {
        p->steps = 0;
    } else if (per_tensor) {
        p->steps = -1;   // three launches with a folded beta: run as bitlinear_linear
    } else if (decode_can_fuse(T, d_in) && !decode_use_tc(T, d_out, d_in)) {
        st = prepare_linear_fused(packed, gamma, d_out, d_in, nullptr, T, norm_gain, rmsnorm, eps,
                                  norm_eps, nullptr, Xq, beta, rowsum, Y, out_dtype,
                                  static_weights, kFmt2Bit, 127.0f, p->ws, &p->rec[0]);
        p->x_field = decode_x_offset();
        p->steps = 1;
    } else {
        st = prepare_quant_act(nullptr, T, d_in, norm_gain, flags & BITLINEAR_RMSNORM, eps,
                               norm_eps, nullptr, Xq, beta, rowsum, nullptr, true, &p->rec[0]);
        p->x_field = 0;
        if (st == BITLINEAR_OK)
            st = T <= 16 && decode_use_tc(T, d_out, d_in)
                     ? prepare_decode_tc(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y,
                                         out_dtype, nullptr, static_weights, p->ws, &p->rec[1])
                 : T <= 16 ? prepare_gemv(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y,
                                        out_dtype, nullptr, static_weights, kFmt2Bit, 127.0f,
                                        p->ws, &p->rec[1])
                         : prepare_gemm_tc_pair(packed, gamma, d_out, d_in, Xq, beta, rowsum, T, Y,
                                                out_dtype, nullptr, &p->rec[1]);
        p->steps = 2;
    }
    if (p->ws && st != BITLINEAR_OK) {
        cudaFree(p->ws);
        p->ws = nullptr;
        p->ws_bytes = 0;
    }
    if (st != BITLINEAR_OK) {
        delete p;
        return st;
    }
    *plan = p;
    return BITLINEAR_OK;
}

extern "C" int bitlinear_linear_plan_run(const bitlinear_plan *plan, const uint16_t *X,
                                         cudaStream_t stream) {
    if (!plan) return BITLINEAR_ERR_INVALID_ARG;
    if (plan->steps == 0) return BITLINEAR_OK;
    if (!X) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(X, 16)) return BITLINEAR_ERR_MISALIGNED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) return BITLINEAR_ERR_DEVICE;
    if (plan->steps < 0)
        return linear_common(plan->packed, plan->gamma, plan->d_out, plan->d_in, X, plan->T,
                             plan->norm_gain, plan->flags, plan->eps, plan->norm_eps, nullptr,
                             plan->Xq, plan->beta, plan->rowsum, plan->Y, plan->out_dtype,
                             kFmt2Bit, plan->ws, plan->ws_bytes, stream);
    LaunchRec first = plan->rec[0];
    first.patch_ptr(0, plan->x_field, X);
    if (first.launch(stream) != cudaSuccess) return BITLINEAR_ERR_CUDA;
    if (plan->steps == 2 && plan->rec[1].launch(stream) != cudaSuccess) return BITLINEAR_ERR_CUDA;
    return BITLINEAR_OK;
}

extern "C" void bitlinear_plan_destroy(bitlinear_plan *plan) {
    if (plan && plan->ws) {
        int prev = -1;
        cudaGetDevice(&prev);
        cudaSetDevice(plan->device);
        cudaFree(plan->ws);
        if (prev >= 0) cudaSetDevice(prev);
    }
    delete plan;
}
