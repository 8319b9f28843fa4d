// pack.cu -- absmean scale and 2-bit ternary packing of latent weights.
//
// "BitNet b1.58: Mathematical Foundations of 1.58-Bit Ternary Quantization,
// Absmean Scaling, and Multiplication-Free LLM Architectures", section 2,
// "Weight Quantization: Absmean Scaling": gamma = mean |W| over the tensor,
// W~ = RoundClip(W / (gamma + eps), -1, 1).  Section 6 (Weight Unpacking)
// names 2-bit packed ternary registers; the tile layout is documented in
// bitlinear.h.
//
// HBM-bound streaming kernels: the reduction reads 4 B per weight, the
// packer reads 4 B and writes 0.25 B per weight.  Both run offline, once per
// weight matrix.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {

constexpr int kRedThreads = 256;
constexpr int kRedMaxBlocks = 148 * 8;

__device__ __forceinline__ double block_sum_f64(double v, double *sh) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sh[warp] = v;
    __syncthreads();
    double r = 0.0;
    if (threadIdx.x == 0) {
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += sh[w];
    }
    __syncthreads();
    return r;  // valid in thread 0
}

// Stage 1: each block sums |W| over a fixed grid-stride set of float4s in
// double and writes one partial.  The order is fixed by (grid, block) sizes,
// so the result is deterministic for a given shape.
__global__ void __launch_bounds__(kRedThreads)
absmean_partial_kernel(const float4 *__restrict__ W4, int64_t n4, double *partial) {
    __shared__ double sh[kRedThreads / 32];
    double acc = 0.0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 v = __ldg(W4 + i);
        acc += fabs((double)v.x) + fabs((double)v.y) + fabs((double)v.z) + fabs((double)v.w);
    }
    double s = block_sum_f64(acc, sh);
    if (threadIdx.x == 0) partial[blockIdx.x] = s;
}

// Stage 2: one block sums the partials in a fixed order; gamma rounded once.
__global__ void __launch_bounds__(kRedThreads)
absmean_final_kernel(const double *partial, int nparts, double count, float *gamma) {
    __shared__ double sh[kRedThreads / 32];
    double acc = 0.0;
    for (int i = threadIdx.x; i < nparts; i += blockDim.x) acc += partial[i];
    double s = block_sum_f64(acc, sh);
    if (threadIdx.x == 0) *gamma = (float)(s / count);
}

// One thread per packed word: 16 consecutive weights of one row.
__global__ void __launch_bounds__(256)
pack_kernel(const float *__restrict__ W, int64_t d_out, int64_t d_in, float eps,
            const float *__restrict__ gamma_ptr, uint32_t *__restrict__ packed,
            float *gamma_out) {
    const float gamma = *gamma_ptr;
    const float den = __fadd_rn(gamma, eps);
    const int64_t tiles_per_row = d_in >> 8;
    const int64_t nwords = (d_out * d_in) >> 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if (blockIdx.x == 0 && threadIdx.x == 0 && gamma_out != gamma_ptr) *gamma_out = gamma;
    for (int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < nwords; wi += stride) {
        const int64_t tile = wi >> 8;
        const int within = (int)(wi & 255);
        const int r = within >> 4, kw = within & 15;
        const int64_t rb = tile / tiles_per_row, kb = tile - rb * tiles_per_row;
        const int64_t o = rb * 16 + r;
        const int64_t k0 = kb * 256 + kw * 16;
        const float4 *src = reinterpret_cast<const float4 *>(W + o * d_in + k0);
        uint32_t word = 0;
        #pragma unroll
        for (int s = 0; s < 4; ++s) {
            float4 v = __ldg(src + s);
            float e[4] = {v.x, v.y, v.z, v.w};
            #pragma unroll
            for (int j = 0; j < 4; ++j) {
                float q = round_half_up_exact(__fdiv_rn(e[j], den));
                q = fminf(fmaxf(q, -1.0f), 1.0f);
                const uint32_t c = (uint32_t)((int)q + 1) & 3u;
                word |= c << (8 * j + 2 * s);
            }
        }
        packed[wi] = word;
    }
}

// Base-3 format (section 4 of the same page, "Memory Bandwidth and Latency
// Bounds": five ternary values per byte, 3^5 = 243 < 256).  Tiles of 16 rows
// x 160 columns (512 bytes), rows padded with W~ = 0; byte B of a tile row
// covers the 20-column group g = B / 4 and, with j = B % 4, holds the codes
// c_i = W~ + 1 of columns 20 g + 4 i + j as sum_i c_i 3^i.  The repacker
// reads the 2-bit tiles, so the conversion is exact; one thread per 32-bit
// word (one 20-column group of one row).  Offline, like the packer.
__global__ void __launch_bounds__(256)
repack_base3_kernel(const uint32_t *__restrict__ packed, int64_t d_out, int64_t d_in,
                    uint32_t *__restrict__ packed3) {
    const int64_t tiles2 = d_in >> 8;
    const int64_t tiles3 = (d_in + 159) / 160;
    const int64_t nwords = d_out * tiles3 * 8;        // 16 rows x 8 words per tile
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < nwords;
         wi += stride) {
        const int64_t tile = wi >> 7;
        const int within = (int)(wi & 127);
        const int r = within >> 3, g = within & 7;
        const int64_t rb = tile / tiles3, kb = tile - rb * tiles3;
        const int64_t k0 = kb * 160 + g * 20;
        uint32_t word = 0;
        #pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t b = 0;
            #pragma unroll
            for (int i = 4; i >= 0; --i) {            // Horner, highest digit first
                const int64_t k = k0 + 4 * i + j;
                uint32_t c = 1;                       // padding: W~ = 0
                if (k < d_in) {
                    const int64_t w2 =
                        ((rb * tiles2 + (k >> 8)) * 16 + r) * 16 + ((k & 255) >> 4);
                    c = (__ldg(packed + w2) >> (8 * (k & 3) + 2 * ((k & 15) >> 2))) & 3u;
                }
                b = b * 3u + c;
            }
            word |= b << (8 * j);
        }
        packed3[wi] = word;
    }
}

// gamma = mean |W| into *gamma_out: the two-stage fixed-order reduction.
static void launch_absmean(const float *W, int64_t n, double *partial, float *gamma_out,
                           cudaStream_t stream) {
    const int64_t n4 = n / 4;
    int blocks = (int)((n4 + kRedThreads * 8 - 1) / (kRedThreads * 8));
    if (blocks > kRedMaxBlocks) blocks = kRedMaxBlocks;
    if (blocks < 1) blocks = 1;
    absmean_partial_kernel<<<blocks, kRedThreads, 0, stream>>>(
        reinterpret_cast<const float4 *>(W), n4, partial);
    absmean_final_kernel<<<1, kRedThreads, 0, stream>>>(partial, blocks, (double)n, gamma_out);
}

// 1-bit format (the W1 of the W1A4 regime on "The End of Matrix
// Multiplications: Welcome to Addition"; the binary alphabet {-1, +1} of
// section 1 of the b1.58 page): W~ = +1 where W >= 0, else -1, with the same
// absmean gamma as scale.  Tiles of 16 rows x 512 columns (1 KiB), rows
// padded with W~ = -1 (bit 0); word kw of a tile row covers columns 32 kw ..
// 32 kw + 31 and the bit c = (W~ + 1) / 2 of column 32 kw + 4 s + j sits at
// bit 8 j + s.  One thread per output word.
__global__ void __launch_bounds__(256)
pack_w1_kernel(const float *__restrict__ W, int64_t d_out, int64_t d_in,
               uint32_t *__restrict__ packed, const float *__restrict__ gamma_src,
               float *gamma_out) {
    const int64_t tiles = (d_in + 511) / 512;
    const int64_t nwords = d_out * tiles * 16;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if (blockIdx.x == 0 && threadIdx.x == 0 && gamma_src && gamma_src != gamma_out)
        *gamma_out = *gamma_src;
    for (int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < nwords; wi += stride) {
        const int64_t tile = wi >> 8;
        const int within = (int)(wi & 255);
        const int r = within >> 4, kw = within & 15;
        const int64_t rb = tile / tiles, kb = tile - rb * tiles;
        const int64_t o = rb * 16 + r;
        const int64_t k0 = kb * 512 + kw * 32;
        uint32_t word = 0;
        if (k0 < d_in) {   // d_in % 256 == 0, so a word is all real or all padding
            const float4 *src = reinterpret_cast<const float4 *>(W + o * d_in + k0);
            #pragma unroll
            for (int s = 0; s < 8; ++s) {
                const float4 v = __ldg(src + s);
                const float e[4] = {v.x, v.y, v.z, v.w};
                #pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (e[j] >= 0.0f) word |= 1u << (8 * j + s);
            }
        }
        packed[wi] = word;
    }
}

}  // namespace bl

using namespace bl;

extern "C" size_t bitlinear_packed_words(int64_t d_out, int64_t d_in) {
    if (d_out <= 0 || d_in <= 0 || d_out % 16 || d_in % 256 || d_in > 65536) return 0;
    return (size_t)(d_out * d_in / 16);
}

extern "C" size_t bitlinear_packed_bytes(int64_t d_out, int64_t d_in) {
    return 4 * bitlinear_packed_words(d_out, d_in);
}

extern "C" size_t bitlinear_pack_workspace_bytes(int64_t d_out, int64_t d_in) {
    if (bitlinear_packed_words(d_out, d_in) == 0) return 0;
    return (size_t)kRedMaxBlocks * sizeof(double);
}

extern "C" int bitlinear_pack_weights(const float *W, int64_t d_out, int64_t d_in, float eps,
                                      const float *gamma_in, void *workspace,
                                      size_t workspace_bytes, uint32_t *packed,
                                      float *gamma_out, cudaStream_t stream) {
    if (!W || !packed || !gamma_out) return BITLINEAR_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BITLINEAR_ERR_INVALID_ARG;
    if (bitlinear_packed_words(d_out, d_in) == 0) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (!gamma_in) {
        if (!workspace) return BITLINEAR_ERR_INVALID_ARG;
        if (workspace_bytes < bitlinear_pack_workspace_bytes(d_out, d_in))
            return BITLINEAR_ERR_INVALID_ARG;
        if (!aligned(workspace, 8)) return BITLINEAR_ERR_MISALIGNED;
    } else if (!aligned(gamma_in, 4)) {
        return BITLINEAR_ERR_MISALIGNED;
    }
    if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(gamma_out, 4))
        return BITLINEAR_ERR_MISALIGNED;
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;

    const int64_t n = d_out * d_in;
    const float *gptr = gamma_in;
    if (!gamma_in) {
        launch_absmean(W, n, static_cast<double *>(workspace), gamma_out, stream);
        gptr = gamma_out;
    }
    const int64_t nwords = n / 16;
    int64_t pblocks = (nwords + 255) / 256;
    if (pblocks > 148 * 16) pblocks = 148 * 16;
    pack_kernel<<<(int)pblocks, 256, 0, stream>>>(W, d_out, d_in, eps, gptr, packed, gamma_out);
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Allocation-free variant of bitlinear_pack_weights.
//
// Some callers cannot allocate device memory at the point where they pack
// weights: code running while a stream is being captured into a CUDA graph
// (cudaMalloc is not permitted during capture), runtimes whose device memory
// is fully reserved up front by their own pool, and hosts without a device
// allocator they may call.  bitlinear_pack_weights needs such callers to hand
// it a device workspace for the partial sums of mean|W|.  This variant keeps
// those partial sums in a fixed array inside the library instead.
//
// The array below lives in every GPU's memory that loads the library, until
// the process exits.  Host code cannot use its name as a device address, so
// the address is looked up once per device with cudaGetSymbolAddress (on the
// first call made with that device current) and passed to the kernels.
// ---------------------------------------------------------------------------
namespace bl {

constexpr int kNoallocPartials = kRedMaxBlocks;   // 1184 doubles = 9,472 bytes

static __device__ __align__(256) double g_pack_partials[kNoallocPartials];

namespace {
std::mutex g_noalloc_mu;
double *g_noalloc_ptr[64];
}  // namespace

// The address is looked up again on every call made outside stream capture,
// so a device reset (after which the array may sit at a new address) never
// leaves a stale pointer in use; during a capture the address remembered
// from the last such call on this device is used.
static bitlinear_status noalloc_scratch(cudaStream_t stream, double **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BITLINEAR_ERR_DEVICE;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return BITLINEAR_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_pack_partials) != cudaSuccess || !p)
            return BITLINEAR_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<double *>(p);
    } else if (!g_noalloc_ptr[dev]) {
        // First use on this device inside a capture: the lookup may have to
        // load the module, which is not allowed while capturing.
        return BITLINEAR_ERR_CUDA;
    }
    *out = g_noalloc_ptr[dev];
    return BITLINEAR_OK;
}

}  // namespace bl

extern "C" int bitlinear_pack_weights_noalloc(const float *W, int64_t d_out, int64_t d_in,
                                              float eps, uint32_t *packed, float *gamma_out,
                                              cudaStream_t stream) {
    if (!W || !packed || !gamma_out) return BITLINEAR_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BITLINEAR_ERR_INVALID_ARG;
    if (bitlinear_packed_words(d_out, d_in) == 0) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(gamma_out, 4))
        return BITLINEAR_ERR_MISALIGNED;
    // Same reduction grid as bitlinear_pack_weights, so gamma is bit-identical.
    const int64_t n = d_out * d_in;
    const int64_t n4 = n / 4;
    int64_t blocks = (n4 + kRedThreads * 8 - 1) / (kRedThreads * 8);
    if (blocks > kRedMaxBlocks) blocks = kRedMaxBlocks;
    if (blocks < 1) blocks = 1;
    // The grid cap above is the array's size, so every accepted shape fits.
    static_assert(kNoallocPartials >= kRedMaxBlocks, "noalloc partials hold the largest grid");
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;
    double *partial = nullptr;
    st = noalloc_scratch(stream, &partial);
    if (st != BITLINEAR_OK) return st;
    // Every partial the final kernel reads is written by this call first, so
    // nothing in the shared array has to start at zero.
    absmean_partial_kernel<<<(int)blocks, kRedThreads, 0, stream>>>(
        reinterpret_cast<const float4 *>(W), n4, partial);
    absmean_final_kernel<<<1, kRedThreads, 0, stream>>>(partial, (int)blocks, (double)n,
                                                         gamma_out);
    int64_t pblocks = (n / 16 + 255) / 256;
    if (pblocks > 148 * 16) pblocks = 148 * 16;
    pack_kernel<<<(int)pblocks, 256, 0, stream>>>(W, d_out, d_in, eps, gamma_out, packed,
                                                  gamma_out);
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

extern "C" size_t bitlinear_base3_bytes(int64_t d_out, int64_t d_in) {
    if (bitlinear_packed_words(d_out, d_in) == 0) return 0;
    return (size_t)(d_out * ((d_in + 159) / 160) * 32);
}

extern "C" int bitlinear_repack_base3(const uint32_t *packed, int64_t d_out, int64_t d_in,
                                      uint8_t *packed3, cudaStream_t stream) {
    if (bitlinear_packed_words(d_out, d_in) == 0) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (!packed || !packed3) return BITLINEAR_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(packed3, 16)) return BITLINEAR_ERR_MISALIGNED;
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;
    const int64_t nwords = (int64_t)(bitlinear_base3_bytes(d_out, d_in) / 4);
    int64_t blocks = (nwords + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    repack_base3_kernel<<<(int)blocks, 256, 0, stream>>>(packed, d_out, d_in,
                                                          reinterpret_cast<uint32_t *>(packed3));
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

extern "C" size_t bitlinear_w1_packed_bytes(int64_t d_out, int64_t d_in) {
    if (bitlinear_packed_words(d_out, d_in) == 0) return 0;
    return (size_t)(d_out * ((d_in + 511) / 512) * 64);
}

extern "C" int bitlinear_pack_weights_w1(const float *W, int64_t d_out, int64_t d_in,
                                         const float *gamma_in, void *workspace,
                                         size_t workspace_bytes, uint32_t *packed1,
                                         float *gamma_out, cudaStream_t stream) {
    if (!W || !packed1 || !gamma_out) return BITLINEAR_ERR_INVALID_ARG;
    if (bitlinear_packed_words(d_out, d_in) == 0) return BITLINEAR_ERR_UNSUPPORTED_SHAPE;
    if (!gamma_in) {
        if (!workspace) return BITLINEAR_ERR_INVALID_ARG;
        if (workspace_bytes < bitlinear_pack_workspace_bytes(d_out, d_in))
            return BITLINEAR_ERR_INVALID_ARG;
        if (!aligned(workspace, 8)) return BITLINEAR_ERR_MISALIGNED;
    } else if (!aligned(gamma_in, 4)) {
        return BITLINEAR_ERR_MISALIGNED;
    }
    if (!aligned(W, 16) || !aligned(packed1, 16) || !aligned(gamma_out, 4))
        return BITLINEAR_ERR_MISALIGNED;
    bitlinear_status st = check_device();
    if (st != BITLINEAR_OK) return st;
    if (!gamma_in) launch_absmean(W, d_out * d_in, static_cast<double *>(workspace), gamma_out,
                                  stream);
    const int64_t nwords = (int64_t)(bitlinear_w1_packed_bytes(d_out, d_in) / 4);
    int64_t blocks = (nwords + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    pack_w1_kernel<<<(int)blocks, 256, 0, stream>>>(W, d_out, d_in, packed1, gamma_in,
                                                    gamma_out);
    return cudaGetLastError() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}
