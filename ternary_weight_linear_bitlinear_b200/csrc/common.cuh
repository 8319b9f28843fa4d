// common.cuh -- device helpers shared by the library's kernels (sm_100a).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "bitlinear.h"

namespace bl {

// Weight formats of the decode kernel: 2-bit ternary tiles, base-3 ternary
// tiles (five codes per byte), 1-bit binary tiles.
constexpr int kFmt2Bit = 0;
constexpr int kFmtBase3 = 1;
constexpr int kFmt1Bit = 2;

// Bits of the device error word.
constexpr uint32_t kErrTimeout = 1u;

// Kernel-side configuration passed by value to every launch.
struct DeviceCtx {
    uint32_t *err;        // device error word (see bitlinear_device_error)
    uint64_t wait_ns;     // bounded-wait limit
};

// Host side: error-word address and wait limit for the current device.
bitlinear_status get_ctx(DeviceCtx *ctx);
// Host side: opt `kernel` in to `bytes` of dynamic shared memory on the
// current device (once per kernel, device and size increase).
cudaError_t ensure_dynamic_smem(const void *kernel, size_t bytes);
// Host side: check the current device is sm_100.
bitlinear_status check_device();

inline bool aligned(const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// A prepared kernel launch: the kernel, its launch shape and copies of its
// parameters, so that a launch can be repeated with one pointer patched
// (the activations of a plan, see bitlinear_linear_plan_run) without
// recomputing anything.  Every entry point launches through one of these,
// so a plan and a direct call run the same launch.
struct LaunchRec {
    const void *func = nullptr;
    dim3 grid{1, 1, 1}, block{1, 1, 1};
    size_t smem = 0;
    unsigned cluster_x = 0;   // 0: no cluster attribute
    bool pdl = false;         // programmatic dependent launch
    int nargs = 0;
    size_t off[16] = {};
    size_t used = 0;
    alignas(128) unsigned char buf[1024];

    template <class V>
    void push(const V &v) {
        const size_t a = alignof(V);
        used = (used + a - 1) & ~(a - 1);
        std::memcpy(buf + used, &v, sizeof(V));
        off[nargs++] = used;
        used += sizeof(V);
    }
    // Overwrite the pointer at byte `field` of parameter `arg`.
    void patch_ptr(int arg, size_t field, const void *p) {
        std::memcpy(buf + off[arg] + field, &p, sizeof p);
    }
    cudaError_t launch(cudaStream_t stream) const {
        void *argv[16];
        for (int i = 0; i < nargs; ++i) argv[i] = const_cast<unsigned char *>(buf + off[i]);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        int na = 0;
        if (cluster_x) {
            attr[na].id = cudaLaunchAttributeClusterDimension;
            attr[na].val.clusterDim.x = cluster_x;
            attr[na].val.clusterDim.y = 1;
            attr[na].val.clusterDim.z = 1;
            ++na;
        }
        if (pdl) {
            attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        cfg.attrs = attr;
        cfg.numAttrs = na;
        return cudaLaunchKernelExC(&cfg, func, argv);
    }
};

// ------------------------------------------------------------- rounding --
// RoundClip's floor(z + 0.5), evaluated exactly on a binary32 z: with
// f = floor(z), z - f is exact whenever it can be near 0.5 (Sterbenz for
// |z| >= 1; plain representability for |z| < 1), so the comparison decides
// the same integer as the exact sum.
__device__ __forceinline__ float round_half_up_exact(float z) {
    float f = floorf(z);
    float frac = __fsub_rn(z, f);
    return (frac >= 0.5f) ? __fadd_rn(f, 1.0f) : f;
}

// The same decision as an int, for |z| < 2^23: fl_rd(z + 0.5) lies in
// [floor(z + 0.5), z + 0.5] (the integer floor(z + 0.5) is representable and
// below z + 0.5, so rounding down cannot pass it), hence its floor is
// floor(z + 0.5).  Larger |z| only ever meet a clip to a small range.
__device__ __forceinline__ int round_half_up_int(float z) {
    return __float2int_rd(__fadd_rd(z, 0.5f));
}

// -------------------------------------------------------------- timers ---
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------ mbarrier ---
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for the phase of parity `parity` to complete.  Returns false
// (after recording kErrTimeout) when `limit_ns` elapses first.  Never traps.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  const DeviceCtx &ctx) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > ctx.wait_ns) {
            atomicOr(ctx.err, kErrTimeout);
            return false;
        }
    }
}

// ------------------------------------------------- programmatic launch ---
// Dependent-launch controls (no-ops when the launch was not programmatic).
__device__ __forceinline__ void pdl_wait_primary() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace bl
