// Shared device helpers for the Loki sm_100a kernels: 16-byte loads, element
// unpacking, warp reductions and the per-device launch-shape cache.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace loki {

constexpr float kLog2e = 1.4426950408889634f;

// 16-byte read-only load that does not allocate in L1 (each byte is used once).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 word.
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Element traits: how many elements one 16-byte vector holds and how to unpack it.
struct ElemF32 {
    using T = float;
    static constexpr int kVec = 4;
    static constexpr int kBytes = 4;
    __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static float load1(const T* p) { return *p; }
    __device__ __forceinline__ static T from_float(float x) { return x; }
};

struct ElemBF16 {
    using T = __nv_bfloat16;
    static constexpr int kVec = 8;
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
        f[0] = bf16_lo(v.x);
        f[1] = bf16_hi(v.x);
        f[2] = bf16_lo(v.y);
        f[3] = bf16_hi(v.y);
        f[4] = bf16_lo(v.z);
        f[5] = bf16_hi(v.z);
        f[6] = bf16_lo(v.w);
        f[7] = bf16_hi(v.w);
    }
    __device__ __forceinline__ static float load1(const T* p) { return __bfloat162float(*p); }
    __device__ __forceinline__ static T from_float(float x) { return __float2bfloat16_rn(x); }
};

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

template <int W>
__device__ __forceinline__ float group_sum(float v) {
    // butterfly over the W lanes of an aligned group (W a power of two <= 32)
#pragma unroll
    for (int off = W / 2; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__device__ __forceinline__ float group_sum_rt(float v, int w) {
    for (int off = w >> 1; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Atomic add with release-acquire semantics at GPU scope: the calling
// thread's earlier writes (and those it has observed, such as its warp's
// after a warp barrier) are visible to whoever reads the new value, and
// writes that preceded values it reads are visible to its later loads.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Programmatic dependent launch. A kernel launched with the programmatic
// stream-serialization attribute may start while its predecessor on the
// stream is still running; griddep_wait() blocks until the predecessor grid
// has completed and its writes are visible (a no-op without the attribute).
// griddep_launch_dependents() lets the next kernel be scheduled early.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" :::);
}

// Stream-K style static split of `total` work items over `grid` CTAs: CTA c
// owns items [c * per, min((c + 1) * per, total)).
struct Split {
    int64_t total;
    int64_t per;
};

// Sets the preferred L1/shared-memory split of `func` (percent of the
// maximum shared memory, or cudaSharedmemCarveoutMaxL1/MaxShared) once per
// device; the first request for a kernel wins. An SM changes its split only
// when it is empty, so kernels meant to be resident side by side (a
// programmatic dependent launched early next to its predecessor) ask for the
// same, largest, shared split; register-gather kernels, whose loads in flight
// land in L1, ask for the largest L1 and are launched onto drained SMs.
cudaError_t prefer_carveout(const void* func, int carveout);

// Launch `kern` on `s`; with pdl the launch carries the programmatic
// stream-serialization attribute (the kernel must griddep_wait() before
// reading anything its predecessor writes).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t s, bool pdl, Args... args) {
    const cudaError_t ec =
        prefer_carveout(reinterpret_cast<const void*>(kern), cudaSharedmemCarveoutMaxShared);
    if (ec != cudaSuccess) return ec;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace loki
