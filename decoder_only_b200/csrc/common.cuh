// Shared device helpers of the llama_b200 library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "llama_b200.h"

typedef __nv_bfloat16 bf16;

#define LLAMA_CUDA_TRY(expr)                               \
    do {                                                   \
        cudaError_t _e = (expr);                           \
        if (_e != cudaSuccess) return LLAMA_ERR_CUDA;      \
    } while (0)

// Every kernel launch is followed by this check, which also counts it.
void llama_count_launches(int64_t n);
#define LLAMA_LAUNCH_CHECK()                               \
    do {                                                   \
        if (cudaPeekAtLastError() != cudaSuccess) {        \
            cudaGetLastError();                            \
            return LLAMA_ERR_CUDA;                         \
        }                                                  \
        llama_count_launches(1);                           \
    } while (0)

// Programmatic dependent launch.  Kernels on the hot path are launched with
// programmatic stream serialisation: each one lets its successor launch
// early (pdl_launch_dependents) and waits for its predecessor's memory
// (pdl_wait) only before it reads or writes data the predecessor touches.
// Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

extern bool g_llama_pdl;   // launch with the attribute (default on; LLAMA_B200_NO_PDL=1 turns it off)

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = g_llama_pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Device error word values (sticky, set by bounded waits)
#define LLAMA_DEVERR_TIMEOUT 1

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Pack two floats into a bf16x2 word (lower address = first)
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&w);
    return __bfloat1622float2(v);
}

// One-time set-up that acts on the current device only (a kernel's
// shared-memory attribute, the address of a __device__ variable): f runs
// once per device, under a lock, with that device current; a failed f is
// retried on the next call.
constexpr int LLAMA_MAX_DEVICES = 64;
struct PerDeviceOnce {
    std::mutex mu;
    bool done[LLAMA_MAX_DEVICES] = {};
};
template <class F>
inline int once_per_device(PerDeviceOnce& pd, F&& f) {
    int dev = -1;
    LLAMA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= LLAMA_MAX_DEVICES) return LLAMA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(pd.mu);
    if (pd.done[dev]) return LLAMA_OK;
    const int rc = f();
    if (rc == LLAMA_OK) pd.done[dev] = true;
    return rc;
}

static inline int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }
