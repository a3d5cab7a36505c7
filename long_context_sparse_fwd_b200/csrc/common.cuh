// common.cuh -- small device helpers shared by the CSA / HCA kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>
#include <utility>
#include <unordered_map>

#include "../../include/csa.h"

namespace csa {

// Status word at the start of every workspace. Kernels record the first data error they find.
__device__ __forceinline__ void report(int32_t *status, int32_t code)
{
    if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf2f(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }
__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint16_t f2bf(float f)
{
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi)
{
    return (uint32_t)f2bf(lo) | ((uint32_t)f2bf(hi) << 16);
}

// Interleaved-pair RoPE angle: pair p of r rope channels at position pos has angle
// pos * theta^(-2p/r) (Hugging Face Transformers docs "DeepSeek-V4", "Hybrid attention":
// partial RoPE on the last qk_rope_head_dim channels, interleaved pairs). The angle is formed
// and reduced in double precision so positions up to 2^20 keep fp32-accurate sines.
__device__ __forceinline__ void rope_cos_sin(double pos, int p, int r, double log2_theta, float *c, float *s)
{
    double freq = exp2(-(2.0 * p / (double)r) * log2_theta);
    double sd, cd;
    sincos(pos * freq, &sd, &cd);
    *c = (float)cd;
    *s = (float)sd;
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key); -0 maps like +0.
__device__ __forceinline__ uint32_t score_key(float x)
{
    uint32_t u = __float_as_uint(x + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- host: per-device settings done once -------------------------------------------------------

constexpr int kMaxDevices = 64;

// Device index and SM count of the current device (the count is queried once per device).
inline cudaError_t current_device_sms(int *dev, int *sms)
{
    static int cached[kMaxDevices];
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    if (*dev < 0 || *dev >= kMaxDevices) return cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, *dev);
    if (cached[*dev] == 0) {
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, *dev)) != cudaSuccess) return e;
        cached[*dev] = n;
    }
    *sms = cached[*dev];
    return cudaSuccess;
}

// Raise a kernel's dynamic shared-memory limit on the current device, once per (device, kernel) and
// only when a larger size than before is asked for.
inline cudaError_t ensure_smem_limit(const void *kernel, size_t bytes)
{
    static std::mutex mu;
    static std::unordered_map<const void *, int> done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    std::lock_guard<std::mutex> lock(mu);
    auto it = done[dev].find(kernel);
    if (it != done[dev].end() && it->second >= (int)bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done[dev][kernel] = (int)bytes;
    return e;
}

// ---- programmatic dependent launch ---------------------------------------------------------------
//
// A kernel launched with launch_dependent() may be scheduled while the kernel before it in the stream
// is still running: it runs its prologue, then grid_dependency_wait() blocks until that kernel has
// completed and its memory is visible. Every such kernel calls grid_dependency_wait() before it
// touches memory written earlier in the chain and before it can exit, so that its own completion still
// implies the completion of everything before it. Both device calls are no-ops when the kernel was
// launched the ordinary way.

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the next kernel in the stream (if launched with launch_dependent) start being scheduled.
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                    Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

__device__ __forceinline__ int64_t visible_entries(int64_t t, int m, int64_t T)
{
    int64_t v = (t + 1) / m;
    return v < T ? v : T;
}

}  // namespace csa
