// decode_noalloc.cu -- csa_decode for callers that cannot allocate device memory.
//
// csa_decode needs device scratch (the per-entry index scores and the selected indices) and asks
// the caller for it. Some callers have no way to provide it: a host runtime that owns no CUDA
// allocator (all device memory was partitioned up front by someone else), or a serving loop that
// must not call cudaMalloc while other work is in flight because the call can synchronise the
// device and stall every stream. This entry point takes the scratch from a fixed array that lives
// inside the library instead, so the caller passes only its inputs and outputs.
//
// The array is a file-scope __device__ variable: each GPU that loads the library holds one copy
// of it until the process exits. Host code cannot use the array's name as a device address (it is
// a host-side stand-in), so the device address is looked up with cudaGetSymbolAddress, with the
// device current, the first time a CUDA context uses this entry point. The address belongs to that
// context: it is cached per device together with the context it was taken in (the driver's current
// context), and taken again when another context is current (after cudaDeviceReset, or under a
// caller that made its own context current).
#include <mutex>

#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;   // 16 MiB per GPU that loads the library
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

struct ScratchAddr {
    void *ctx;    // the driver context the address was taken in
    void *addr;
};
ScratchAddr g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

typedef int (*CtxGetCurrentFn)(void **);

// cuCtxGetCurrent through the runtime's driver entry point table (the library links no libcuda).
CtxGetCurrentFn ctx_get_current_fn()
{
    static CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<CtxGetCurrentFn>(p);
        return nullptr;
    }();
    return fn;
}

// Device address of the scratch array in the current device's current context.
csa_status scratch_on_current_device(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return CSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return CSA_ERR_UNSUPPORTED;
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (get_ctx == nullptr) return CSA_ERR_CUDA;
    void *ctx = nullptr;
    if (get_ctx(&ctx) != 0) return CSA_ERR_CUDA;   // null while no context is current on this thread yet
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (ctx == nullptr || g_scratch[dev].addr == nullptr || g_scratch[dev].ctx != ctx) {
        void *p = nullptr;
        // looks the symbol up in the current context, making the device's primary context current
        // first when none is
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) return CSA_ERR_CUDA;
        if (get_ctx(&ctx) != 0 || ctx == nullptr) return CSA_ERR_CUDA;
        g_scratch[dev].ctx = ctx;
        g_scratch[dev].addr = p;
    }
    *out = g_scratch[dev].addr;
    return CSA_OK;
}

}  // namespace

extern "C" {

size_t csa_decode_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

csa_status csa_decode_noalloc(const void *q, const void *qI, const float *w, const void *kI, const void *C,
                              const uint8_t *c8, const float *c8_scale, const void *c_rope, const void *win,
                              const float *sinks, int32_t B, int32_t H, int32_t D, int64_t T, int32_t HI, int32_t dI,
                              int32_t k, int32_t W, int32_t rope_dim, int64_t P, double theta_tok, double theta_cmp,
                              float softmax_scale, int32_t *idx_out, float *o, void *stream)
{
    if (B < 0 || T < 0 || k < 1) return CSA_ERR_INVALID_ARG;
    // sizes whose byte counts would overflow are refused before any size is computed
    if (!csa::decode_sizes_representable(B, T, k)) return CSA_ERR_INVALID_ARG;
    if (csa::decode_workspace_min(B, T, k) > kNoAllocScratchBytes) return CSA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const csa_status s = scratch_on_current_device(&scratch);
    if (s != CSA_OK) return s;
    // csa_decode zeroes the status word at the start of the scratch and writes every score, index
    // and attention partial it later reads, so nothing left over from an earlier call is used. It
    // takes as many attention splits per sequence as the rest of the array holds.
    return csa_decode(q, qI, w, kI, C, c8, c8_scale, c_rope, win, sinks, B, H, D, T, HI, dI, k, W, rope_dim, P,
                      theta_tok, theta_cmp, softmax_scale, idx_out, o, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
