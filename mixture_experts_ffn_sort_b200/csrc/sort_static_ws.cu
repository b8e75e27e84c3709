// sort_static_ws.cu -- moe_sort with scratch owned by the library
// (moe_sort_static_ws).
//
// For callers that cannot allocate device memory, the sort's scratch (the
// per-chunk expert counters of its multi-kernel path) lives in a file-scope
// __device__ array instead of a caller-provided workspace.  Its device address
// is looked up with cudaGetSymbolAddress once per device and context (the
// first call on a device, or the first after that device's context was
// replaced, e.g. by cudaDeviceReset); the array's host-side name is only a
// stand-in and is never passed to a kernel.
#include <stdio.h>

#include <mutex>

#include "../../include/moe_ffn.h"
#include "launch.h"

namespace moe {
int api_error(int code, const char* msg);
void api_clear_error();
}  // namespace moe

namespace {

constexpr size_t kScratchBytes = MOE_SORT_STATIC_WS_BYTES;
__device__ __align__(256) unsigned char g_sort_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Per device: the context the address was looked up in, and the address.
struct ScratchSlot {
    CUcontext ctx;
    void* ptr;
};
ScratchSlot g_slot[kMaxDevices];

int err(int code, const char* fmt, long a = 0, long b = 0) {
    char buf[256];
    snprintf(buf, sizeof buf, fmt, a, b);
    return moe::api_error(code, buf);
}

// The driver's cuCtxGetCurrent, fetched through the runtime (the library does
// not link libcuda); NULL if the driver does not provide it.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
    static std::once_flag once;
    static CtxGetCurrentFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

CUcontext current_context() {
    CUcontext c = nullptr;
    CtxGetCurrentFn fn = ctx_get_current();
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// Device address of g_sort_scratch on the current device, looked up again
// whenever the current context is not the one of the cached address.
int scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return moe::api_error(MOE_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return err(MOE_ERR_CUDA, "moe_sort_static_ws: device %ld out of range", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    ScratchSlot& slot = g_slot[dev];
    const CUcontext ctx = current_context();
    if (!slot.ptr || !ctx || slot.ctx != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_sort_scratch);
        if (e != cudaSuccess || !p)
            return moe::api_error(MOE_ERR_CUDA, e != cudaSuccess ? cudaGetErrorString(e)
                                                                 : "cudaGetSymbolAddress returned NULL");
        slot.ptr = p;
        slot.ctx = current_context();  // the lookup has made the device's context current
    }
    *out = slot.ptr;
    return MOE_OK;
}

}  // namespace

extern "C" MOE_API int moe_sort_static_ws(const int32_t* topk_ids, int T, int K, int E, int32_t* expert_offsets,
                                          int32_t* sorted_route, int32_t* inv_route, int32_t* status,
                                          moe_stream_t stream) {
    moe::api_clear_error();
    if (T < 0 || T > MOE_MAX_T) return err(MOE_ERR_INVALID_ARG, "moe_sort_static_ws: T=%ld out of range", T);
    if (E < 1 || E > MOE_MAX_E)
        return err(MOE_ERR_UNSUPPORTED_SHAPE, "moe_sort_static_ws: num_experts=%ld must be in 1..=%ld", E, MOE_MAX_E);
    if (K < 1 || K > MOE_MAX_K)
        return err(MOE_ERR_INVALID_ARG, "moe_sort_static_ws: top_k=%ld must be in 1..=%ld", K, MOE_MAX_K);
    if (!expert_offsets || (T > 0 && (!topk_ids || !sorted_route || !inv_route)))
        return err(MOE_ERR_INVALID_ARG, "moe_sort_static_ws: NULL tensor pointer");
    const uintptr_t mis = reinterpret_cast<uintptr_t>(topk_ids) | reinterpret_cast<uintptr_t>(expert_offsets) |
                          reinterpret_cast<uintptr_t>(sorted_route) | reinterpret_cast<uintptr_t>(inv_route);
    if ((mis & 15u) || (reinterpret_cast<uintptr_t>(status) & 3u))
        return err(MOE_ERR_MISALIGNED,
                   "moe_sort_static_ws: tensor bases must be 16-byte aligned and status 4-byte aligned");
    const long R = static_cast<long>(T) * K;
    const size_t need = moe::sort_workspace_bytes(R, E);
    if (need > kScratchBytes)
        return err(MOE_ERR_UNSUPPORTED_SHAPE,
                   "moe_sort_static_ws: this size needs %ld bytes of scratch; the library's array holds %ld "
                   "(use moe_sort with a workspace)",
                   static_cast<long>(need), static_cast<long>(kScratchBytes));
    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != MOE_OK) return rc;
    cudaError_t e;
    if (T == 0)
        e = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), stream);
    else
        e = moe::launch_sort(topk_ids, R, E, expert_offsets, sorted_route, inv_route, scratch, status, stream);
    if (e != cudaSuccess) return moe::api_error(MOE_ERR_CUDA, cudaGetErrorString(e));
    return MOE_OK;
}
