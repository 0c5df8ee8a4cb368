// ldl_noalloc.cu -- bakron_ldl_noalloc: bakron_ldl with its scratch in a fixed device array.
//
// Some callers cannot allocate device memory where they factor a Hessian: a process whose
// framework allocator has already reserved the device's memory (a second allocator's
// cudaMalloc then fails or fragments it), a latency-critical loop that must not call
// cudaMalloc / cudaFree because they can synchronise the whole device, or a deployment that
// fixes all device memory when the library is loaded. For them this entry point takes only
// inputs and outputs and uses a scratch array that is part of the library image itself.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds it
// (kNoallocScratchBytes, 20 MiB) until the process exits. In host code the variable's name is
// only a host-side stand-in, not a device address, so the address is taken with
// cudaGetSymbolAddress once per device, with that device current, by the first call made on
// that device. The address belongs to the device's CUDA context: it is cached together with
// the context's unique id, and a call that finds another context current (the primary context
// was destroyed and created again, e.g. after cudaDeviceReset) looks it up again instead of
// using a stale address. A lookup is refused while the call's stream is capturing
// (BAKRON_ERR_CAPTURE): it may load the module, which a capture does not allow, so the first
// call on a device (or context) must come before any capture. All calls share the array, so
// calls that overlap on the GPU (other streams, other host threads) race.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace bakron {
namespace {

constexpr int kNoallocMaxN = 2048;
constexpr size_t kNoallocScratchBytes = (size_t)20 << 20;   // 20 MiB

static __device__ __align__(256) unsigned char g_ldl_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct CachedAddr {
    unsigned long long ctx_id;   // unique id of the context the address belongs to
    void* addr;
};
CachedAddr g_addr[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The unique id of the current context (0 when none is current or the query fails).
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array in the current device's current context (looked up on
// the first call in that context, never while `stream` is capturing).
int scratch_address(cudaStream_t stream, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return BAKRON_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long id = current_ctx_id();
    if (id != 0 && g_addr[dev].addr && g_addr[dev].ctx_id == id) {
        *out = g_addr[dev].addr;
        return BAKRON_OK;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return BAKRON_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return BAKRON_ERR_CAPTURE;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ldl_scratch) != cudaSuccess || !p) return BAKRON_ERR_CUDA;
    const unsigned long long id_now = current_ctx_id();   // the lookup made a context current
    g_addr[dev] = CachedAddr{id_now, id_now ? p : nullptr};
    *out = p;
    return BAKRON_OK;
}

}  // namespace
}  // namespace bakron

using namespace bakron;

extern "C" int bakron_ldl_noalloc_max_n(void) { return kNoallocMaxN; }

extern "C" int bakron_ldl_noalloc(const float* H, int n, float* L, float* D, int* dev_status,
                                  void* stream) {
    if (n < 1 || n > kNoallocMaxN || !H || !L || !D || !dev_status) return BAKRON_ERR_INVALID_ARG;
    const size_t need = bakron_ldl_workspace_bytes(n);
    if (need > kNoallocScratchBytes) return BAKRON_ERR_WORKSPACE;
    void* ws = nullptr;
    int e = scratch_address(static_cast<cudaStream_t>(stream), &ws);
    if (e) return e;
    // The factorisation needs no part of its scratch to start at zero: every plane it reads is
    // written earlier in the same call.
    return bakron_ldl(H, n, L, D, ws, kNoallocScratchBytes, dev_status, stream);
}
