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
// that device; that first call should come before any stream capture. All calls share the
// array, so calls that overlap on the GPU (other streams, other host threads) race.
#include <mutex>

#include "common.cuh"

namespace bakron {
namespace {

constexpr int kNoallocMaxN = 2048;
constexpr size_t kNoallocScratchBytes = (size_t)20 << 20;   // 20 MiB

static __device__ __align__(256) unsigned char g_ldl_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on first use).
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return BAKRON_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ldl_scratch) != cudaSuccess || !p) return BAKRON_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
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
    int e = scratch_address(&ws);
    if (e) return e;
    // The factorisation needs no part of its scratch to start at zero: every plane it reads is
    // written earlier in the same call.
    return bakron_ldl(H, n, L, D, ws, kNoallocScratchBytes, dev_status, stream);
}
