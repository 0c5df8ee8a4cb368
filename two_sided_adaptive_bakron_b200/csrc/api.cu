// api.cu -- status helpers and library-wide settings of the BaKron C ABI.
#include <cstdlib>

#include "common.cuh"

namespace bakron {

uint64_t spin_limit_ns() {
    // Default: 4 s per dependency wait, far above any legitimate wait of a solve.
    static const uint64_t v = [] {
        const char* s = std::getenv("BAKRON_SPIN_LIMIT_NS");
        if (s && *s) {
            const long long x = std::atoll(s);
            if (x > 0) return (uint64_t)x;
        }
        return (uint64_t)4000000000ULL;
    }();
    return v;
}

static unsigned long long g_launches = 0;
void count_launches(long long k) { __atomic_fetch_add(&g_launches, (unsigned long long)k, __ATOMIC_RELAXED); }

}  // namespace bakron

extern "C" unsigned long long bakron_kernel_launches(void) {
    return __atomic_load_n(&bakron::g_launches, __ATOMIC_RELAXED);
}

extern "C" int bakron_read_status(const int* dev_status, void* stream) {
    if (!dev_status) return BAKRON_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int h = 0;
    if (cudaMemcpyAsync(&h, dev_status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return BAKRON_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BAKRON_ERR_CUDA;
    return h;
}

extern "C" const char* bakron_status_string(int code) {
    switch (code) {
        case BAKRON_OK: return "ok";
        case BAKRON_ERR_INVALID_ARG: return "invalid argument";
        case BAKRON_ERR_NOT_PD: return "matrix not positive definite (pivot <= 0 or non-finite)";
        case BAKRON_ERR_CUDA: return "CUDA error";
        case BAKRON_ERR_TIMEOUT: return "device-side dependency wait timed out";
        case BAKRON_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case BAKRON_ERR_NONFINITE: return "non-finite value on the device";
        case BAKRON_ERR_CAPTURE: return "set-up step refused under stream capture";
        default: return "unknown status";
    }
}

extern "C" int bakron_version(void) { return 200; }
