// common.cuh -- shared device/host helpers of the BaKron CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include "bakron.h"

namespace bakron {

constexpr size_t kWsAlign = 256;

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Carves aligned sub-buffers out of a caller-provided workspace.
struct WsCarver {
    char* base;
    size_t off;
    __host__ explicit WsCarver(void* p) : base(static_cast<char*>(p)), off(0) {}
    template <typename T>
    __host__ T* take(size_t count) {
        off = align_up(off, kWsAlign);
        T* p = reinterpret_cast<T*>(base + off);
        off += count * sizeof(T);
        return p;
    }
};

// Host-side size accounting that mirrors WsCarver::take.
struct WsSizer {
    size_t off = 0;
    template <typename T>
    void take(size_t count) {
        off = align_up(off, kWsAlign);
        off += count * sizeof(T);
    }
    size_t bytes() const { return align_up(off, kWsAlign) + kWsAlign; }
};

// ------------------------------------------------------------------------------ device status
// First error wins: the status word only moves away from BAKRON_OK once.
__device__ __forceinline__ void set_status(int* status, int code) {
    atomicCAS(status, (int)BAKRON_OK, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(int* p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait until *flag != 0. Returns false when the wait gave up: either the time limit
// passed (the status word gets BAKRON_ERR_TIMEOUT and the abort word is raised so that every
// other block stops too) or another block already raised the abort word.
__device__ __forceinline__ bool wait_flag(const int* flag, int* abort_word, int* status,
                                          uint64_t limit_ns) {
    if (ld_acquire_gpu(flag) != 0) return true;
    const uint64_t t0 = globaltimer_ns();
    unsigned ns = 32;
    while (true) {
        if (ld_acquire_gpu(flag) != 0) return true;
        if (ld_acquire_gpu(abort_word) != 0) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            set_status(status, BAKRON_ERR_TIMEOUT);
            atomicExch(abort_word, 1);
            return false;
        }
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
    }
}

// Bounded wait until *counter >= target; same give-up rules as wait_flag.
__device__ __forceinline__ bool wait_geq(const int* counter, int target, int* abort_word,
                                         int* status, uint64_t limit_ns) {
    if (ld_acquire_gpu(counter) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    unsigned ns = 32;
    while (true) {
        if (ld_acquire_gpu(counter) >= target) return true;
        if (ld_acquire_gpu(abort_word) != 0) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            set_status(status, BAKRON_ERR_TIMEOUT);
            atomicExch(abort_word, 1);
            return false;
        }
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
    }
}

__device__ __forceinline__ void red_add_release_gpu(int* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_add_f32(float* p, float v) {
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// Default limit of one dependency wait; BAKRON_SPIN_LIMIT_NS in the environment overrides it
// (used by the tests to exercise the timeout path without hanging anything).
uint64_t spin_limit_ns();

// Counts the kernels this library has launched in this process (diagnostics).
void count_launches(long long k);

inline int cuda_err(cudaError_t e) { return e == cudaSuccess ? BAKRON_OK : BAKRON_ERR_CUDA; }

inline bool ws_ok(const void* ws, size_t have, size_t need) {
    return ws != nullptr && have >= need &&
           (reinterpret_cast<uintptr_t>(ws) % kWsAlign) == 0;
}

}  // namespace bakron
