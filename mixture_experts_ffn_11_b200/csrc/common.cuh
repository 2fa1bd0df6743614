// Shared definitions of the CUDA path: the device error word, bf16 packing, warp helpers.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "moe.h"
#include "sm100.cuh"

namespace moe {

// Device error word: kernels set MOE_DEVERR_* bits here instead of faulting. One per device (this
// translation unit holds every kernel of the library, so there is exactly one definition).
__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void flag_error(unsigned int bit) { atomicOr(&g_device_error, bit); }

// A pipeline wait gives up after this long and reports MOE_DEVERR_WAIT_TIMEOUT. No legitimate wait in
// these kernels lasts more than a few hundred microseconds. The limit is a device variable so that a test can
// shorten it (moe_test_set_wait); kernels read it when a wait does not succeed at once.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;
// Test hook (moe_test_set_wait): when non-zero, the MMA-issuing warp of each bf16 grouped GEMM first waits on a
// barrier that nothing arrives on, so the bounded wait runs out and the kernel takes its abort path.
__device__ int g_wait_stall = 0;

__device__ __forceinline__ uint64_t wait_limit_ns() { return *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns); }

// Bounded wait on an mbarrier phase. Returns false if `abort_flag` was raised by another role, or if
// the time limit passed (then it raises the flag and the error bit itself).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const uint32_t addr = smem_u32(bar);
    if (mbar_try_wait(addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = wait_limit_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(addr, parity)) return true;
        if ((spin & 63u) == 0u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit) {
                *abort_flag = 1;
                flag_error(MOE_DEVERR_WAIT_TIMEOUT);
                return false;
            }
        }
    }
}

// As mbar_wait_bounded, for a role that is off the critical path (a warp waiting a whole tile for its turn): it
// sleeps `sleep_ns` between polls instead of spinning, leaving issue slots to the warps that do the work.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  unsigned sleep_ns) {
    const uint32_t addr = smem_u32(bar);
    if (mbar_try_wait(addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = wait_limit_ns();
    for (;;) {
        __nanosleep(sleep_ns);
        if (mbar_try_wait(addr, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit) {
            *abort_flag = 1;
            flag_error(MOE_DEVERR_WAIT_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait without an abort flag (used while draining on the way out).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint32_t addr = smem_u32(bar);
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = wait_limit_ns();
    while (!mbar_try_wait(addr, parity)) {
        if (globaltimer_ns() - t0 > limit) {
            flag_error(MOE_DEVERR_WAIT_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Test hook: with g_wait_stall set, wait (bounded) on `never_bar`, a barrier initialised with one expected
// arrival that nothing ever gives, and return false when the wait runs out; otherwise return true at once.
__device__ __forceinline__ bool test_stall(uint64_t* never_bar, volatile int* abort_flag) {
    if (*reinterpret_cast<volatile int*>(&g_wait_stall) == 0) return true;
    return mbar_wait_bounded(never_bar, 0, abort_flag);
}

// Programmatic dependent launch. The library launches its kernels so that the next kernel in a stream may
// start while this one finishes: grid_dep_wait() returns once every earlier kernel in the stream has completed
// and its memory writes are visible (a no-op when the kernel was launched without the attribute). A kernel reads
// and writes global memory only after it; what comes before is prologue (barrier setup, TMEM allocation, tensor
// map prefetch). grid_dep_trigger() allows the next kernel's CTAs to be launched; they take SMs as they free up.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace moe
