// nvfp4kv_pipeline.cuh -- mbarrier waits and arrivals shared by the
// warp-specialized tensor-core kernels (decode and chunked-prefill
// attention).  Every wait is bounded: after a number of sleeping polls it
// sets the CTA's abort flag and reports NVFP4_ERR_TIMEOUT, so a stalled
// pipeline ends with an error status instead of hanging the GPU.
#pragma once

#include <cstdint>

#include "nvfp4kv_device.cuh"

namespace nvfp4kv {

// non-blocking test of the phase with the given parity
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait of one thread: gives up when the CTA's abort flag is set or
// after `polls` sleeping polls (then sets the flag and reports a timeout).
// Inlined: a call would spill the live registers of the caller.
__device__ __forceinline__ bool wait_one(uint64_t* bar, uint32_t parity, int32_t* abort_flag,
                                         int32_t* status, uint32_t polls) {
    if (mbar_test_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < polls; ++i) {
        if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
        if (*reinterpret_cast<volatile int32_t*>(abort_flag)) return false;
    }
    atomicExch(abort_flag, 1);
    report(status, NVFP4_ERR_TIMEOUT);
    return false;
}

// The same for a whole warp; the result is warp-uniform.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, int32_t* abort_flag,
                                          int32_t* status, uint32_t polls) {
    const bool ok = wait_one(bar, parity, abort_flag, status, polls);
    return __all_sync(0xFFFFFFFFu, ok);
}

}  // namespace nvfp4kv
