// common.cuh -- small device helpers shared by the kernels of libgdn.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// Device status word: the first bounded wait that gives up records its code
// here (never overwritten until read and cleared by gdn_device_status).
__device__ unsigned int g_status_word;

__device__ __forceinline__ void record_status(unsigned code) {
    atomicCAS(&g_status_word, 0u, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// softplus at beta = 1 with the strict threshold 20, on an fp32 argument,
// evaluated in fp64 (log1p keeps the far-negative tail).
__device__ __forceinline__ double softplus_f64(float x) {
    return (x > 20.0f) ? (double)x : log1p(exp((double)x));
}

// g = -exp(A_log) * softplus(a + dt_bias): one fp32 add, fp64 transcendentals,
// one rounding to fp32.
__device__ __forceinline__ float decay_gate(float a, float dt_bias, float A_log) {
    float x = __fadd_rn(a, dt_bias);
    return __double2float_rn(-exp((double)A_log) * softplus_f64(x));
}

// beta = sigmoid(b) in fp64, rounded once.
__device__ __forceinline__ float write_gate(float b) {
    return __double2float_rn(1.0 / (1.0 + exp(-(double)b)));
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar_addr), "r"(phase)
        : "memory");
    return ok != 0;
}

// Bounded wait on the given phase parity.  Returns false (and records
// GDN_ERR_TIMEOUT) after `polls` unsuccessful polls; each poll is itself
// bounded by the hardware's try_wait time limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase, uint32_t polls) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t i = 0; i < polls; ++i)
        if (mbar_try_wait(a, phase)) return true;
    record_status(GDN_ERR_TIMEOUT);
    return false;
}

}  // namespace gdn
