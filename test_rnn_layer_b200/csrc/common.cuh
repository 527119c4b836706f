// Device-side helpers shared by the TTT-MLP kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace ttt {


// erf-GELU and its derivative (paper notes page, "关键设计 / TTT-MLP 层": the
// hidden MLP uses GELU; the erf form is the exact one).  erff/expf are the
// CUDA math library's; 1/sqrt(2) and 1/sqrt(2 pi) are plain constants.
__device__ __forceinline__ float gelu(float a) {
    return 0.5f * a * (1.0f + erff(a * 0.70710678118654752f));
}

__device__ __forceinline__ void gelu_and_prime(float a, float& g, float& gp) {
    const float Phi = 0.5f * (1.0f + erff(a * 0.70710678118654752f));
    const float phi = 0.39894228040143268f * expf(-0.5f * a * a);
    g = a * Phi;
    gp = Phi + a * phi;
}

__device__ __forceinline__ float load_elem(const void* p, long long idx, int is_bf16) {
    if (is_bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[idx]);
    return reinterpret_cast<const float*>(p)[idx];
}

__device__ __forceinline__ void store_elem(void* p, long long idx, int is_bf16, float v) {
    if (is_bf16) reinterpret_cast<__nv_bfloat16*>(p)[idx] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(p)[idx] = v;
}

}  // namespace ttt
