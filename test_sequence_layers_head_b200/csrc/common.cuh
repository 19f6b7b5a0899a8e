// Shared definitions of the TTT CUDA library (device side).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/ttt.h"

namespace ttt {

// Bits of the per-device status word written by kernels.
enum : int { kStatusTimeout = 1, kStatusBadSmem = 2 };

// Default limit of one device-side wait.
constexpr unsigned kDefaultWaitMs = 2000;

// Storage types of Q/K/V/Z.
template <typename IO>
struct IoTraits;
template <>
struct IoTraits<float> {
    __device__ __forceinline__ static float load(const float* p, size_t i) { return p[i]; }
    __device__ __forceinline__ static void store(float* p, size_t i, float v) { p[i] = v; }
};
template <>
struct IoTraits<__nv_bfloat16> {
    __device__ __forceinline__ static float load(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
    __device__ __forceinline__ static void store(__nv_bfloat16* p, size_t i, float v) {
        p[i] = __float2bfloat16_rn(v);
    }
};

// Exact-erf GELU and its derivative (x Phi(x) and Phi(x) + x phi(x)), using
// CUDA's erff / expf.
__device__ __forceinline__ float gelu_f(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float x) {
    const float Phi = 0.5f * (1.0f + erff(x * 0.70710678118654752f));
    const float phi = 0.39894228040143268f * expf(-0.5f * x * x);
    return Phi + x * phi;
}

}  // namespace ttt
