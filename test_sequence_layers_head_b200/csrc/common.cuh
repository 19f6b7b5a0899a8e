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
// CUDA's erff / expf (the fp32 CUDA-core path).
__device__ __forceinline__ float gelu_f(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float x) {
    const float Phi = 0.5f * (1.0f + erff(x * 0.70710678118654752f));
    const float phi = 0.39894228040143268f * expf(-0.5f * x * x);
    return Phi + x * phi;
}

// GELU'' = phi(x) (2 - x^2), the derivative of Phi + x phi (phi' = -x phi), for the
// backward of the MLP's GELU' term
__device__ __forceinline__ float gelu_grad2_f(float x) {
    return 0.39894228040143268f * expf(-0.5f * x * x) * (2.0f - x * x);
}

// GELU and GELU' together for the tensor-core MLP kernel: erf by the rational
// approximation of Abramowitz & Stegun, Handbook of Mathematical Functions,
// formula 7.1.26 (|error| <= 1.5e-7 for every argument), on z = |x| / sqrt(2);
// the factor exp(-z^2) it needs is also exp(-x^2 / 2) = sqrt(2 pi) phi(x), so
// one exponential serves Phi and phi.
__device__ __forceinline__ float gelu_phi_fast(float x, float& ez) {
    const float z = fabsf(x) * 0.70710678118654752f;
    const float t = __fdividef(1.f, fmaf(0.3275911f, z, 1.f));
    const float poly =
        t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, 1.061405429f, -1.453152027f), 1.421413741f), -0.284496736f), 0.254829592f);
    ez = __expf(-z * z);
    const float erf_abs = fmaf(-poly, ez, 1.f);   // erf(|x| / sqrt 2)
    return 0.5f * (1.f + copysignf(erf_abs, x));  // Phi(x)
}
__device__ __forceinline__ void gelu_and_grad_fast(float x, float& g, float& gp) {
    float ez;
    const float Phi = gelu_phi_fast(x, ez);
    g = x * Phi;
    gp = fmaf(x * 0.39894228040143268f, ez, Phi);   // Phi + x phi
}
__device__ __forceinline__ float gelu_fast(float x) {
    float ez;
    return x * gelu_phi_fast(x, ez);
}

}  // namespace ttt
