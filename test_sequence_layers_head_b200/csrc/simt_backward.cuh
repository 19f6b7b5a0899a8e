// fp32 CUDA-core kernel of the TTT-Linear backward (no LN): the outer-loop
// gradients of the prefill (paper digest "论文速览 | TTT", section 3.4: the
// outer loop's gradients pass through the inner loop's updates; section
// 6.12: only the state at each mini-batch boundary is kept, kappa = T/b
// states, and everything inside a mini-batch is recomputed).
//
// Per mini-batch, in the dual form of section 3.6 with W the batch-start
// state, A = diag(eta) E and M = tril(Q K^T) (causal mask s <= t):
//     E = K W - V,   Z = Q W - M A,   W_next = W - K^T A.
// Given dZ and G = dL/dW_next, the reverse step is
//     P  = mask(dZ A^T)                         (b x b)
//     dA = -M^T dZ - K G,   dE = diag(eta) dA,   deta_s = dA_s . E_s
//     dQ = dZ W^T - P K
//     dK = -P^T Q - A G^T + dE W^T
//     dV = -dE
//     dL/dW = G + Q^T dZ + K^T dE
// and the mini-batches are visited last to first, G starting at dL/dW_out.
// The batch-start states come from the forward (its W_states output).
//
// One CTA per (sequence, head) unit; W, G and the mini-batch's tiles live in
// shared memory.
#pragma once
#include "common.cuh"
#include "simt.cuh"

namespace ttt {

struct SimtBackwardParams {
    int H, T, b;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W_states;   // [units, T/b, D, D]
    const void* dZ;          // [units, T, D] or null (zero)
    const float* dW_out;     // [units, D, D] or null (zero)
    void* dQ;
    void* dK;
    void* dV;
    float* deta;             // [units, T] or null (not wanted)
    float* dW0;              // [units, D, D]
};

inline size_t simt_backward_smem(int D, int b) {
    return sizeof(float) * (2 * (size_t)D * D + 5 * (size_t)b * D + 2 * (size_t)b * b + (size_t)b);
}

template <int D, typename IO>
__global__ void __launch_bounds__(kSimtThreads) simt_linear_backward_kernel(SimtBackwardParams p) {
    extern __shared__ __align__(16) float sm[];
    const int b = p.b;
    float* W = sm;               // D*D   batch-start state
    float* G = W + D * D;        // D*D   dL/d(state after the batch), then before it
    float* Kt = G + D * D;       // b*D
    float* Qt = Kt + b * D;      // b*D
    float* Et = Qt + b * D;      // b*D   V, then E
    float* dZt = Et + b * D;     // b*D
    float* dA = dZt + b * D;     // b*D   dA, then dE
    float* M = dA + b * D;       // b*b   tril(Q K^T)
    float* P = M + b * b;        // b*b   mask(dZ A^T)
    float* et = P + b * b;       // b
    const int tid = threadIdx.x;
    const int warp = tid / 32, lane = tid % 32, nwarps = kSimtThreads / 32;
    const int unit = blockIdx.x;
    const int nb = p.T / b;
    const size_t tok = (size_t)unit * p.T * D;
    const IO* Q = static_cast<const IO*>(p.Q) + tok;
    const IO* K = static_cast<const IO*>(p.K) + tok;
    const IO* V = static_cast<const IO*>(p.V) + tok;
    const IO* dZ = p.dZ ? static_cast<const IO*>(p.dZ) + tok : nullptr;
    IO* dQ = static_cast<IO*>(p.dQ) + tok;
    IO* dK = static_cast<IO*>(p.dK) + tok;
    IO* dV = static_cast<IO*>(p.dV) + tok;
    for (int e = tid; e < D * D; e += kSimtThreads) G[e] = p.dW_out ? p.dW_out[(size_t)unit * D * D + e] : 0.f;
    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * b;
        const float* Ws = p.W_states + ((size_t)unit * nb + i) * D * D;
        for (int e = tid; e < D * D; e += kSimtThreads) W[e] = Ws[e];
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const size_t g = (size_t)t0 * D + e;
            Kt[e] = IoTraits<IO>::load(K, g);
            Qt[e] = IoTraits<IO>::load(Q, g);
            Et[e] = IoTraits<IO>::load(V, g);
            dZt[e] = dZ ? IoTraits<IO>::load(dZ, g) : 0.f;
        }
        for (int t = tid; t < b; t += kSimtThreads)
            et[t] = p.eta ? p.eta[(size_t)unit * p.T + t0 + t] : p.eta_const;
        __syncthreads();
        // E = K W - V ;  M = tril(Q K^T)
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int t = e / D, j = e % D;
            float acc = 0.f;
#pragma unroll 8
            for (int a = 0; a < D; ++a) acc += Kt[t * D + a] * W[a * D + j];
            Et[e] = acc - Et[e];
        }
        for (int e = tid; e < b * b; e += kSimtThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t) {
#pragma unroll 8
                for (int a = 0; a < D; ++a) acc += Qt[t * D + a] * Kt[s * D + a];
            }
            M[e] = acc;
        }
        __syncthreads();
        // P = mask(dZ A^T) ;  dA = -M^T dZ - K G
        for (int e = tid; e < b * b; e += kSimtThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t) {
#pragma unroll 8
                for (int j = 0; j < D; ++j) acc += dZt[t * D + j] * Et[s * D + j];
                acc *= et[s];
            }
            P[e] = acc;
        }
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int s = e / D, j = e % D;
            float acc = 0.f;
            for (int t = s; t < b; ++t) acc += M[t * b + s] * dZt[t * D + j];
#pragma unroll 8
            for (int a = 0; a < D; ++a) acc += Kt[s * D + a] * G[a * D + j];
            dA[e] = -acc;
        }
        __syncthreads();
        // deta_s = dA_s . E_s ; dE = diag(eta) dA ; dV = -dE
        for (int s = warp; s < b; s += nwarps) {
            float acc = 0.f;
            for (int j = lane; j < D; j += 32) acc += dA[s * D + j] * Et[s * D + j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0 && p.deta) p.deta[(size_t)unit * p.T + t0 + s] = acc;
            for (int j = lane; j < D; j += 32) {
                const float de = et[s] * dA[s * D + j];
                dA[s * D + j] = de;
                IoTraits<IO>::store(dV, (size_t)(t0 + s) * D + j, -de);
            }
        }
        __syncthreads();
        // dQ = dZ W^T - P K ;  dK = -P^T Q - A G^T + dE W^T   (G is still dL/dW_next)
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int t = e / D, a = e % D;
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; ++j) acc += dZt[t * D + j] * W[a * D + j];
            for (int s = 0; s <= t; ++s) acc -= P[t * b + s] * Kt[s * D + a];
            IoTraits<IO>::store(dQ, (size_t)(t0 + t) * D + a, acc);
        }
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int s = e / D, a = e % D;
            float acc = 0.f;
            for (int t = s; t < b; ++t) acc -= P[t * b + s] * Qt[t * D + a];
            float ag = 0.f, dw = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; ++j) {
                ag += Et[s * D + j] * G[a * D + j];
                dw += dA[s * D + j] * W[a * D + j];
            }
            IoTraits<IO>::store(dK, (size_t)(t0 + s) * D + a, acc - et[s] * ag + dw);
        }
        __syncthreads();
        // dL/dW = G + Q^T dZ + K^T dE
        for (int e = tid; e < D * D; e += kSimtThreads) {
            const int a = e / D, j = e % D;
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += Qt[t * D + a] * dZt[t * D + j] + Kt[t * D + a] * dA[t * D + j];
            G[e] += acc;
        }
        __syncthreads();
    }
    for (int e = tid; e < D * D; e += kSimtThreads) p.dW0[(size_t)unit * D * D + e] = G[e];
}

}  // namespace ttt
