// fp32 CUDA-core kernels of the TTT inner-loop forward (dual form).
//
// One CTA per (sequence, head) unit; the state lives in shared memory for
// the whole sequence.  These kernels serve the fp32 workloads (where the
// tolerance is tighter than bf16 tensor-core operands allow), head dims the
// tensor-core kernels do not cover, and any mini-batch size b <= 64.
//
// Per mini-batch (paper digest "论文速览 | TTT", sections 3.6-3.7):
//   linear:  E = K W0 - V;  Z = Q W0 - (tril(Q K^T) * eta_s) E;  W -= K^T diag(eta) E
//   LN+res:  Y = K W0 + c; Delta = LN backward of 1/2||K + LN(Y) - V||^2;
//            Z = Q + LN(Q W0 + c - (tril(Q K^T + 1) * eta_s) Delta);
//            W -= K^T diag(eta) Delta;  c -= eta^T Delta
//   MLP:     A = K W1 + c1, Hk = GELU(A), E = Hk W2 + c2 - V,
//            D1 = (E W2^T) * GELU'(A),
//            Aq = Q W1 + c1 - (tril(Q K^T + 1) * eta_s) D1, Hq = GELU(Aq),
//            Z = Hq W2 + c2 - (tril(Hq Hk^T + 1) * eta_s) E,
//            W1 -= K^T diag(eta) D1, c1 -= eta^T D1, W2 -= Hk^T diag(eta) E, c2 -= eta^T E
#pragma once
#include "common.cuh"

namespace ttt {

constexpr int kSimtThreads = 256;

struct SimtLinearParams {
    int H, T, b;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W0;
    long long W0_bstride;
    const float* c0;
    long long c0_bstride;
    const float* gamma;
    const float* beta;
    float eps;
    void* Z;           // null: only the state is computed (no outputs)
    float* W_out;
    float* c_out;
    float* W_states;   // optional [units, T/b, D, D]: the state at the start of every mini-batch
    float* c_states;   // LN, with W_states: [units, T/b, D], the bias at the start of every mini-batch
};

// Row statistics helper: LN over n features of row `row` (warp-cooperative).
// Returns mean and 1/sqrt(var + eps) to every lane.
__device__ __forceinline__ void warp_ln_stats(const float* row, int n, float eps, float& mu, float& r) {
    float s = 0.f;
    for (int j = threadIdx.x % 32; j < n; j += 32) s += row[j];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    mu = s / n;
    float v = 0.f;
    for (int j = threadIdx.x % 32; j < n; j += 32) {
        const float t = row[j] - mu;
        v += t * t;
    }
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    r = rsqrtf(v / n + eps);
}

template <int D, bool LN, typename IO>
__global__ void __launch_bounds__(kSimtThreads) simt_linear_kernel(SimtLinearParams p) {
    extern __shared__ __align__(16) float sm[];
    const int b = p.b;
    float* W = sm;               // D*D
    float* c = W + D * D;        // D
    float* Kt = c + D;           // b*D
    float* Qt = Kt + b * D;      // b*D
    float* Vt = Qt + b * D;      // b*D  (later: Delta)
    float* Yt = Vt + b * D;      // b*D  (Y, then Zpre)
    float* S = Yt + b * D;       // b*b
    float* et = S + b * b;       // b
    float* stat = et + b;        // 2*b  (mu, r) per row
    const int tid = threadIdx.x;
    const int unit = blockIdx.x;
    const int n = unit / p.H, h = unit % p.H;
    const IO* Q = static_cast<const IO*>(p.Q) + (size_t)unit * p.T * D;
    const IO* K = static_cast<const IO*>(p.K) + (size_t)unit * p.T * D;
    const IO* V = static_cast<const IO*>(p.V) + (size_t)unit * p.T * D;
    IO* Z = static_cast<IO*>(p.Z) + (size_t)unit * p.T * D;
    const float* W0 = p.W0 + (size_t)n * p.W0_bstride + (size_t)h * D * D;
    for (int e = tid; e < D * D; e += kSimtThreads) W[e] = W0[e];
    if (LN) {
        for (int j = tid; j < D; j += kSimtThreads)
            c[j] = p.c0 ? p.c0[(size_t)n * p.c0_bstride + (size_t)h * D + j] : 0.f;
    }
    const float* gam = LN ? p.gamma + (size_t)h * D : nullptr;
    const float* bet = LN ? p.beta + (size_t)h * D : nullptr;
    const int warp = tid / 32, nwarps = kSimtThreads / 32;
    __syncthreads();
    for (int t0 = 0; t0 < p.T; t0 += b) {
        if (p.W_states) {
            float* ws = p.W_states + ((size_t)unit * (p.T / b) + t0 / b) * D * D;
            for (int e = tid; e < D * D; e += kSimtThreads) ws[e] = W[e];
            if (LN) {
                float* cs = p.c_states + ((size_t)unit * (p.T / b) + t0 / b) * D;
                for (int j = tid; j < D; j += kSimtThreads) cs[j] = c[j];
            }
        }
        // load the mini-batch
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const size_t g = (size_t)t0 * D + e;
            Kt[e] = IoTraits<IO>::load(K, g);
            Qt[e] = IoTraits<IO>::load(Q, g);
            Vt[e] = IoTraits<IO>::load(V, g);
        }
        for (int t = tid; t < b; t += kSimtThreads)
            et[t] = p.eta ? p.eta[(size_t)unit * p.T + t0 + t] : p.eta_const;
        __syncthreads();
        // Y = K W0 (+ c)
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int t = e / D, j = e % D;
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < D; ++i) acc += Kt[t * D + i] * W[i * D + j];
            Yt[e] = LN ? acc + c[j] : acc;
        }
        // S = tril(Q K^T (+1)) * eta_s
        for (int e = tid; p.Z && e < b * b; e += kSimtThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t) {
#pragma unroll 8
                for (int i = 0; i < D; ++i) acc += Qt[t * D + i] * Kt[s * D + i];
                if (LN) acc += 1.f;
                acc *= et[s];
            }
            S[e] = acc;
        }
        __syncthreads();
        if (!LN) {
            for (int e = tid; e < b * D; e += kSimtThreads) Vt[e] = Yt[e] - Vt[e];  // Delta = E
        } else {
            for (int t = warp; t < b; t += nwarps) {
                float mu, r;
                warp_ln_stats(Yt + t * D, D, p.eps, mu, r);
                // g = gamma * e, e = k + gamma*xh + beta - v
                float s1 = 0.f, s2 = 0.f;
                for (int j = tid % 32; j < D; j += 32) {
                    const float xh = (Yt[t * D + j] - mu) * r;
                    const float e = Kt[t * D + j] + gam[j] * xh + bet[j] - Vt[t * D + j];
                    const float g = gam[j] * e;
                    s1 += g;
                    s2 += g * xh;
                }
                for (int o = 16; o > 0; o >>= 1) {
                    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
                }
                s1 /= D;
                s2 /= D;
                for (int j = tid % 32; j < D; j += 32) {
                    const float xh = (Yt[t * D + j] - mu) * r;
                    const float e = Kt[t * D + j] + gam[j] * xh + bet[j] - Vt[t * D + j];
                    const float g = gam[j] * e;
                    Vt[t * D + j] = r * (g - s1 - xh * s2);  // Delta
                }
            }
        }
        __syncthreads();
        // Zpre = Q W0 (+ c) - S Delta
        for (int e = tid; p.Z && e < b * D; e += kSimtThreads) {
            const int t = e / D, j = e % D;
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < D; ++i) acc += Qt[t * D + i] * W[i * D + j];
            float corr = 0.f;
            for (int s = 0; s <= t; ++s) corr += S[t * b + s] * Vt[s * D + j];
            Yt[e] = (LN ? acc + c[j] : acc) - corr;
        }
        __syncthreads();
        if (!p.Z) {
        } else if (!LN) {
            for (int e = tid; e < b * D; e += kSimtThreads) IoTraits<IO>::store(Z, (size_t)t0 * D + e, Yt[e]);
        } else {
            for (int t = warp; t < b; t += nwarps) {
                float mu, r;
                warp_ln_stats(Yt + t * D, D, p.eps, mu, r);
                for (int j = tid % 32; j < D; j += 32) {
                    const float z = Qt[t * D + j] + gam[j] * (Yt[t * D + j] - mu) * r + bet[j];
                    IoTraits<IO>::store(Z, (size_t)(t0 + t) * D + j, z);
                }
            }
        }
        // W -= K^T diag(eta) Delta ; c -= eta^T Delta
        for (int e = tid; e < D * D; e += kSimtThreads) {
            const int i = e / D, j = e % D;
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += Kt[t * D + i] * et[t] * Vt[t * D + j];
            W[e] -= acc;
        }
        if (LN) {
            for (int j = tid; j < D; j += kSimtThreads) {
                float acc = 0.f;
                for (int t = 0; t < b; ++t) acc += et[t] * Vt[t * D + j];
                c[j] -= acc;
            }
        }
        __syncthreads();
    }
    for (int e = tid; e < D * D; e += kSimtThreads) p.W_out[(size_t)unit * D * D + e] = W[e];
    if (LN && p.c_out)
        for (int j = tid; j < D; j += kSimtThreads) p.c_out[(size_t)unit * D + j] = c[j];
}

inline size_t simt_linear_smem(int D, int b) {
    return sizeof(float) * ((size_t)D * D + D + 5 * (size_t)b * D + (size_t)b * b + 3 * (size_t)b);
}

// ---------------------------------------------------------------------------
// MLP
// ---------------------------------------------------------------------------
struct SimtMlpParams {
    int H, T, b;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W1;
    const float* c1;
    const float* W2;
    const float* c2;
    int per_seq;
    void* Z;
    float* W1_out;
    float* c1_out;
    float* W2_out;
    float* c2_out;
    const float* gamma;   // LN+residual on the output layer: [H, D]
    const float* beta;
    float eps;
    float* W_states;      // [units, T / b, 2 D M + M + D] batch-start states (W1, c1, W2, c2), or null
};

// LN = true: f(x) = x + gamma LN(GELU(x W1 + c1) W2 + c2) + beta; the residual E of
// layer 2 is replaced by the LN+residual backward Delta2 (as in the linear model),
// and the outputs pass through the same LN and residual.
template <int D, typename IO, bool LN>
__global__ void __launch_bounds__(kSimtThreads) simt_mlp_kernel(SimtMlpParams p) {
    constexpr int M = 4 * D;
    extern __shared__ __align__(16) float sm[];
    const int b = p.b;
    float* W1 = sm;              // D*M
    float* W2 = W1 + D * M;      // M*D
    float* c1 = W2 + M * D;      // M
    float* c2 = c1 + M;          // D
    float* Kt = c2 + D;          // b*D
    float* Qt = Kt + b * D;      // b*D
    float* Et = Qt + b * D;      // b*D  (V, then E)
    float* At = Et + b * D;      // b*M  (A, then D1)
    float* Hk = At + b * M;      // b*M
    float* Hq = Hk + b * M;      // b*M  (Aq, then Hq)
    float* S = Hq + b * M;       // b*b
    float* et = S + b * b;       // b
    float* Yt = et + b;          // b*D  (LN: pre-activation of the output layer)
    const int tid = threadIdx.x;
    const int warp = tid / 32, nwarps = kSimtThreads / 32;
    const int unit = blockIdx.x;
    const int pu = p.per_seq ? unit : unit % p.H;
    const float* gam = LN ? p.gamma + (size_t)(unit % p.H) * D : nullptr;
    const float* bet = LN ? p.beta + (size_t)(unit % p.H) * D : nullptr;
    const IO* Q = static_cast<const IO*>(p.Q) + (size_t)unit * p.T * D;
    const IO* K = static_cast<const IO*>(p.K) + (size_t)unit * p.T * D;
    const IO* V = static_cast<const IO*>(p.V) + (size_t)unit * p.T * D;
    IO* Z = static_cast<IO*>(p.Z) + (size_t)unit * p.T * D;
    for (int e = tid; e < D * M; e += kSimtThreads) {
        W1[e] = p.W1[(size_t)pu * D * M + e];
        W2[e] = p.W2[(size_t)pu * M * D + e];
    }
    for (int e = tid; e < M; e += kSimtThreads) c1[e] = p.c1 ? p.c1[(size_t)pu * M + e] : 0.f;
    for (int e = tid; e < D; e += kSimtThreads) c2[e] = p.c2 ? p.c2[(size_t)pu * D + e] : 0.f;
    __syncthreads();
    for (int t0 = 0; t0 < p.T; t0 += b) {
        if (p.W_states) {
            // the state at the start of this mini-batch: W1 [D][M], c1 [M], W2 [M][D], c2 [D]
            float* st = p.W_states + ((size_t)unit * (p.T / b) + t0 / b) * (2 * (size_t)D * M + M + D);
            for (int e = tid; e < D * M; e += kSimtThreads) {
                st[e] = W1[e];
                st[(size_t)D * M + M + e] = W2[e];
            }
            for (int e = tid; e < M; e += kSimtThreads) st[(size_t)D * M + e] = c1[e];
            for (int e = tid; e < D; e += kSimtThreads) st[2 * (size_t)D * M + M + e] = c2[e];
        }
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const size_t g = (size_t)t0 * D + e;
            Kt[e] = IoTraits<IO>::load(K, g);
            Qt[e] = IoTraits<IO>::load(Q, g);
            Et[e] = IoTraits<IO>::load(V, g);
        }
        for (int t = tid; t < b; t += kSimtThreads)
            et[t] = p.eta ? p.eta[(size_t)unit * p.T + t0 + t] : p.eta_const;
        __syncthreads();
        // A = K W1 + c1, Hk = GELU(A); S1 = tril(Q K^T + 1) * eta_s
        for (int e = tid; e < b * M; e += kSimtThreads) {
            const int t = e / M, q = e % M;
            float acc = c1[q];
            for (int i = 0; i < D; ++i) acc += Kt[t * D + i] * W1[i * M + q];
            At[e] = acc;
            Hk[e] = gelu_f(acc);
        }
        for (int e = tid; e < b * b; e += kSimtThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t) {
                for (int i = 0; i < D; ++i) acc += Qt[t * D + i] * Kt[s * D + i];
                acc = (acc + 1.f) * et[s];
            }
            S[e] = acc;
        }
        __syncthreads();
        // E = Hk W2 + c2 - V   (LN: Delta2 = LN+residual backward at Y = Hk W2 + c2)
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int t = e / D, j = e % D;
            float acc = c2[j];
            for (int q = 0; q < M; ++q) acc += Hk[t * M + q] * W2[q * D + j];
            if (LN)
                Yt[e] = acc;
            else
                Et[e] = acc - Et[e];
        }
        __syncthreads();
        if (LN) {
            for (int t = warp; t < b; t += nwarps) {
                float mu, r;
                warp_ln_stats(Yt + t * D, D, p.eps, mu, r);
                float s1 = 0.f, s2 = 0.f;
                for (int j = tid % 32; j < D; j += 32) {
                    const float xh = (Yt[t * D + j] - mu) * r;
                    const float g = gam[j] * (Kt[t * D + j] + gam[j] * xh + bet[j] - Et[t * D + j]);
                    s1 += g;
                    s2 += g * xh;
                }
                for (int o = 16; o > 0; o >>= 1) {
                    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
                }
                s1 /= D;
                s2 /= D;
                for (int j = tid % 32; j < D; j += 32) {
                    const float xh = (Yt[t * D + j] - mu) * r;
                    const float g = gam[j] * (Kt[t * D + j] + gam[j] * xh + bet[j] - Et[t * D + j]);
                    Et[t * D + j] = r * (g - s1 - xh * s2);   // Delta2 in place of V
                }
            }
            __syncthreads();
        }
        // D1 = (E W2^T) * GELU'(A)   (in place of A)
        for (int e = tid; e < b * M; e += kSimtThreads) {
            const int t = e / M, q = e % M;
            float acc = 0.f;
            for (int j = 0; j < D; ++j) acc += Et[t * D + j] * W2[q * D + j];
            At[e] = acc * gelu_grad_f(At[e]);
        }
        __syncthreads();
        // Aq = Q W1 + c1 - S1 D1 ; Hq = GELU(Aq)
        for (int e = tid; e < b * M; e += kSimtThreads) {
            const int t = e / M, q = e % M;
            float acc = c1[q];
            for (int i = 0; i < D; ++i) acc += Qt[t * D + i] * W1[i * M + q];
            for (int s = 0; s <= t; ++s) acc -= S[t * b + s] * At[s * M + q];
            Hq[e] = gelu_f(acc);
        }
        __syncthreads();
        // S2 = tril(Hq Hk^T + 1) * eta_s
        for (int e = tid; e < b * b; e += kSimtThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t) {
                for (int q = 0; q < M; ++q) acc += Hq[t * M + q] * Hk[s * M + q];
                acc = (acc + 1.f) * et[s];
            }
            S[e] = acc;
        }
        __syncthreads();
        // Z = Hq W2 + c2 - S2 E   (LN: Z = Q + gamma LN(that) + beta)
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int t = e / D, j = e % D;
            float acc = c2[j];
            for (int q = 0; q < M; ++q) acc += Hq[t * M + q] * W2[q * D + j];
            for (int s = 0; s <= t; ++s) acc -= S[t * b + s] * Et[s * D + j];
            if (LN)
                Yt[e] = acc;
            else
                IoTraits<IO>::store(Z, (size_t)t0 * D + e, acc);
        }
        __syncthreads();
        if (LN) {
            for (int t = warp; t < b; t += nwarps) {
                float mu, r;
                warp_ln_stats(Yt + t * D, D, p.eps, mu, r);
                for (int j = tid % 32; j < D; j += 32)
                    IoTraits<IO>::store(Z, (size_t)(t0 + t) * D + j,
                                        Qt[t * D + j] + gam[j] * (Yt[t * D + j] - mu) * r + bet[j]);
            }
        }
        // state update
        for (int e = tid; e < D * M; e += kSimtThreads) {
            const int i = e / M, q = e % M;
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += Kt[t * D + i] * et[t] * At[t * M + q];
            W1[e] -= acc;
        }
        for (int e = tid; e < M * D; e += kSimtThreads) {
            const int q = e / D, j = e % D;
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += Hk[t * M + q] * et[t] * Et[t * D + j];
            W2[e] -= acc;
        }
        for (int q = tid; q < M; q += kSimtThreads) {
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += et[t] * At[t * M + q];
            c1[q] -= acc;
        }
        for (int j = tid; j < D; j += kSimtThreads) {
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += et[t] * Et[t * D + j];
            c2[j] -= acc;
        }
        __syncthreads();
    }
    for (int e = tid; e < D * M; e += kSimtThreads) {
        p.W1_out[(size_t)unit * D * M + e] = W1[e];
        p.W2_out[(size_t)unit * M * D + e] = W2[e];
    }
    if (p.c1_out)
        for (int e = tid; e < M; e += kSimtThreads) p.c1_out[(size_t)unit * M + e] = c1[e];
    if (p.c2_out)
        for (int e = tid; e < D; e += kSimtThreads) p.c2_out[(size_t)unit * D + e] = c2[e];
}

inline size_t simt_mlp_smem(int D, int b, bool ln) {
    const size_t M = 4 * (size_t)D;
    return sizeof(float) * (2 * D * M + M + D + (ln ? 4 : 3) * (size_t)b * D + 3 * (size_t)b * M + (size_t)b * b + b);
}

}  // namespace ttt
