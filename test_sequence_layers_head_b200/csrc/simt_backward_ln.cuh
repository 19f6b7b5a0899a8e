// fp32 CUDA-core kernel of the LN+residual TTT-Linear backward,
// f(x) = x + gamma LN(x W + c) + beta (paper digest "论文速览 | TTT", section
// 4.4; outer-loop gradients through the inner loop, section 3.4; only the
// mini-batch boundary states are kept, section 6.12).
//
// Per mini-batch, with (W, c) the batch-start state and rows t, s of the
// mini-batch:
//   forward (recomputed)
//     Y = K W + c,  Xh = LN(Y) (r per row),  E = K + gamma Xh + beta - V,
//     G = gamma E,  U = G - mean(G) - Xh mean(G Xh),  Delta = diag(r) U,
//     A = diag(eta) Delta,  M = tril(Q K^T + 1),
//     P = Q W + c - M A,  Xo = LN(P) (ro per row),  Z = Q + gamma Xo + beta,
//     W' = W - K^T A,  c' = c - 1^T A
//   reverse, given dZ and (GW, Gc) = dL/d(W', c')
//     dgamma += sum_t dZ Xo,  dbeta += sum_t dZ,  dP = LN adjoint of gamma dZ
//     dM = -mask(dP A^T),   dQ = dZ + dP W^T + dM K,   dK = dM^T Q + ...
//     dA = -M^T dP - K GW - 1 Gc^T,   deta_s = dA_s . Delta_s,   dDelta = diag(eta) dA
//     dDelta -> (dY, de) through the LN+residual backward (row by row):
//        dr = dDelta . U,  dU = r dDelta,  dG = dU - mean(dU) - Xh mean(dU Xh),
//        dXh = -dU mean(G Xh) - G mean(dU Xh) + gamma de,   de = gamma dG,
//        dgamma += E dG + Xh de,  dbeta += de,  dK += de,  dV = -de,
//        dY = LN adjoint of dXh - dr r^2 Xh / d
//     dK += -A GW^T + dY W^T
//     GW <- GW + Q^T dP + K^T dY,   Gc <- Gc + sum_t dP + sum_s dY
// ("LN adjoint" of dX at X = LN(Y): r (dX - mean(dX) - X mean(dX X)).)
//
// One CTA per (sequence, head) unit, everything in shared memory.
#pragma once
#include "common.cuh"
#include "simt.cuh"

namespace ttt {

struct SimtLnBackwardParams {
    int H, T, b;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W_states;   // [units, T/b, D, D]
    const float* c_states;   // [units, T/b, D]
    const float* gamma;      // [H, D]
    const float* beta;
    float eps;
    const void* dZ;          // [units, T, D] or null
    const float* dW_out;     // [units, D, D] or null
    const float* dc_out;     // [units, D] or null
    void* dQ;
    void* dK;
    void* dV;
    float* deta;             // [units, T] or null
    float* dW0;              // [units, D, D]
    float* dc0;              // [units, D]
    float* dgamma;           // [units, D]
    float* dbeta;            // [units, D]
};

inline size_t simt_ln_backward_smem(int D, int b) {
    return sizeof(float) * (2 * (size_t)D * D + 14 * (size_t)b * D + 2 * (size_t)b * b + 4 * (size_t)b +
                            6 * (size_t)D);
}

template <int D, typename IO>
__global__ void __launch_bounds__(kSimtThreads) simt_ln_backward_kernel(SimtLnBackwardParams p) {
    extern __shared__ __align__(16) float sm[];
    const int b = p.b;
    float* W = sm;                 // D*D batch-start W
    float* GW = W + D * D;         // D*D dL/dW (state after the mini-batch, then before it)
    float* Kt = GW + D * D;        // b*D
    float* Qt = Kt + b * D;        // b*D
    float* Et = Qt + b * D;        // b*D  V, then E
    float* dZt = Et + b * D;       // b*D
    float* Xh = dZt + b * D;       // b*D  LN(Y)
    float* Gt = Xh + b * D;        // b*D  G = gamma E
    float* Ut = Gt + b * D;        // b*D  U
    float* Dl = Ut + b * D;        // b*D  Delta
    float* Xo = Dl + b * D;        // b*D  P, then LN(P)
    float* dP = Xo + b * D;        // b*D
    float* dA = dP + b * D;        // b*D  dA, then dDelta
    float* dY = dA + b * D;        // b*D
    float* dEt = dY + b * D;       // b*D  de
    float* gpart = dEt + b * D;    // b*D  dgamma contributions of the mini-batch's rows
    float* M = gpart + b * D;      // b*b  tril(Q K^T + 1)
    float* dM = M + b * b;         // b*b
    float* et = dM + b * b;        // b
    float* rr = et + b;            // b    r of Y rows
    float* ro = rr + b;            // b    r of P rows
    float* mgx = ro + b;           // b    mean(G Xh)
    float* c = mgx + b;            // D
    float* Gc = c + D;             // D
    float* gam = Gc + D;           // D
    float* bet = gam + D;          // D
    float* dgam = bet + D;         // D
    float* dbet = dgam + D;        // D
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32, nwarps = kSimtThreads / 32;
    const int unit = blockIdx.x, hd = unit % p.H;
    const int nb = p.T / b;
    const size_t tok = (size_t)unit * p.T * D;
    const IO* Q = static_cast<const IO*>(p.Q) + tok;
    const IO* K = static_cast<const IO*>(p.K) + tok;
    const IO* V = static_cast<const IO*>(p.V) + tok;
    const IO* dZ = p.dZ ? static_cast<const IO*>(p.dZ) + tok : nullptr;
    IO* dQg = static_cast<IO*>(p.dQ) + tok;
    IO* dKg = static_cast<IO*>(p.dK) + tok;
    IO* dVg = static_cast<IO*>(p.dV) + tok;
    for (int e = tid; e < D * D; e += kSimtThreads) GW[e] = p.dW_out ? p.dW_out[(size_t)unit * D * D + e] : 0.f;
    for (int j = tid; j < D; j += kSimtThreads) {
        Gc[j] = p.dc_out ? p.dc_out[(size_t)unit * D + j] : 0.f;
        gam[j] = p.gamma[(size_t)hd * D + j];
        bet[j] = p.beta[(size_t)hd * D + j];
        dgam[j] = 0.f;
        dbet[j] = 0.f;
    }
    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * b;
        const float* Ws = p.W_states + ((size_t)unit * nb + i) * D * D;
        const float* cs = p.c_states + ((size_t)unit * nb + i) * D;
        for (int e = tid; e < D * D; e += kSimtThreads) W[e] = Ws[e];
        for (int j = tid; j < D; j += kSimtThreads) c[j] = cs[j];
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const size_t g = (size_t)t0 * D + e;
            Kt[e] = IoTraits<IO>::load(K, g);
            Qt[e] = IoTraits<IO>::load(Q, g);
            Et[e] = IoTraits<IO>::load(V, g);
            dZt[e] = dZ ? IoTraits<IO>::load(dZ, g) : 0.f;
        }
        for (int t = tid; t < b; t += kSimtThreads) et[t] = p.eta ? p.eta[(size_t)unit * p.T + t0 + t] : p.eta_const;
        __syncthreads();
        // Y = K W + c (into Xh), P0 = Q W + c (into Xo), M = tril(Q K^T + 1)
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int t = e / D, j = e % D;
            float y = c[j], q = c[j];
#pragma unroll 8
            for (int a = 0; a < D; ++a) {
                y += Kt[t * D + a] * W[a * D + j];
                q += Qt[t * D + a] * W[a * D + j];
            }
            Xh[e] = y;
            Xo[e] = q;
        }
        for (int e = tid; e < b * b; e += kSimtThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t) {
#pragma unroll 8
                for (int a = 0; a < D; ++a) acc += Qt[t * D + a] * Kt[s * D + a];
                acc += 1.f;
            }
            M[e] = acc;
        }
        __syncthreads();
        // per row s: LN of Y, E (in place of V), G, U, Delta
        for (int s = warp; s < b; s += nwarps) {
            float mu, r;
            warp_ln_stats(Xh + s * D, D, p.eps, mu, r);
            float mg = 0.f, mgx_ = 0.f;
            for (int j = lane; j < D; j += 32) {
                const float x = (Xh[s * D + j] - mu) * r;
                Xh[s * D + j] = x;
                const float ev = Kt[s * D + j] + gam[j] * x + bet[j] - Et[s * D + j];
                Et[s * D + j] = ev;
                const float g = gam[j] * ev;
                Gt[s * D + j] = g;
                mg += g;
                mgx_ += g * x;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mg += __shfl_xor_sync(0xffffffffu, mg, o);
                mgx_ += __shfl_xor_sync(0xffffffffu, mgx_, o);
            }
            mg /= D;
            mgx_ /= D;
            for (int j = lane; j < D; j += 32) {
                const float u = Gt[s * D + j] - mg - Xh[s * D + j] * mgx_;
                Ut[s * D + j] = u;
                Dl[s * D + j] = r * u;
            }
            if (lane == 0) {
                rr[s] = r;
                mgx[s] = mgx_;
            }
        }
        __syncthreads();
        // P = P0 - M A   (A = diag(eta) Delta)
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int t = e / D, j = e % D;
            float acc = Xo[e];
            for (int s = 0; s <= t; ++s) acc -= M[t * b + s] * et[s] * Dl[s * D + j];
            Xo[e] = acc;
        }
        __syncthreads();
        // per row t: Xo = LN(P), dP = LN adjoint of gamma dZ; dgamma/dbeta of the outputs
        for (int t = warp; t < b; t += nwarps) {
            float mu, r;
            warp_ln_stats(Xo + t * D, D, p.eps, mu, r);
            float m1 = 0.f, m2 = 0.f;
            for (int j = lane; j < D; j += 32) {
                const float x = (Xo[t * D + j] - mu) * r;
                Xo[t * D + j] = x;
                const float dx = gam[j] * dZt[t * D + j];
                m1 += dx;
                m2 += dx * x;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                m1 += __shfl_xor_sync(0xffffffffu, m1, o);
                m2 += __shfl_xor_sync(0xffffffffu, m2, o);
            }
            m1 /= D;
            m2 /= D;
            for (int j = lane; j < D; j += 32) {
                const float x = Xo[t * D + j];
                dP[t * D + j] = r * (gam[j] * dZt[t * D + j] - m1 - x * m2);
            }
            if (lane == 0) ro[t] = r;
        }
        __syncthreads();
        // dM = -mask(dP A^T) ; dA = -M^T dP - K GW - Gc
        for (int e = tid; e < b * b; e += kSimtThreads) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t) {
#pragma unroll 8
                for (int j = 0; j < D; ++j) acc += dP[t * D + j] * Dl[s * D + j];
                acc *= -et[s];
            }
            dM[e] = acc;
        }
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int s = e / D, j = e % D;
            float acc = Gc[j];
            for (int t = s; t < b; ++t) acc += M[t * b + s] * dP[t * D + j];
#pragma unroll 8
            for (int a = 0; a < D; ++a) acc += Kt[s * D + a] * GW[a * D + j];
            dA[e] = -acc;
        }
        __syncthreads();
        // dQ = dZ + dP W^T + dM K
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int t = e / D, a = e % D;
            float acc = dZt[e];
#pragma unroll 8
            for (int j = 0; j < D; ++j) acc += dP[t * D + j] * W[a * D + j];
            for (int s = 0; s <= t; ++s) acc += dM[t * b + s] * Kt[s * D + a];
            IoTraits<IO>::store(dQg, (size_t)t0 * D + e, acc);
        }
        // per row s: deta, dDelta = eta dA, and the LN+residual backward to dY and de
        for (int s = warp; s < b; s += nwarps) {
            float de_ = 0.f, dr = 0.f;
            for (int j = lane; j < D; j += 32) {
                de_ += dA[s * D + j] * Dl[s * D + j];
                const float dd = et[s] * dA[s * D + j];
                dA[s * D + j] = dd;
                dr += dd * Ut[s * D + j];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                de_ += __shfl_xor_sync(0xffffffffu, de_, o);
                dr += __shfl_xor_sync(0xffffffffu, dr, o);
            }
            if (lane == 0 && p.deta) p.deta[(size_t)unit * p.T + t0 + s] = de_;
            const float r = rr[s];
            float mdu = 0.f, mdux = 0.f;
            for (int j = lane; j < D; j += 32) {
                const float du = r * dA[s * D + j];
                mdu += du;
                mdux += du * Xh[s * D + j];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                mdu += __shfl_xor_sync(0xffffffffu, mdu, o);
                mdux += __shfl_xor_sync(0xffffffffu, mdux, o);
            }
            mdu /= D;
            mdux /= D;
            float m1 = 0.f, m2 = 0.f;
            for (int j = lane; j < D; j += 32) {
                const float x = Xh[s * D + j];
                const float du = r * dA[s * D + j];
                const float dg = du - mdu - x * mdux;
                const float de = gam[j] * dg;
                const float dx = -du * mgx[s] - Gt[s * D + j] * mdux + gam[j] * de;
                dEt[s * D + j] = de;
                gpart[s * D + j] = Et[s * D + j] * dg + x * de;
                IoTraits<IO>::store(dVg, (size_t)(t0 + s) * D + j, -de);
                dY[s * D + j] = dx;   // dXh for now
                m1 += dx;
                m2 += dx * x;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                m1 += __shfl_xor_sync(0xffffffffu, m1, o);
                m2 += __shfl_xor_sync(0xffffffffu, m2, o);
            }
            m1 /= D;
            m2 /= D;
            for (int j = lane; j < D; j += 32) {
                const float x = Xh[s * D + j];
                dY[s * D + j] = r * (dY[s * D + j] - m1 - x * m2) - dr * r * r * x / D;
            }
        }
        __syncthreads();
        // dK = dM^T Q - A GW^T + de + dY W^T   (GW is still dL/dW')
        for (int e = tid; e < b * D; e += kSimtThreads) {
            const int s = e / D, a = e % D;
            float acc = dEt[e];
            for (int t = s; t < b; ++t) acc += dM[t * b + s] * Qt[t * D + a];
            float ag = 0.f, yw = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; ++j) {
                ag += Dl[s * D + j] * GW[a * D + j];
                yw += dY[s * D + j] * W[a * D + j];
            }
            IoTraits<IO>::store(dKg, (size_t)(t0 + s) * D + a, acc - et[s] * ag + yw);
        }
        // dgamma, dbeta of the mini-batch (one thread per feature)
        for (int j = tid; j < D; j += kSimtThreads) {
            float g = 0.f, bb = 0.f;
            for (int t = 0; t < b; ++t) {
                g += dZt[t * D + j] * Xo[t * D + j] + gpart[t * D + j];
                bb += dZt[t * D + j] + dEt[t * D + j];
            }
            dgam[j] += g;
            dbet[j] += bb;
        }
        __syncthreads();
        // GW += Q^T dP + K^T dY ;  Gc += sum dP + sum dY
        for (int e = tid; e < D * D; e += kSimtThreads) {
            const int a = e / D, j = e % D;
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += Qt[t * D + a] * dP[t * D + j] + Kt[t * D + a] * dY[t * D + j];
            GW[e] += acc;
        }
        for (int j = tid; j < D; j += kSimtThreads) {
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += dP[t * D + j] + dY[t * D + j];
            Gc[j] += acc;
        }
        __syncthreads();
    }
    for (int e = tid; e < D * D; e += kSimtThreads) p.dW0[(size_t)unit * D * D + e] = GW[e];
    for (int j = tid; j < D; j += kSimtThreads) {
        p.dc0[(size_t)unit * D + j] = Gc[j];
        p.dgamma[(size_t)unit * D + j] = dgam[j];
        p.dbeta[(size_t)unit * D + j] = dbet[j];
    }
}

}  // namespace ttt
