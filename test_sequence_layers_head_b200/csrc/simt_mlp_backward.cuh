// Outer-loop backward of the TTT-MLP prefill, f(x) = GELU(x W1 + c1) W2 + c2
// (no LN), on fp32 CUDA cores: one CTA per (sequence, head) unit, the
// mini-batches in reverse order, each from its batch-start state, which the
// forward wrote as a checkpoint (paper digest "论文速览 | TTT", section 6.12;
// the outer loop's gradients pass through the inner loop's updates, section
// 3.4).
//
// The forward of one mini-batch in matrix form (the dual form of section 3.7),
// from the batch-start state (W1, c1, W2, c2), with
// L1 = tril(Q K^T + 1) diag(eta) and L2 = tril(Hq Hk^T + 1) diag(eta):
//   A = K W1 + c1,  Hk = GELU(A),  E = Hk W2 + c2 - V,  M = E W2^T,  D1 = M * GELU'(A),
//   Aq = Q W1 + c1 - L1 D1,  Hq = GELU(Aq),  Z = Hq W2 + c2 - L2 E,
//   W1' = W1 - K^T diag(eta) D1,  c1' = c1 - D1^T eta,  W2' = W2 - Hk^T diag(eta) E,  c2' = c2 - E^T eta.
// The kernel runs its reverse: from dZ and the adjoint of (W1', c1', W2', c2')
// to dQ, dK, dV, deta and the adjoint of the batch-start state, which is the
// next (earlier) mini-batch's end-state adjoint.  The running adjoint lives in
// the gradient outputs dW1, dc1, dW2, dc2 (global memory, L2-resident), and
// each phase that reads the end-state adjoint runs before the phase that adds
// this mini-batch's terms to it.
//
// Every phase is a loop of the CTA's threads over the elements it produces,
// separated by __syncthreads(); the batch's token tiles and the b x m and
// b x b intermediates are in shared memory, the state is read from the
// checkpoint.
#pragma once
#include "common.cuh"
#include "simt.cuh"

namespace ttt {

struct SimtMlpBackwardParams {
    int H, T, b;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;          // [units, T] or null (eta_const)
    float eta_const;
    const float* W_states;     // [units, T / b, 2 D M + M + D]: W1 [D][M], c1 [M], W2 [M][D], c2 [D]
    const void* dZ;            // [units, T, D] or null
    const float* dW1_out;      // adjoints of the final state, [units, ...] or null
    const float* dc1_out;
    const float* dW2_out;
    const float* dc2_out;
    void* dQ;
    void* dK;
    void* dV;
    float* deta;               // [units, T] or null
    float* dW1;                // adjoints of the initial state, [units, ...]
    float* dc1;
    float* dW2;
    float* dc2;
    // LN+residual on the output layer (the LN template instance only): gamma, beta [H, D], eps; the
    // per-unit gradients dgamma, dbeta [units, D]
    const float* gamma;
    const float* beta;
    float eps;
    float* dgamma;
    float* dbeta;
};

inline size_t simt_mlp_backward_smem(int D, int b, bool ln = false) {
    const size_t M = 4 * (size_t)D;
    return sizeof(float) * ((ln ? 13 : 7) * (size_t)b * D + 9 * (size_t)b * M + 4 * (size_t)b * b +
                            (ln ? 5 : 2) * (size_t)b + (ln ? 4 * (size_t)D : 0));
}

// LN = true: f(x) = x + gamma LN(GELU(x W1 + c1) W2 + c2) + beta.  Delta2, the LN+residual backward at
// Y = Hk W2 + c2, takes E's place in every product (the dual form's updates use it); the outputs pass
// through the LN, so dP (the LN adjoint of gamma dZ at the recomputed P) takes dZ's place; and the
// complete adjoint of Delta2 goes through the LN+residual backward of each row to dY (for Hk, W2, c2)
// and de (for K, V, gamma, beta), as in the linear model with LN.
template <int D, typename IO, bool LN = false>
__global__ void __launch_bounds__(kSimtThreads) simt_mlp_backward_kernel(SimtMlpBackwardParams p) {
    constexpr int M = 4 * D;
    constexpr int NT = kSimtThreads;
    constexpr size_t SZ = 2 * (size_t)D * M + M + D;   // one checkpoint
    extern __shared__ __align__(16) float sm[];
    const int b = p.b;
    const int bD = b * D, bM = b * M, bb = b * b;
    float* Kt = sm;           // b x D
    float* Qt = Kt + bD;      // b x D
    float* Et = Qt + bD;      // b x D   V, then E
    float* dZt = Et + bD;     // b x D
    float* dE = dZt + bD;     // b x D   dc2' + Hk dW2', then dE
    float* dQt = dE + bD;     // b x D
    float* dKt = dQt + bD;    // b x D
    float* A = dKt + bD;      // b x M
    float* Hk = A + bM;       // b x M
    float* Mv = Hk + bM;      // b x M   M = E W2^T, then dA
    float* D1 = Mv + bM;      // b x M
    float* Aq = D1 + bM;      // b x M
    float* Hq = Aq + bM;      // b x M
    float* dAq = Hq + bM;     // b x M   dHq, then dAq
    float* dD1 = dAq + bM;    // b x M   dc1' + K dW1', then dD1, then dM
    float* dHk = dD1 + bM;    // b x M
    float* P1 = dHk + bM;     // b x b   tril(Q K^T + 1)
    float* P2 = P1 + bb;      // b x b   tril(Hq Hk^T + 1)
    float* dL2 = P2 + bb;     // b x b   tril(-dZ E^T)
    float* dL1 = dL2 + bb;    // b x b   tril(-dAq D1^T)
    float* et = dL1 + bb;     // b
    float* det = et + b;      // b
    // LN only: Xh (LN(Y), then the output's LN(P)), Ev (E = K + gamma Xh + beta - V), dZr (dZ as given),
    // dYt, deT (b x D); per row r, mean(G), mean(G Xh); gamma, beta, dgamma, dbeta (D)
    float* Xh = det + b;
    float* Ev = Xh + (LN ? bD : 0);
    float* Xo = Ev + (LN ? bD : 0);
    float* dZr = Xo + (LN ? bD : 0);
    float* dYt = dZr + (LN ? bD : 0);
    float* deT = dYt + (LN ? bD : 0);
    float* rr = deT + (LN ? bD : 0);
    float* mgv = rr + (LN ? b : 0);
    float* mgx = mgv + (LN ? b : 0);
    float* gam = mgx + (LN ? b : 0);
    float* bet = gam + (LN ? D : 0);
    float* dgam = bet + (LN ? D : 0);
    float* dbet = dgam + (LN ? D : 0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = NT / 32;
    const int unit = blockIdx.x;
    const int T = p.T, nb = T / b;
    const size_t tok = (size_t)unit * T * D;
    const IO* Q = static_cast<const IO*>(p.Q) + tok;
    const IO* K = static_cast<const IO*>(p.K) + tok;
    const IO* V = static_cast<const IO*>(p.V) + tok;
    const IO* dZ = p.dZ ? static_cast<const IO*>(p.dZ) + tok : nullptr;
    IO* dQ = static_cast<IO*>(p.dQ) + tok;
    IO* dK = static_cast<IO*>(p.dK) + tok;
    IO* dV = static_cast<IO*>(p.dV) + tok;
    float* gW1 = p.dW1 + (size_t)unit * D * M;
    float* gc1 = p.dc1 + (size_t)unit * M;
    float* gW2 = p.dW2 + (size_t)unit * M * D;
    float* gc2 = p.dc2 + (size_t)unit * D;

    // the adjoint of the final state: the upstream gradients, or zero
    for (int e = tid; e < D * M; e += NT) {
        gW1[e] = p.dW1_out ? p.dW1_out[(size_t)unit * D * M + e] : 0.f;
        gW2[e] = p.dW2_out ? p.dW2_out[(size_t)unit * M * D + e] : 0.f;
    }
    for (int e = tid; e < M; e += NT) gc1[e] = p.dc1_out ? p.dc1_out[(size_t)unit * M + e] : 0.f;
    for (int e = tid; e < D; e += NT) gc2[e] = p.dc2_out ? p.dc2_out[(size_t)unit * D + e] : 0.f;
    if (LN)
        for (int j = tid; j < D; j += NT) {
            gam[j] = p.gamma[(size_t)(unit % p.H) * D + j];
            bet[j] = p.beta[(size_t)(unit % p.H) * D + j];
            dgam[j] = 0.f;
            dbet[j] = 0.f;
        }
    __syncthreads();

    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * b;
        const float* W1s = p.W_states + ((size_t)unit * nb + i) * SZ;
        const float* c1s = W1s + (size_t)D * M;
        const float* W2s = c1s + M;
        const float* c2s = W2s + (size_t)M * D;
        // ---- the mini-batch's tokens
        for (int e = tid; e < bD; e += NT) {
            const size_t g = (size_t)t0 * D + e;
            Kt[e] = IoTraits<IO>::load(K, g);
            Qt[e] = IoTraits<IO>::load(Q, g);
            Et[e] = IoTraits<IO>::load(V, g);
            dZt[e] = dZ ? IoTraits<IO>::load(dZ, g) : 0.f;
        }
        for (int t = tid; t < b; t += NT) {
            et[t] = p.eta ? p.eta[(size_t)unit * T + t0 + t] : p.eta_const;
            det[t] = 0.f;
        }
        __syncthreads();
        // ---- forward: A, Hk; P1
        for (int e = tid; e < bM; e += NT) {
            const int s = e / M, q = e % M;
            float acc = c1s[q];
            for (int a = 0; a < D; ++a) acc += Kt[s * D + a] * W1s[a * M + q];
            A[e] = acc;
            Hk[e] = gelu_f(acc);
        }
        for (int e = tid; e < bb; e += NT) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t) {
                for (int a = 0; a < D; ++a) acc += Qt[t * D + a] * Kt[s * D + a];
                acc += 1.f;
            }
            P1[e] = acc;
        }
        __syncthreads();
        // E = Hk W2 + c2 - V (in place of V); LN: Y = Hk W2 + c2 (into Xh), then per row the LN+residual
        // backward Delta2 (in place of V), with E, Xh, r, mean(G), mean(G Xh) kept
        for (int e = tid; e < bD; e += NT) {
            const int s = e / D, j = e % D;
            float acc = c2s[j];
            for (int q = 0; q < M; ++q) acc += Hk[s * M + q] * W2s[q * D + j];
            if (LN)
                Xh[e] = acc;
            else
                Et[e] = acc - Et[e];
        }
        __syncthreads();
        if (LN) {
            for (int s = warp; s < b; s += nwarps) {
                float mu, r;
                warp_ln_stats(Xh + s * D, D, p.eps, mu, r);
                float mg = 0.f, mgx_ = 0.f;
                for (int j = lane; j < D; j += 32) {
                    const float x = (Xh[s * D + j] - mu) * r;
                    Xh[s * D + j] = x;
                    const float ev = Kt[s * D + j] + gam[j] * x + bet[j] - Et[s * D + j];
                    Ev[s * D + j] = ev;
                    mg += gam[j] * ev;
                    mgx_ += gam[j] * ev * x;
                }
                for (int o = 16; o > 0; o >>= 1) {
                    mg += __shfl_xor_sync(0xffffffffu, mg, o);
                    mgx_ += __shfl_xor_sync(0xffffffffu, mgx_, o);
                }
                mg /= D;
                mgx_ /= D;
                for (int j = lane; j < D; j += 32)
                    Et[s * D + j] = r * (gam[j] * Ev[s * D + j] - mg - Xh[s * D + j] * mgx_);   // Delta2
                if (lane == 0) {
                    rr[s] = r;
                    mgv[s] = mg;
                    mgx[s] = mgx_;
                }
            }
            __syncthreads();
        }
        // M = E W2^T, D1 = M GELU'(A)
        for (int e = tid; e < bM; e += NT) {
            const int s = e / M, q = e % M;
            float acc = 0.f;
            for (int j = 0; j < D; ++j) acc += Et[s * D + j] * W2s[q * D + j];
            Mv[e] = acc;
            D1[e] = acc * gelu_grad_f(A[e]);
        }
        __syncthreads();
        // Aq = Q W1 + c1 - L1 D1, Hq = GELU(Aq)
        for (int e = tid; e < bM; e += NT) {
            const int t = e / M, q = e % M;
            float acc = c1s[q];
            for (int a = 0; a < D; ++a) acc += Qt[t * D + a] * W1s[a * M + q];
            for (int s = 0; s <= t; ++s) acc -= P1[t * b + s] * et[s] * D1[s * M + q];
            Aq[e] = acc;
            Hq[e] = gelu_f(acc);
        }
        __syncthreads();
        if (LN) {
            // the outputs' pre-LN P = Hq W2 + c2 - L2 Delta2 (L2 = tril(Hq Hk^T + 1) diag(eta)), its LN, and
            // dP = the LN adjoint of gamma dZ, which takes dZ's place below (dZ kept in dZr)
            for (int e = tid; e < bb; e += NT) {
                const int t = e / b, s = e % b;
                float acc = 0.f;
                if (s <= t) {
                    for (int q = 0; q < M; ++q) acc += Hq[t * M + q] * Hk[s * M + q];
                    acc += 1.f;
                }
                P2[e] = acc;
            }
            __syncthreads();
            for (int e = tid; e < bD; e += NT) {
                const int t = e / D, j = e % D;
                float acc = c2s[j];
                for (int q = 0; q < M; ++q) acc += Hq[t * M + q] * W2s[q * D + j];
                for (int s = 0; s <= t; ++s) acc -= P2[t * b + s] * et[s] * Et[s * D + j];
                Xo[e] = acc;
                dZr[e] = dZt[e];
            }
            __syncthreads();
            for (int t = warp; t < b; t += nwarps) {
                float mu, r;
                warp_ln_stats(Xo + t * D, D, p.eps, mu, r);
                float m1 = 0.f, m2 = 0.f;
                for (int j = lane; j < D; j += 32) {
                    const float x = (Xo[t * D + j] - mu) * r;
                    Xo[t * D + j] = x;
                    const float g = gam[j] * dZr[t * D + j];
                    m1 += g;
                    m2 += g * x;
                }
                for (int o = 16; o > 0; o >>= 1) {
                    m1 += __shfl_xor_sync(0xffffffffu, m1, o);
                    m2 += __shfl_xor_sync(0xffffffffu, m2, o);
                }
                m1 /= D;
                m2 /= D;
                for (int j = lane; j < D; j += 32) {
                    const float x = Xo[t * D + j];
                    dZt[t * D + j] = r * (gam[j] * dZr[t * D + j] - m1 - x * m2);   // dP
                }
            }
            __syncthreads();
        }
        // ---- backward.  First every product with the end-state adjoint (read before
        // this mini-batch adds to it), P2, dHq = dZ W2^T and dL2 = tril(-dZ E^T)
        // (LN: dP in dZ's place and Delta2 in E's)
        for (int e = tid; e < bb; e += NT) {
            const int t = e / b, s = e % b;
            float acc = 0.f, acc2 = 0.f;
            if (s <= t) {
                for (int q = 0; q < M; ++q) acc += Hq[t * M + q] * Hk[s * M + q];
                acc += 1.f;
                for (int j = 0; j < D; ++j) acc2 -= dZt[t * D + j] * Et[s * D + j];
            }
            P2[e] = acc;
            dL2[e] = acc2;
        }
        for (int e = tid; e < bD; e += NT) {
            const int s = e / D, x = e % D;
            float g2 = gc2[x], dk = 0.f;
            for (int q = 0; q < M; ++q) {
                g2 += Hk[s * M + q] * gW2[q * D + x];     // (dc2' + Hk dW2')[s][x]
                dk += D1[s * M + q] * gW1[x * M + q];     // (D1 dW1'^T)[s][x]
            }
            dE[e] = g2;
            dKt[e] = -et[s] * dk;
        }
        for (int e = tid; e < bM; e += NT) {
            const int s = e / M, q = e % M;
            float g1 = gc1[q], eh = 0.f, dh = 0.f;
            for (int a = 0; a < D; ++a) g1 += Kt[s * D + a] * gW1[a * M + q];   // dc1' + K dW1'
            for (int j = 0; j < D; ++j) {
                eh += Et[s * D + j] * gW2[q * D + j];   // (E dW2'^T)[s][q]
                dh += dZt[s * D + j] * W2s[q * D + j];  // (dZ W2^T)[s][q]
            }
            dD1[e] = g1;
            dHk[e] = -et[s] * eh;
            dAq[e] = dh;
        }
        __syncthreads();
        // deta from the state updates and the layer-2 outputs
        for (int s = warp; s < b; s += nwarps) {
            float acc = 0.f;
            for (int j = lane; j < D; j += 32) acc -= dE[s * D + j] * Et[s * D + j];
            for (int q = lane; q < M; q += 32) acc -= dD1[s * M + q] * D1[s * M + q];
            for (int t = s + lane; t < b; t += 32) acc += dL2[t * b + s] * P2[t * b + s];
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) det[s] += acc;
        }
        __syncthreads();
        // dE = -eta (dc2' + Hk dW2') - L2^T dZ;  dD1 = -eta (dc1' + K dW1')
        for (int e = tid; e < bD; e += NT) {
            const int s = e / D, j = e % D;
            float acc = 0.f;
            for (int t = s; t < b; ++t) acc += P2[t * b + s] * dZt[t * D + j];
            dE[e] = -et[s] * (dE[e] + acc);
        }
        for (int e = tid; e < bM; e += NT) dD1[e] *= -et[e / M];
        __syncthreads();
        // with dP2 = dL2 diag(eta):  dAq = (dHq + dP2 Hk) GELU'(Aq);  dHk += dP2^T Hq
        for (int e = tid; e < bM; e += NT) {
            const int r = e / M, q = e % M;
            float acc = dAq[e];
            for (int s = 0; s <= r; ++s) acc += dL2[r * b + s] * et[s] * Hk[s * M + q];
            dAq[e] = acc * gelu_grad_f(Aq[e]);
            float acc2 = 0.f;
            for (int t = r; t < b; ++t) acc2 += dL2[t * b + r] * Hq[t * M + q];
            dHk[e] += et[r] * acc2;
        }
        __syncthreads();
        // dQ = dAq W1^T;  dL1 = tril(-dAq D1^T);  dD1 -= L1^T dAq
        for (int e = tid; e < bD; e += NT) {
            const int t = e / D, a = e % D;
            float acc = 0.f;
            for (int q = 0; q < M; ++q) acc += dAq[t * M + q] * W1s[a * M + q];
            dQt[e] = acc;
        }
        for (int e = tid; e < bb; e += NT) {
            const int t = e / b, s = e % b;
            float acc = 0.f;
            if (s <= t)
                for (int q = 0; q < M; ++q) acc -= dAq[t * M + q] * D1[s * M + q];
            dL1[e] = acc;
        }
        for (int e = tid; e < bM; e += NT) {
            const int s = e / M, q = e % M;
            float acc = 0.f;
            for (int t = s; t < b; ++t) acc += P1[t * b + s] * dAq[t * M + q];
            dD1[e] -= et[s] * acc;
        }
        __syncthreads();
        // deta from the layer-1 outputs;  dM = dD1 GELU'(A) (in place of dD1) and the
        // first part of dA, dD1 M GELU''(A) (in place of M)
        for (int s = warp; s < b; s += nwarps) {
            float acc = 0.f;
            for (int t = s + lane; t < b; t += 32) acc += dL1[t * b + s] * P1[t * b + s];
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) det[s] += acc;
        }
        for (int e = tid; e < bM; e += NT) {
            const float x = A[e], dd = dD1[e];
            Mv[e] = dd * Mv[e] * gelu_grad2_f(x);
            dD1[e] = dd * gelu_grad_f(x);
        }
        __syncthreads();
        // with dP1 = dL1 diag(eta):  dQ += dP1 K;  dK += dP1^T Q;  dE += dM W2
        for (int e = tid; e < bD; e += NT) {
            const int r = e / D, x = e % D;
            float aq = 0.f, ak = 0.f, ae = 0.f;
            for (int s = 0; s <= r; ++s) aq += dL1[r * b + s] * et[s] * Kt[s * D + x];
            for (int t = r; t < b; ++t) ak += dL1[t * b + r] * Qt[t * D + x];
            for (int q = 0; q < M; ++q) ae += dD1[r * M + q] * W2s[q * D + x];
            dQt[e] += aq;
            dKt[e] += et[r] * ak;
            dE[e] += ae;
        }
        __syncthreads();
        if (LN) {
            // dE holds the adjoint of Delta2 = r U: per row, the LN+residual backward to de (E's adjoint,
            // for K, V, gamma, beta) and dY (Y = Hk W2 + c2); the dgamma terms of the row go to Ev
            for (int s = warp; s < b; s += nwarps) {
                const float r = rr[s];
                float dr = 0.f, mdu = 0.f, mdux = 0.f;
                for (int j = lane; j < D; j += 32) {
                    const float x = Xh[s * D + j];
                    const float u = gam[j] * Ev[s * D + j] - mgv[s] - x * mgx[s];
                    const float dd = dE[s * D + j];
                    dr += dd * u;
                    mdu += r * dd;
                    mdux += r * dd * x;
                }
                for (int o = 16; o > 0; o >>= 1) {
                    dr += __shfl_xor_sync(0xffffffffu, dr, o);
                    mdu += __shfl_xor_sync(0xffffffffu, mdu, o);
                    mdux += __shfl_xor_sync(0xffffffffu, mdux, o);
                }
                mdu /= D;
                mdux /= D;
                float m1 = 0.f, m2 = 0.f;
                for (int j = lane; j < D; j += 32) {
                    const float x = Xh[s * D + j];
                    const float du = r * dE[s * D + j];
                    const float dg = du - mdu - x * mdux;
                    const float de = gam[j] * dg;
                    const float dx = -du * mgx[s] - gam[j] * Ev[s * D + j] * mdux + gam[j] * de;
                    Ev[s * D + j] = Ev[s * D + j] * dg + x * de;   // the row's dgamma terms
                    deT[s * D + j] = de;
                    dYt[s * D + j] = dx;   // dXh for now
                    m1 += dx;
                    m2 += dx * x;
                }
                for (int o = 16; o > 0; o >>= 1) {
                    m1 += __shfl_xor_sync(0xffffffffu, m1, o);
                    m2 += __shfl_xor_sync(0xffffffffu, m2, o);
                }
                m1 /= D;
                m2 /= D;
                for (int j = lane; j < D; j += 32) {
                    const float x = Xh[s * D + j];
                    dYt[s * D + j] = r * (dYt[s * D + j] - m1 - x * m2) - dr * r * r * x / D;
                }
            }
            __syncthreads();
        }
        // the adjoint that reaches Hk, W2 and c2 (E's, or with LN Y's) and the one that reaches K and V
        const float* dYu = LN ? dYt : dE;
        const float* dEv = LN ? deT : dE;
        // dHk += dE W2^T;  dA = dD1 M GELU''(A) + dHk GELU'(A) (in Mv);  dV = -dE;  dQ out
        for (int e = tid; e < bM; e += NT) {
            const int s = e / M, q = e % M;
            float acc = dHk[e];
            for (int j = 0; j < D; ++j) acc += dYu[s * D + j] * W2s[q * D + j];
            Mv[e] += acc * gelu_grad_f(A[e]);
        }
        for (int e = tid; e < bD; e += NT) {
            IoTraits<IO>::store(dV, (size_t)t0 * D + e, -dEv[e]);
            IoTraits<IO>::store(dQ, (size_t)t0 * D + e, dQt[e] + (LN ? dZr[e] : 0.f));
        }
        __syncthreads();
        // dK += dA W1^T;  this mini-batch's terms of the start-state adjoint
        for (int e = tid; e < bD; e += NT) {
            const int s = e / D, a = e % D;
            float acc = dKt[e] + (LN ? deT[e] : 0.f);
            for (int q = 0; q < M; ++q) acc += Mv[s * M + q] * W1s[a * M + q];
            IoTraits<IO>::store(dK, (size_t)t0 * D + e, acc);
        }
        for (int e = tid; e < D * M; e += NT) {
            const int a = e / M, q = e % M;
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += Qt[t * D + a] * dAq[t * M + q] + Kt[t * D + a] * Mv[t * M + q];
            gW1[e] += acc;
        }
        for (int e = tid; e < M * D; e += NT) {
            const int q = e / D, j = e % D;
            float acc = 0.f;
            for (int t = 0; t < b; ++t)
                acc += Hq[t * M + q] * dZt[t * D + j] + dD1[t * M + q] * Et[t * D + j] + Hk[t * M + q] * dYu[t * D + j];
            gW2[e] += acc;
        }
        for (int q = tid; q < M; q += NT) {
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += dAq[t * M + q] + Mv[t * M + q];
            gc1[q] += acc;
        }
        for (int j = tid; j < D; j += NT) {
            float acc = 0.f;
            for (int t = 0; t < b; ++t) acc += dZt[t * D + j] + dYu[t * D + j];
            gc2[j] += acc;
            if (LN) {
                float g = 0.f, bb_ = 0.f;
                for (int t = 0; t < b; ++t) {
                    g += dZr[t * D + j] * Xo[t * D + j] + Ev[t * D + j];
                    bb_ += dZr[t * D + j] + deT[t * D + j];
                }
                dgam[j] += g;
                dbet[j] += bb_;
            }
        }
        if (p.deta)
            for (int t = tid; t < b; t += NT) p.deta[(size_t)unit * T + t0 + t] = det[t];
        __syncthreads();
    }
    if (LN)
        for (int j = tid; j < D; j += NT) {
            p.dgamma[(size_t)unit * D + j] = dgam[j];
            p.dbeta[(size_t)unit * D + j] = dbet[j];
        }
}

}  // namespace ttt
