// Decode step of TTT-Linear: one token per (sequence, head) unit, the b = 1
// primal update (paper digest "论文速览 | TTT", section 6.11: generation is
// token by token and uses the primal form; section 3.1: update, then output):
//
//     u = k W,  e = u - v,  W <- W - eta k^T e,  z = q W_new = q W - eta (q.k) e
//
// The step is bound by one read and one write of W (d*d fp32 per unit).  One
// CTA per unit; thread (rg, cg) owns a 4x4 block of W (rows 4rg.., columns
// 4cg..) in registers between the read and the write, so W crosses HBM
// exactly twice.
#pragma once
#include "common.cuh"

namespace ttt {

struct DecodeParams {
    float* W;
    const void* q;
    const void* k;
    const void* v;
    const float* eta;
    float eta_const;
    void* z;
};

template <int D, typename IO>
__global__ void __launch_bounds__((D / 4) * (D / 4)) decode_kernel(DecodeParams p) {
    constexpr int G = D / 4;         // 4-wide groups per row / column
    constexpr int NT = G * G;        // threads
    __shared__ float sq[D], sk[D], sv[D];
    __shared__ float su[G][D], sp[G][D];
    const int tid = threadIdx.x;
    const int unit = blockIdx.x;
    const int cg = tid % G, rg = tid / G;
    const IO* q = static_cast<const IO*>(p.q) + (size_t)unit * D;
    const IO* k = static_cast<const IO*>(p.k) + (size_t)unit * D;
    const IO* v = static_cast<const IO*>(p.v) + (size_t)unit * D;
    for (int i = tid; i < D; i += NT) {
        sq[i] = IoTraits<IO>::load(q, i);
        sk[i] = IoTraits<IO>::load(k, i);
        sv[i] = IoTraits<IO>::load(v, i);
    }
    float4* W = reinterpret_cast<float4*>(p.W + (size_t)unit * D * D);
    float4 w[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) w[r] = W[(size_t)(4 * rg + r) * G + cg];
    __syncthreads();
    // partial u = k W and p = q W over this thread's 4 rows
    float pu[4] = {0.f, 0.f, 0.f, 0.f}, pp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float kr = sk[4 * rg + r], qr = sq[4 * rg + r];
        pu[0] += kr * w[r].x; pu[1] += kr * w[r].y; pu[2] += kr * w[r].z; pu[3] += kr * w[r].w;
        pp[0] += qr * w[r].x; pp[1] += qr * w[r].y; pp[2] += qr * w[r].z; pp[3] += qr * w[r].w;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        su[rg][4 * cg + c] = pu[c];
        sp[rg][4 * cg + c] = pp[c];
    }
    __syncthreads();
    const float eta = p.eta ? p.eta[unit] : p.eta_const;
    float qk = 0.f;
    for (int i = 0; i < D; ++i) qk += sq[i] * sk[i];
    // every thread needs e for its 4 columns
    float e[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int j = 4 * cg + c;
        float uj = 0.f, pj = 0.f;
        for (int g = 0; g < G; ++g) {
            uj += su[g][j];
            pj += sp[g][j];
        }
        e[c] = uj - sv[j];
        if (rg == 0) IoTraits<IO>::store(static_cast<IO*>(p.z), (size_t)unit * D + j, pj - eta * qk * e[c]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float a = eta * sk[4 * rg + r];
        w[r].x -= a * e[0]; w[r].y -= a * e[1]; w[r].z -= a * e[2]; w[r].w -= a * e[3];
        W[(size_t)(4 * rg + r) * G + cg] = w[r];
    }
}

}  // namespace ttt
