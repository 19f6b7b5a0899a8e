// Decode step of TTT-Linear: one token per (sequence, head) unit, the b = 1
// primal update (paper digest "论文速览 | TTT", section 6.11: generation is
// token by token and uses the primal form; section 3.1: update, then output):
//
//     u = k W,  e = u - v,  W <- W - eta k^T e,  z = q W_new = q W - eta (q.k) e
//
// The step is bound by one read and one write of W (d*d fp32 per unit).  One
// CTA per unit, D/8 warps; warp w owns columns 8w..8w+7 over all D rows, lane
// l owns the float4 column group (l & 1) of rows (l >> 1) + 16 r, so the
// reduction over rows stays inside the warp (shuffles, no shared memory) and
// W crosses memory exactly twice.
//
// Launched with programmatic dependent launch: the launch of step n+1
// overlaps the tail of step n, and griddepcontrol.wait (before any global
// read) orders every read after the previous kernel's writes, so q, k, v may
// even alias the previous step's z.
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

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <int D, typename IO>
__global__ void __launch_bounds__(D * 4) decode_kernel(DecodeParams p) {
    constexpr int R = D / 16;        // rows per lane
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int unit = blockIdx.x;
    const int col = 8 * w + 4 * (lane & 1);   // first of this lane's 4 columns
    const int row0 = lane >> 1;               // rows row0 + 16 r
    grid_dependency_wait();   // the previous kernel in the stream is complete and visible
    const IO* q = static_cast<const IO*>(p.q) + (size_t)unit * D;
    const IO* k = static_cast<const IO*>(p.k) + (size_t)unit * D;
    const IO* v = static_cast<const IO*>(p.v) + (size_t)unit * D;
    float kr[R], qr[R], vc[4];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        kr[r] = IoTraits<IO>::load(k, row0 + 16 * r);
        qr[r] = IoTraits<IO>::load(q, row0 + 16 * r);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) vc[c] = IoTraits<IO>::load(v, col + c);
    const float eta = p.eta ? p.eta[unit] : p.eta_const;
    // q . k: every lane holds R (q, k) pairs of distinct rows (lane pairs repeat them)
    float qk = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) qk += qr[r] * kr[r];
    qk *= ((lane & 1) == 0) ? 1.f : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, o);

    float4* W = reinterpret_cast<float4*>(p.W + (size_t)unit * D * D);
    float4 wr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) wr[r] = W[(size_t)(row0 + 16 * r) * (D / 4) + (col >> 2)];
    grid_dependents_launch();

    float u[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < R; ++r) {
        u[0] += kr[r] * wr[r].x; u[1] += kr[r] * wr[r].y; u[2] += kr[r] * wr[r].z; u[3] += kr[r] * wr[r].w;
        pq[0] += qr[r] * wr[r].x; pq[1] += qr[r] * wr[r].y; pq[2] += qr[r] * wr[r].z; pq[3] += qr[r] * wr[r].w;
    }
    // sum over the 16 row groups (lane bits 1..4)
#pragma unroll
    for (int o = 2; o < 32; o <<= 1)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            u[c] += __shfl_xor_sync(0xffffffffu, u[c], o);
            pq[c] += __shfl_xor_sync(0xffffffffu, pq[c], o);
        }
    float e[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) e[c] = u[c] - vc[c];
    if (row0 == 0) {
        IO* z = static_cast<IO*>(p.z) + (size_t)unit * D;
#pragma unroll
        for (int c = 0; c < 4; ++c) IoTraits<IO>::store(z, col + c, pq[c] - eta * qk * e[c]);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float a = eta * kr[r];
        wr[r].x -= a * e[0]; wr[r].y -= a * e[1]; wr[r].z -= a * e[2]; wr[r].w -= a * e[3];
        W[(size_t)(row0 + 16 * r) * (D / 4) + (col >> 2)] = wr[r];
    }
}

}  // namespace ttt
