// Decode step of TTT-MLP, f(x) = GELU(x W1 + c1) W2 + c2 with hidden size
// m = 4 d: one token per (sequence, head) unit, the b = 1 primal update
// (paper digest "论文速览 | TTT", section 6.11: generation is token by token
// and uses the primal form; section 3.1: update, then output; section 4.4:
// the two-layer MLP with GELU):
//
//     a = k W1 + c1,  h = GELU(a),  e = h W2 + c2 - v
//     delta1 = (e W2^T) * GELU'(a)
//     W1 <- W1 - eta k^T delta1,  c1 <- c1 - eta delta1
//     W2 <- W2 - eta h^T e,       c2 <- c2 - eta e
//     z = GELU(q W1_new + c1_new) W2_new + c2_new,
//         q W1_new + c1_new = q W1 + c1 - eta ((q.k) + 1) delta1
//
// One CTA of m threads per unit; the state (2 d m fp32) is read and written
// once.  Thread t owns hidden column t of W1 (d registers; each warp-wide
// access is one coalesced row segment).  W2 ([m][d]) is tiled like the
// linear decode's W: thread t owns the float4 column group t % (d/4) of rows
// t / (d/4) + 16 r, r < d/4.  Sums over hidden rows (e, z) go through
// shuffles and one shared-memory exchange across warps; sums over the d
// columns (e W2^T) reduce the d/4 column-group lanes by recursive halving,
// which leaves lane cg with the complete sum of its row slot r = cg.
//
// GELU and GELU' use CUDA's erff / expf (the decode is bound by the state
// traffic, not by these).
#pragma once
#include "common.cuh"

namespace ttt {

struct MlpDecodeParams {
    float* W1;   // [units, D, 4D]
    float* c1;   // [units, 4D]
    float* W2;   // [units, 4D, D]
    float* c2;   // [units, D]
    const void* q;
    const void* k;
    const void* v;
    const float* eta;
    float eta_const;
    void* z;
};

template <int D, typename IO>
__global__ void __launch_bounds__(4 * D) mlp_decode_kernel(MlpDecodeParams p) {
    constexpr int M = 4 * D;        // hidden size = threads
    constexpr int NW = M / 32;      // warps
    constexpr int CG = D / 4;       // float4 column groups of a W2 row
    constexpr int R2 = M / 16;      // W2 rows per thread (= CG)
    static_assert(R2 == CG, "one row slot per column-group lane");
    __shared__ float s_k[D], s_q[D];
    __shared__ float s_h[M], s_hq[M], s_eps[M];
    __shared__ float4 s_red[2][NW][CG];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int unit = blockIdx.x;
    const int cg = t % CG, row0 = t / CG;   // W2 rows row0 + 16 r

    const IO* qg = static_cast<const IO*>(p.q) + (size_t)unit * D;
    const IO* kg = static_cast<const IO*>(p.k) + (size_t)unit * D;
    const IO* vg = static_cast<const IO*>(p.v) + (size_t)unit * D;
    float* W1 = p.W1 + (size_t)unit * D * M;
    float4* W2 = reinterpret_cast<float4*>(p.W2 + (size_t)unit * M * D);
    float w1[D];
#pragma unroll
    for (int i = 0; i < D; ++i) w1[i] = W1[(size_t)i * M + t];
    float4 w2[R2];
#pragma unroll
    for (int r = 0; r < R2; ++r) w2[r] = W2[(size_t)(row0 + 16 * r) * CG + cg];
    if (t < D) {
        s_k[t] = IoTraits<IO>::load(kg, t);
        s_q[t] = IoTraits<IO>::load(qg, t);
    }
    const float eta = p.eta ? p.eta[unit] : p.eta_const;
    float vc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) vc[c] = IoTraits<IO>::load(vg, 4 * cg + c);
    const float4 c2v = reinterpret_cast<const float4*>(p.c2 + (size_t)unit * D)[cg];
    const float c1t = p.c1[(size_t)unit * M + t];
    __syncthreads();

    // layer 1 on hidden column t
    float a = c1t, aq = 0.f, qk = 0.f;
#pragma unroll
    for (int i = 0; i < D; ++i) {
        const float ki = s_k[i], qi = s_q[i];
        a += ki * w1[i];
        aq += qi * w1[i];
        qk += qi * ki;
    }
    const float h = gelu_f(a), gp = gelu_grad_f(a);
    s_h[t] = h;
    __syncthreads();

    // e = h W2 + c2 - v for this thread's four columns
    float pe[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < R2; ++r) {
        const float hr = s_h[row0 + 16 * r];
        pe[0] += hr * w2[r].x; pe[1] += hr * w2[r].y; pe[2] += hr * w2[r].z; pe[3] += hr * w2[r].w;
    }
#pragma unroll
    for (int o = CG; o < 32; o <<= 1)
#pragma unroll
        for (int c = 0; c < 4; ++c) pe[c] += __shfl_xor_sync(0xffffffffu, pe[c], o);
    if (lane < CG) s_red[0][w][lane] = make_float4(pe[0], pe[1], pe[2], pe[3]);
    __syncthreads();
    float e[4] = {c2v.x - vc[0], c2v.y - vc[1], c2v.z - vc[2], c2v.w - vc[3]};
#pragma unroll
    for (int x = 0; x < NW; ++x) {
        const float4 s = s_red[0][x][cg];
        e[0] += s.x; e[1] += s.y; e[2] += s.z; e[3] += s.w;
    }

    // (e W2^T) of this thread's R2 rows: partial over its four columns, then
    // recursive halving over the CG column-group lanes
    {
        float l[R2];
#pragma unroll
        for (int r = 0; r < R2; ++r) l[r] = w2[r].x * e[0] + w2[r].y * e[1] + w2[r].z * e[2] + w2[r].w * e[3];
#pragma unroll
        for (int n = R2, m = CG / 2; m >= 1; n >>= 1, m >>= 1) {
            const bool up = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < n / 2; ++i) {
                const float keep = up ? l[n / 2 + i] : l[i], send = up ? l[i] : l[n / 2 + i];
                l[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        s_eps[row0 + 16 * cg] = l[0];   // lane cg holds row slot r = cg
    }
    __syncthreads();

    // layer 1 update and the output pre-activation of hidden unit t
    const float d1 = s_eps[t] * gp;
#pragma unroll
    for (int i = 0; i < D; ++i) W1[(size_t)i * M + t] = w1[i] - eta * s_k[i] * d1;
    const float c1n = c1t - eta * d1;
    p.c1[(size_t)unit * M + t] = c1n;
    s_hq[t] = gelu_f(aq + c1n - eta * qk * d1);
    // layer 2 update
#pragma unroll
    for (int r = 0; r < R2; ++r) {
        const float a2 = eta * s_h[row0 + 16 * r];
        w2[r].x -= a2 * e[0]; w2[r].y -= a2 * e[1]; w2[r].z -= a2 * e[2]; w2[r].w -= a2 * e[3];
        W2[(size_t)(row0 + 16 * r) * CG + cg] = w2[r];
    }
    __syncthreads();

    // z = GELU(q W1_new + c1_new) W2_new + c2_new
    float pz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < R2; ++r) {
        const float hr = s_hq[row0 + 16 * r];
        pz[0] += hr * w2[r].x; pz[1] += hr * w2[r].y; pz[2] += hr * w2[r].z; pz[3] += hr * w2[r].w;
    }
#pragma unroll
    for (int o = CG; o < 32; o <<= 1)
#pragma unroll
        for (int c = 0; c < 4; ++c) pz[c] += __shfl_xor_sync(0xffffffffu, pz[c], o);
    if (lane < CG) s_red[1][w][lane] = make_float4(pz[0], pz[1], pz[2], pz[3]);
    __syncthreads();
    if (t < CG) {
        const float c2n[4] = {c2v.x - eta * e[0], c2v.y - eta * e[1], c2v.z - eta * e[2], c2v.w - eta * e[3]};
        float zz[4] = {c2n[0], c2n[1], c2n[2], c2n[3]};
#pragma unroll
        for (int x = 0; x < NW; ++x) {
            const float4 s = s_red[1][x][cg];
            zz[0] += s.x; zz[1] += s.y; zz[2] += s.z; zz[3] += s.w;
        }
        IO* zg = static_cast<IO*>(p.z) + (size_t)unit * D;
#pragma unroll
        for (int c = 0; c < 4; ++c) IoTraits<IO>::store(zg, 4 * cg + c, zz[c]);
        reinterpret_cast<float4*>(p.c2 + (size_t)unit * D)[cg] = make_float4(c2n[0], c2n[1], c2n[2], c2n[3]);
    }
}

}  // namespace ttt
