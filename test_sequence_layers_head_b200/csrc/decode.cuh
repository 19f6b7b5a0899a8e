// Decode step of TTT-Linear: one token per (sequence, head) unit, the b = 1
// primal update (paper digest "论文速览 | TTT", section 6.11: generation is
// token by token and uses the primal form; section 3.1: update, then output):
//
//     u = k W,  e = u - v,  W <- W - eta k^T e,  z = q W_new = q W - eta (q.k) e
//
// LN+residual (section 4.4), f(x) = x + LN(x W + c), gamma and beta fixed:
//
//     y = k W + c,  xhat = (y - mean y) r,  r = 1 / sqrt(var y + eps)
//     g = gamma * (k + gamma xhat + beta - v)
//     delta = r (g - mean g - xhat mean(g xhat))
//     W <- W - eta k^T delta,  c <- c - eta delta
//     z = q + gamma LN(q W_new + c_new) + beta,
//         q W_new + c_new = q W + c - eta ((q.k) + 1) delta
//
// (means and variances over the d features; the variance is the biased one).
//
// The step reads and writes W once (d*d fp32 per unit).  One CTA per unit,
// 4 D threads.  Thread t owns the float4 column group t % (D/4) of rows
// t / (D/4) + 16 r, so each warp-wide access covers whole rows (512
// contiguous bytes at D = 64) and touches the fewest cache lines; the sums
// over rows go through shuffles inside the warp, then one shared-memory
// exchange across the D/8 warps.
//
// Plain stream order between steps: with 512 units, programmatic dependent
// launch measured slower (the next step's early CTAs take residency from the
// current one) at every unit count tried (64, 148, 512).
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
    // LN+residual only
    float* c;             // [units, D], updated in place
    const float* gamma;   // [H, D]
    const float* beta;    // [H, D]
    float eps;
    int H;
};

// sum over the D features of a per-thread partial over its 4 columns: the
// column groups of a row sit on lanes cg = lane % (D/4)
template <int CG>
__device__ __forceinline__ float feature_sum(float x) {
#pragma unroll
    for (int o = 1; o < CG; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <int D, typename IO, bool LN>
__global__ void __launch_bounds__(D * 4) decode_kernel(DecodeParams p) {
    constexpr int NT = 4 * D, NW = NT / 32;   // threads, warps
    constexpr int CG = D / 4;                 // float4 column groups per row
    constexpr int R = D / 16;                 // rows per thread
    __shared__ float4 red[NW][2][CG];         // per-warp partial k W and q W
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int unit = blockIdx.x;
    const int cg = t % CG, row0 = t / CG;     // rows row0 + 16 r
    const IO* q = static_cast<const IO*>(p.q) + (size_t)unit * D;
    const IO* k = static_cast<const IO*>(p.k) + (size_t)unit * D;
    const IO* v = static_cast<const IO*>(p.v) + (size_t)unit * D;
    float4* W = reinterpret_cast<float4*>(p.W + (size_t)unit * D * D);
    float4 wr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) wr[r] = W[(size_t)(row0 + 16 * r) * CG + cg];
    float kr[R], qr[R], vc[4];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        kr[r] = IoTraits<IO>::load(k, row0 + 16 * r);
        qr[r] = IoTraits<IO>::load(q, row0 + 16 * r);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) vc[c] = IoTraits<IO>::load(v, 4 * cg + c);
    const float eta = p.eta ? p.eta[unit] : p.eta_const;
    // q . k, complete in every warp
    float qk = 0.f;
    for (int i = lane; i < D; i += 32) qk += IoTraits<IO>::load(q, i) * IoTraits<IO>::load(k, i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, o);

    float u[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < R; ++r) {
        u[0] += kr[r] * wr[r].x; u[1] += kr[r] * wr[r].y; u[2] += kr[r] * wr[r].z; u[3] += kr[r] * wr[r].w;
        pq[0] += qr[r] * wr[r].x; pq[1] += qr[r] * wr[r].y; pq[2] += qr[r] * wr[r].z; pq[3] += qr[r] * wr[r].w;
    }
    // rows of this warp: lanes cg, cg + CG, ... share the column group
#pragma unroll
    for (int o = CG; o < 32; o <<= 1)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            u[c] += __shfl_xor_sync(0xffffffffu, u[c], o);
            pq[c] += __shfl_xor_sync(0xffffffffu, pq[c], o);
        }
    if (lane < CG) {
        red[w][0][lane] = make_float4(u[0], u[1], u[2], u[3]);
        red[w][1][lane] = make_float4(pq[0], pq[1], pq[2], pq[3]);
    }
    __syncthreads();
    float4 su = red[0][0][cg], sq = red[0][1][cg];
#pragma unroll
    for (int x = 1; x < NW; ++x) {
        const float4 a = red[x][0][cg], b = red[x][1][cg];
        su.x += a.x; su.y += a.y; su.z += a.z; su.w += a.w;
        sq.x += b.x; sq.y += b.y; sq.z += b.z; sq.w += b.w;
    }
    if constexpr (!LN) {
        const float e[4] = {su.x - vc[0], su.y - vc[1], su.z - vc[2], su.w - vc[3]};
        if (t < CG) {
            IO* z = static_cast<IO*>(p.z) + (size_t)unit * D;
            IoTraits<IO>::store(z, 4 * cg + 0, sq.x - eta * qk * e[0]);
            IoTraits<IO>::store(z, 4 * cg + 1, sq.y - eta * qk * e[1]);
            IoTraits<IO>::store(z, 4 * cg + 2, sq.z - eta * qk * e[2]);
            IoTraits<IO>::store(z, 4 * cg + 3, sq.w - eta * qk * e[3]);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float a = eta * kr[r];
            wr[r].x -= a * e[0]; wr[r].y -= a * e[1]; wr[r].z -= a * e[2]; wr[r].w -= a * e[3];
            W[(size_t)(row0 + 16 * r) * CG + cg] = wr[r];
        }
    } else {
        // this thread's four features j = 4 cg + c
        const int hd = unit % p.H;
        const float4 c4 = reinterpret_cast<const float4*>(p.c + (size_t)unit * D)[cg];
        const float4 g4 = reinterpret_cast<const float4*>(p.gamma + (size_t)hd * D)[cg];
        const float4 b4 = reinterpret_cast<const float4*>(p.beta + (size_t)hd * D)[cg];
        const float cj[4] = {c4.x, c4.y, c4.z, c4.w}, gj[4] = {g4.x, g4.y, g4.z, g4.w};
        const float bj[4] = {b4.x, b4.y, b4.z, b4.w};
        const float uk[4] = {su.x, su.y, su.z, su.w}, uq[4] = {sq.x, sq.y, sq.z, sq.w};
        float kj[4], qj[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            kj[c] = IoTraits<IO>::load(k, 4 * cg + c);
            qj[c] = IoTraits<IO>::load(q, 4 * cg + c);
        }
        // LN forward of y = k W + c
        float y[4], s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            y[c] = uk[c] + cj[c];
            s1 += y[c];
            s2 += y[c] * y[c];
        }
        s1 = feature_sum<CG>(s1);
        s2 = feature_sum<CG>(s2);
        const float mu = s1 * (1.f / D);
        const float rr = rsqrtf(fmaxf(s2 * (1.f / D) - mu * mu, 0.f) + p.eps);
        // backward to the pre-activation
        float xh[4], g[4], t1 = 0.f, t2 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            xh[c] = (y[c] - mu) * rr;
            g[c] = gj[c] * (kj[c] + gj[c] * xh[c] + bj[c] - vc[c]);
            t1 += g[c];
            t2 += g[c] * xh[c];
        }
        t1 = feature_sum<CG>(t1) * (1.f / D);
        t2 = feature_sum<CG>(t2) * (1.f / D);
        float dl[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) dl[c] = rr * (g[c] - t1 - xh[c] * t2);
        // output: LN of q W_new + c_new
        float pre[4], o1 = 0.f, o2 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            pre[c] = uq[c] + cj[c] - eta * (qk + 1.f) * dl[c];
            o1 += pre[c];
            o2 += pre[c] * pre[c];
        }
        o1 = feature_sum<CG>(o1);
        o2 = feature_sum<CG>(o2);
        const float muo = o1 * (1.f / D);
        const float ro = rsqrtf(fmaxf(o2 * (1.f / D) - muo * muo, 0.f) + p.eps);
        if (t < CG) {
            IO* z = static_cast<IO*>(p.z) + (size_t)unit * D;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                IoTraits<IO>::store(z, 4 * cg + c, qj[c] + gj[c] * (pre[c] - muo) * ro + bj[c]);
            reinterpret_cast<float4*>(p.c + (size_t)unit * D)[cg] =
                make_float4(cj[0] - eta * dl[0], cj[1] - eta * dl[1], cj[2] - eta * dl[2], cj[3] - eta * dl[3]);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float a = eta * kr[r];
            wr[r].x -= a * dl[0]; wr[r].y -= a * dl[1]; wr[r].z -= a * dl[2]; wr[r].w -= a * dl[3];
            W[(size_t)(row0 + 16 * r) * CG + cg] = wr[r];
        }
    }
}

}  // namespace ttt
