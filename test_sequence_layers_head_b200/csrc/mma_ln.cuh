// Tensor-core (mma.sync, bf16 operands, fp32 accumulation) training kernels of
// TTT-Linear with LN+residual, f(x) = x + gamma LN(x W + c) + beta (paper
// digest "论文速览 | TTT", section 4.4), for d = 64, b = 16 with bf16 inputs
// and outputs: the forward that writes the batch-start states (W, c) and the
// outer-loop backward that reads them (sections 3.4 and 6.12).
//
// Per mini-batch, with (W, c) the batch-start state:
//   Y = K W + c,  Xh = LN(Y) (r per row),  E = K + gamma Xh + beta - V,
//   G = gamma E,  U = G - mean(G) - Xh mean(G Xh),  Delta = diag(r) U,
//   A = diag(eta) Delta,  M = tril(Q K^T + 1),
//   P = Q W + c - M A,  Xo = LN(P) (ro per row),  Z = Q + gamma Xo + beta,
//   W' = W - K^T A,  c' = c - 1^T A.
// The backward runs the reverse of these steps (the same steps as the fp32
// CUDA-core kernel, simt_backward_ln.cuh), from dZ and (GW, Gc) = dL/d(W', c'):
//   dP = LN adjoint of gamma dZ at Xo,   dM = -mask(dP A^T),
//   dA = -M^T dP - K GW - 1 Gc^T,   deta_s = dA_s . Delta_s,   dDelta = diag(eta) dA,
//   dDelta -> dY, de through the LN+residual backward of each row,
//   dQ = dZ + dP W^T + dM K,   dK = de + dM^T Q - A GW^T + dY W^T,   dV = -de,
//   GW <- GW + Q^T dP + K^T dY,   Gc <- Gc + 1^T dP + 1^T dY,
//   dgamma += sum (dZ Xo + E dG + Xh de),   dbeta += sum (dZ + de),
// with "LN adjoint" of dX at X = LN(Y): r (dX - mean(dX) - X mean(dX X)).
//
// Layout as in the plain kernels (mma_backward.cuh): one CTA of four warps per
// unit; warp w owns features 16 w .. 16 w + 15 of every 16 x 64 product and
// state rows 16 w .. 16 w + 15 of W (forward) or GW (backward), kept in fp32
// registers.  A lane holds rows r and r + 8 of four features of each 16 x 64
// product, so the LN's sums over the 64 features of a row are a quad shuffle
// and one exchange of the four warps' partials through shared memory.  c,
// gamma, beta and their adjoints are per-lane registers for the lane's
// features.
#pragma once
#include "mma_backward.cuh"
#include "simt_backward_ln.cuh"

namespace ttt {
namespace mbk {

struct FwdLnStatesParams {
    int H, T;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W0;
    long long W0_bstride;
    const float* c0;        // or null (zero)
    long long c0_bstride;
    const float* gamma;     // [H, 64]
    const float* beta;
    float eps;
    void* Z;                // or null (state only)
    float* W_out;
    float* c_out;           // or null
    float* W_states;        // [units, T/16, 64, 64]
    float* c_states;        // [units, T/16, 64]
};

// one exchange site: 4 warps x 16 rows x up to 4 quantities (fp32)
constexpr int kRedFloats = 4 * kB * 4;

// shared memory of the forward (bytes): W (bf16 64 x 64), tiles K, Q, A (bf16 16 x 64), eta, 3 exchange sites
constexpr int kLFOffW = 0, kLFOffK = 8192, kLFOffQ = kLFOffK + 2048, kLFOffA = kLFOffQ + 2048;
constexpr int kLFOffEta = kLFOffA + 2048, kLFOffRed = kLFOffEta + 64;
constexpr int kLFSmemBytes = kLFOffRed + 3 * kRedFloats * 4;

// shared memory of the backward (bytes): W, GW (bf16 64 x 64), tiles K, Q, dZ, A, dP, dY (bf16 16 x 64),
// eta, 6 exchange sites
constexpr int kLBOffW = 0, kLBOffG = 8192, kLBOffK = 16384, kLBOffQ = kLBOffK + 2048, kLBOffDZ = kLBOffQ + 2048;
constexpr int kLBOffA = kLBOffDZ + 2048, kLBOffDP = kLBOffA + 2048, kLBOffDY = kLBOffDP + 2048;
constexpr int kLBOffEta = kLBOffDY + 2048, kLBOffRed = kLBOffEta + 64;
constexpr int kLBSmemBytes = kLBOffRed + 6 * kRedFloats * 4;

// Sums over the 64 features of rows r and r + 8: v[k][h] holds the lane's partial of quantity k for row
// r + 8 h and is replaced by the row's sum.  `buf` is an exchange site that no other call of this
// mini-batch uses; the call contains a CTA barrier.
template <int NQ>
__device__ __forceinline__ void row_sums(float (&v)[NQ][2], float* buf, int w, int r, int c) {
#pragma unroll
    for (int k = 0; k < NQ; ++k)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            v[k][h] += __shfl_xor_sync(0xffffffffu, v[k][h], 1);
            v[k][h] += __shfl_xor_sync(0xffffffffu, v[k][h], 2);
        }
    if (c == 0)
#pragma unroll
        for (int k = 0; k < NQ; ++k)
#pragma unroll
            for (int h = 0; h < 2; ++h) buf[(w * kB + r + 8 * h) * NQ + k] = v[k][h];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < NQ; ++k)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float s = 0.f;
#pragma unroll
            for (int ww = 0; ww < 4; ++ww) s += buf[(ww * kB + r + 8 * h) * NQ + k];
            v[k][h] = s;
        }
}

// Column sums over the 16 rows of a mini-batch: v[nt][k] holds the lane's rows r and r + 8 already
// added; the result (the sum over all 16 rows) is in every lane of the column.
__device__ __forceinline__ void col_sums(float (&v)[2][2]) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            v[nt][k] += __shfl_xor_sync(0xffffffffu, v[nt][k], 4);
            v[nt][k] += __shfl_xor_sync(0xffffffffu, v[nt][k], 8);
            v[nt][k] += __shfl_xor_sync(0xffffffffu, v[nt][k], 16);
        }
}

// the bf16 pair (row, 2 c + 8 nt + f0 ..) of a swizzled 16 x 64 tile, as two floats
__device__ __forceinline__ float2 tile_pair(const uint8_t* smem, int off, int row, int f0, int nt, int c) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(smem + off + toff(row, (f0 >> 3) + nt) + 4 * c);
    return make_float2(__bfloat162float(v.x), __bfloat162float(v.y));
}

__global__ void __launch_bounds__(kThreads) mma_ln_forward_states_kernel(FwdLnStatesParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sW = smem_u32(smem + kLFOffW), sK = smem_u32(smem + kLFOffK), sQ = smem_u32(smem + kLFOffQ);
    const uint32_t sA = smem_u32(smem + kLFOffA);
    float* s_eta = reinterpret_cast<float*>(smem + kLFOffEta);
    float* red = reinterpret_cast<float*>(smem + kLFOffRed);
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, r = l >> 2, c = l & 3;
    const int unit = blockIdx.x;
    const int n = unit / p.H, hd = unit % p.H;
    const int nb = p.T / kB;
    const size_t tok = (size_t)unit * p.T * kD;
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.Q) + tok;
    const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(p.K) + tok;
    const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(p.V) + tok;
    __nv_bfloat16* Z = p.Z ? static_cast<__nv_bfloat16*>(p.Z) + tok : nullptr;
    const int f0 = 16 * w;
    const float inv_d = 1.f / kD;

    // W (fp32): rows f0 + r (+8), columns 8 nt + 2c (+1)
    float wr[8][4];
    {
        const float* W0 = p.W0 + (size_t)n * p.W0_bstride + (size_t)hd * kD * kD;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 v = *reinterpret_cast<const float2*>(W0 + (size_t)(f0 + r + 8 * h) * kD + 8 * nt + 2 * c);
                wr[nt][2 * h] = v.x;
                wr[nt][2 * h + 1] = v.y;
            }
    }
    // c, gamma, beta of this lane's features f0 + 8 nt + 2 c + k
    float cr[2][2], gm[2][2], bt[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int j = f0 + 8 * nt + 2 * c + k;
            cr[nt][k] = p.c0 ? p.c0[(size_t)n * p.c0_bstride + (size_t)hd * kD + j] : 0.f;
            gm[nt][k] = p.gamma[(size_t)hd * kD + j];
            bt[nt][k] = p.beta[(size_t)hd * kD + j];
        }
    uint4 pkq[2];
    uint32_t pv[2][2];
    float pe = 0.f;
    auto prefetch = [&](int i) {
        const int t0 = i * kB, row = tid >> 3, ch = tid & 7;
        const size_t gi = (size_t)(t0 + row) * kD + 8 * ch;
        pkq[0] = *reinterpret_cast<const uint4*>(K + gi);
        pkq[1] = *reinterpret_cast<const uint4*>(Q + gi);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                pv[nt][h] = *reinterpret_cast<const uint32_t*>(V + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c);
        if (tid < kB) pe = p.eta ? p.eta[(size_t)unit * p.T + t0 + tid] : p.eta_const;
    };
    if (nb > 0) prefetch(0);
    for (int i = 0; i < nb; ++i) {
        const int t0 = i * kB;
        // ---- batch-start state to the checkpoints (fp32) and to shared memory (bf16 W); the tiles
        float* Ws = p.W_states + ((size_t)unit * nb + i) * kD * kD;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = f0 + r + 8 * h;
                *reinterpret_cast<float2*>(Ws + (size_t)row * kD + 8 * nt + 2 * c) =
                    make_float2(wr[nt][2 * h], wr[nt][2 * h + 1]);
                *reinterpret_cast<uint32_t*>(smem + kLFOffW + toff(row, nt) + 4 * c) =
                    pk(wr[nt][2 * h], wr[nt][2 * h + 1]);
            }
        if (r == 0)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int k = 0; k < 2; ++k)
                    p.c_states[((size_t)unit * nb + i) * kD + f0 + 8 * nt + 2 * c + k] = cr[nt][k];
        uint32_t vcur[2][2];
        {
            const int row = tid >> 3, ch = tid & 7;
            *reinterpret_cast<uint4*>(smem + kLFOffK + toff(row, ch)) = pkq[0];
            *reinterpret_cast<uint4*>(smem + kLFOffQ + toff(row, ch)) = pkq[1];
            if (tid < kB) s_eta[tid] = pe;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) vcur[nt][h] = pv[nt][h];
        }
        if (i + 1 < nb) prefetch(i + 1);
        __syncthreads();
        const float eta_r[2] = {s_eta[r], s_eta[r + 8]};
        // ---- Y = K W + c and P0 = Q W + c on this warp's features
        float y[2][4], z[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) y[nt][q] = z[nt][q] = cr[nt][q & 1];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4], aq[4], b[4];
            ldsm4(a_addr(sK, 0, ks, l), a);
            ldsm4(a_addr(sQ, 0, ks, l), aq);
            ldsm4t(bt_addr(sW, f0, ks, l), b);
            mma(y[0], a, b[0], b[1]);
            mma(y[1], a, b[2], b[3]);
            mma(z[0], aq, b[0], b[1]);
            mma(z[1], aq, b[2], b[3]);
        }
        // ---- LN of the rows of Y
        float sy[2][2] = {};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                sy[0][q >> 1] += y[nt][q];
                sy[1][q >> 1] += y[nt][q] * y[nt][q];
            }
        row_sums<2>(sy, red, w, r, c);
        float rr[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float mu = sy[0][h] * inv_d;
            rr[h] = rsqrtf(fmaxf(sy[1][h] * inv_d - mu * mu, 0.f) + p.eps);
            sy[0][h] = mu;
        }
        // Xh (in y), G = gamma E (in z's place later: kept in g_), and the sums of G and G Xh
        float g_[2][4], sg[2][2] = {};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 kv = tile_pair(smem, kLFOffK, r + 8 * h, f0, nt, c);
                const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&vcur[nt][h]);
                const float vv[2] = {__bfloat162float(v2.x), __bfloat162float(v2.y)};
                const float kk[2] = {kv.x, kv.y};
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int q = 2 * h + k;
                    const float x = (y[nt][q] - sy[0][h]) * rr[h];
                    y[nt][q] = x;
                    const float g = gm[nt][k] * (kk[k] + gm[nt][k] * x + bt[nt][k] - vv[k]);
                    g_[nt][q] = g;
                    sg[0][h] += g;
                    sg[1][h] += g * x;
                }
            }
        row_sums<2>(sg, red + kRedFloats, w, r, c);
        // A = diag(eta) r (G - mean(G) - Xh mean(G Xh)) -> shared (bf16); fp32 copy for the bias update
        float av[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int h = q >> 1;
                av[nt][q] = eta_r[h] * rr[h] * (g_[nt][q] - sg[0][h] * inv_d - y[nt][q] * sg[1][h] * inv_d);
            }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint32_t*>(smem + kLFOffA + toff(r + 8 * h, (f0 >> 3) + nt) + 4 * c) =
                    pk(av[nt][2 * h], av[nt][2 * h + 1]);
        // ---- -M = -tril(Q K^T + 1) as an A operand
        uint32_t mA[4];
        {
            float x[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4];
                ldsm4(a_addr(sQ, 0, ks, l), a);
                ldsm4(b_addr(sK, 0, ks, l), b);
                mma(x[0], a, b[0], b[1]);
                mma(x[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    x[nt][q] = (8 * nt + 2 * c + (q & 1) > r + 8 * (q >> 1)) ? 0.f : -(x[nt][q] + 1.f);
            acc_to_a(x, mA);
        }
        __syncthreads();   // A complete (every feature: the state update reads all of it)
        // ---- P = P0 - M A, its LN, Z = Q + gamma LN(P) + beta
        {
            uint32_t b[4];
            ldsm4t(bt_addr(sA, f0, 0, l), b);
            mma(z[0], mA, b[0], b[1]);
            mma(z[1], mA, b[2], b[3]);
        }
        if (Z) {
            float sz[2][2] = {};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sz[0][q >> 1] += z[nt][q];
                    sz[1][q >> 1] += z[nt][q] * z[nt][q];
                }
            row_sums<2>(sz, red + 2 * kRedFloats, w, r, c);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float mu = sz[0][h] * inv_d;
                const float ro = rsqrtf(fmaxf(sz[1][h] * inv_d - mu * mu, 0.f) + p.eps);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const float2 qv = tile_pair(smem, kLFOffQ, r + 8 * h, f0, nt, c);
                    const float o0 = qv.x + gm[nt][0] * (z[nt][2 * h] - mu) * ro + bt[nt][0];
                    const float o1 = qv.y + gm[nt][1] * (z[nt][2 * h + 1] - mu) * ro + bt[nt][1];
                    *reinterpret_cast<__nv_bfloat162*>(Z + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c) =
                        __floats2bfloat162_rn(o0, o1);
                }
            }
        }
        // ---- W <- W - K^T A on this warp's state rows (the K^T fragment negated); c <- c - 1^T A
        {
            uint32_t ak[4];
            ldsm4t(at_addr(sK, f0, l), ak);
#pragma unroll
            for (int q = 0; q < 4; ++q) ak[q] ^= 0x80008000u;
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b[4];
                ldsm4t(bt_addr(sA, 16 * np, 0, l), b);
                mma(wr[2 * np], ak, b[0], b[1]);
                mma(wr[2 * np + 1], ak, b[2], b[3]);
            }
        }
        {
            float cs[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int k = 0; k < 2; ++k) cs[nt][k] = av[nt][k] + av[nt][2 + k];
            col_sums(cs);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int k = 0; k < 2; ++k) cr[nt][k] -= cs[nt][k];
        }
        __syncthreads();   // every read of this mini-batch's shared tiles is done
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<float2*>(p.W_out + (size_t)unit * kD * kD + (size_t)(f0 + r + 8 * h) * kD + 8 * nt + 2 * c) =
                make_float2(wr[nt][2 * h], wr[nt][2 * h + 1]);
    if (p.c_out && r == 0)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int k = 0; k < 2; ++k) p.c_out[(size_t)unit * kD + f0 + 8 * nt + 2 * c + k] = cr[nt][k];
}

__global__ void __launch_bounds__(kThreads) mma_ln_backward_kernel(SimtLnBackwardParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sW = smem_u32(smem + kLBOffW), sG = smem_u32(smem + kLBOffG), sK = smem_u32(smem + kLBOffK);
    const uint32_t sQ = smem_u32(smem + kLBOffQ), sDZ = smem_u32(smem + kLBOffDZ), sA = smem_u32(smem + kLBOffA);
    const uint32_t sDP = smem_u32(smem + kLBOffDP), sDY = smem_u32(smem + kLBOffDY);
    float* s_eta = reinterpret_cast<float*>(smem + kLBOffEta);
    float* red = reinterpret_cast<float*>(smem + kLBOffRed);
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, r = l >> 2, c = l & 3;
    const int unit = blockIdx.x, hd = unit % p.H;
    const int nb = p.T / kB;
    const size_t tok = (size_t)unit * p.T * kD;
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.Q) + tok;
    const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(p.K) + tok;
    const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(p.V) + tok;
    const __nv_bfloat16* dZ = p.dZ ? static_cast<const __nv_bfloat16*>(p.dZ) + tok : nullptr;
    __nv_bfloat16* dQ = static_cast<__nv_bfloat16*>(p.dQ) + tok;
    __nv_bfloat16* dK = static_cast<__nv_bfloat16*>(p.dK) + tok;
    __nv_bfloat16* dV = static_cast<__nv_bfloat16*>(p.dV) + tok;
    const int f0 = 16 * w;
    const float inv_d = 1.f / kD;

    // GW (fp32): state rows f0 + r (+8), columns 8 nt + 2c (+1)
    float g[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            g[nt][e] = p.dW_out ? p.dW_out[(size_t)unit * kD * kD + (size_t)(f0 + r + 8 * (e >> 1)) * kD +
                                           8 * nt + 2 * c + (e & 1)]
                                : 0.f;
    // per-lane values of this lane's features f0 + 8 nt + 2 c + k: gamma, beta, Gc (replicated over the
    // lane's rows), and the lane's partial sums of dgamma and dbeta (its rows only)
    float gm[2][2], bt[2][2], gc[2][2], dgp[2][2] = {}, dbp[2][2] = {};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int j = f0 + 8 * nt + 2 * c + k;
            gm[nt][k] = p.gamma[(size_t)hd * kD + j];
            bt[nt][k] = p.beta[(size_t)hd * kD + j];
            gc[nt][k] = p.dc_out ? p.dc_out[(size_t)unit * kD + j] : 0.f;
        }
    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * kB;
        // ---- operands: batch-start state (bf16 W, fp32 c), bf16 GW, tiles K, Q, dZ, V pairs, eta
        {
            const float4* Ws = reinterpret_cast<const float4*>(p.W_states + ((size_t)unit * nb + i) * kD * kD);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int idx = tid + kThreads * q;   // float4 index: row idx / 16, columns 4 (idx % 16) ..
                const float4 v = Ws[idx];
                const int row = idx >> 4, c4 = idx & 15;
                *reinterpret_cast<uint2*>(smem + kLBOffW + toff(row, c4 >> 1) + 8 * (c4 & 1)) =
                    make_uint2(pk(v.x, v.y), pk(v.z, v.w));
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<uint32_t*>(smem + kLBOffG + toff(f0 + r + 8 * h, nt) + 4 * c) =
                        pk(g[nt][2 * h], g[nt][2 * h + 1]);
            const int row = tid >> 3, ch = tid & 7;
            const size_t gi = (size_t)(t0 + row) * kD + 8 * ch;
            *reinterpret_cast<uint4*>(smem + kLBOffK + toff(row, ch)) = *reinterpret_cast<const uint4*>(K + gi);
            *reinterpret_cast<uint4*>(smem + kLBOffQ + toff(row, ch)) = *reinterpret_cast<const uint4*>(Q + gi);
            *reinterpret_cast<uint4*>(smem + kLBOffDZ + toff(row, ch)) =
                dZ ? *reinterpret_cast<const uint4*>(dZ + gi) : make_uint4(0u, 0u, 0u, 0u);
            if (tid < kB) s_eta[tid] = p.eta ? p.eta[(size_t)unit * p.T + t0 + tid] : p.eta_const;
        }
        float cr[2][2];
        uint32_t vcur[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int k = 0; k < 2; ++k)
                cr[nt][k] = p.c_states[((size_t)unit * nb + i) * kD + f0 + 8 * nt + 2 * c + k];
#pragma unroll
            for (int h = 0; h < 2; ++h)
                vcur[nt][h] = *reinterpret_cast<const uint32_t*>(V + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c);
        }
        __syncthreads();
        const float eta_r[2] = {s_eta[r], s_eta[r + 8]};
        // ---- forward of the mini-batch: Y = K W + c, P0 = Q W + c
        float xh[2][4], z[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) xh[nt][q] = z[nt][q] = cr[nt][q & 1];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4], aq[4], b[4];
            ldsm4(a_addr(sK, 0, ks, l), a);
            ldsm4(a_addr(sQ, 0, ks, l), aq);
            ldsm4t(bt_addr(sW, f0, ks, l), b);
            mma(xh[0], a, b[0], b[1]);
            mma(xh[1], a, b[2], b[3]);
            mma(z[0], aq, b[0], b[1]);
            mma(z[1], aq, b[2], b[3]);
        }
        // LN of Y: Xh (in place), r
        float rr[2];
        {
            float sy[2][2] = {};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sy[0][q >> 1] += xh[nt][q];
                    sy[1][q >> 1] += xh[nt][q] * xh[nt][q];
                }
            row_sums<2>(sy, red, w, r, c);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float mu = sy[0][h] * inv_d;
                rr[h] = rsqrtf(fmaxf(sy[1][h] * inv_d - mu * mu, 0.f) + p.eps);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int k = 0; k < 2; ++k) xh[nt][2 * h + k] = (xh[nt][2 * h + k] - mu) * rr[h];
            }
        }
        // E = K + gamma Xh + beta - V; mean(G), mean(G Xh) with G = gamma E
        float ev[2][4], mg[2], mgx[2];
        {
            float sg[2][2] = {};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float2 kv = tile_pair(smem, kLBOffK, r + 8 * h, f0, nt, c);
                    const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&vcur[nt][h]);
                    const float vv[2] = {__bfloat162float(v2.x), __bfloat162float(v2.y)};
                    const float kk[2] = {kv.x, kv.y};
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int q = 2 * h + k;
                        const float e = kk[k] + gm[nt][k] * xh[nt][q] + bt[nt][k] - vv[k];
                        ev[nt][q] = e;
                        sg[0][h] += gm[nt][k] * e;
                        sg[1][h] += gm[nt][k] * e * xh[nt][q];
                    }
                }
            row_sums<2>(sg, red + kRedFloats, w, r, c);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mg[h] = sg[0][h] * inv_d;
                mgx[h] = sg[1][h] * inv_d;
            }
        }
        // U = G - mean(G) - Xh mean(G Xh),  Delta = r U,  A = eta Delta -> shared (bf16)
        auto u_of = [&](int nt, int q) {
            return gm[nt][q & 1] * ev[nt][q] - mg[q >> 1] - xh[nt][q] * mgx[q >> 1];
        };
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint32_t*>(smem + kLBOffA + toff(r + 8 * h, (f0 >> 3) + nt) + 4 * c) =
                    pk(eta_r[h] * rr[h] * u_of(nt, 2 * h), eta_r[h] * rr[h] * u_of(nt, 2 * h + 1));
        // -M = -tril(Q K^T + 1) and M^T = triu(K Q^T + 1) as A operands
        uint32_t mA[4], mtA[4];
        {
            float x[2][4] = {}, y[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4], a2[4], b2[4];
                ldsm4(a_addr(sQ, 0, ks, l), a);
                ldsm4(b_addr(sK, 0, ks, l), b);
                mma(x[0], a, b[0], b[1]);
                mma(x[1], a, b[2], b[3]);
                ldsm4(a_addr(sK, 0, ks, l), a2);
                ldsm4(b_addr(sQ, 0, ks, l), b2);
                mma(y[0], a2, b2[0], b2[1]);
                mma(y[1], a2, b2[2], b2[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int row = r + 8 * (q >> 1), col = 8 * nt + 2 * c + (q & 1);
                    x[nt][q] = col > row ? 0.f : -(x[nt][q] + 1.f);
                    y[nt][q] = row > col ? 0.f : y[nt][q] + 1.f;
                }
            acc_to_a(x, mA);
            acc_to_a(y, mtA);
        }
        __syncthreads();   // A complete
        // ---- P = P0 - M A, Xo = LN(P), dP = LN adjoint of gamma dZ -> shared (bf16); dgamma, dbeta
        float dp[2][4];
        {
            uint32_t b[4];
            ldsm4t(bt_addr(sA, f0, 0, l), b);
            mma(z[0], mA, b[0], b[1]);
            mma(z[1], mA, b[2], b[3]);
            float sz[2][2] = {};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sz[0][q >> 1] += z[nt][q];
                    sz[1][q >> 1] += z[nt][q] * z[nt][q];
                }
            row_sums<2>(sz, red + 2 * kRedFloats, w, r, c);
            float ro[2], sd[2][2] = {};
            float dz[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float mu = sz[0][h] * inv_d;
                ro[h] = rsqrtf(fmaxf(sz[1][h] * inv_d - mu * mu, 0.f) + p.eps);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const float2 dv = tile_pair(smem, kLBOffDZ, r + 8 * h, f0, nt, c);
                    dz[nt][2 * h] = dv.x;
                    dz[nt][2 * h + 1] = dv.y;
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int q = 2 * h + k;
                        const float xo = (z[nt][q] - mu) * ro[h];
                        z[nt][q] = xo;
                        const float gd = gm[nt][k] * dz[nt][q];
                        sd[0][h] += gd;
                        sd[1][h] += gd * xo;
                        dgp[nt][k] += dz[nt][q] * xo;
                        dbp[nt][k] += dz[nt][q];
                    }
                }
            }
            row_sums<2>(sd, red + 3 * kRedFloats, w, r, c);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int h = q >> 1;
                    dp[nt][q] = ro[h] * (gm[nt][q & 1] * dz[nt][q] - sd[0][h] * inv_d - z[nt][q] * sd[1][h] * inv_d);
                }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<uint32_t*>(smem + kLBOffDP + toff(r + 8 * h, (f0 >> 3) + nt) + 4 * c) =
                        pk(dp[nt][2 * h], dp[nt][2 * h + 1]);
            // dQ starts as dZ (kept in z's registers from here on)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) z[nt][q] = dz[nt][q];
        }
        __syncthreads();   // dP complete
        // ---- dM = -mask(dP A^T) and dM^T = -mask(A dP^T) as A operands
        uint32_t dmA[4], dmtA[4];
        {
            float x[2][4] = {}, y[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4], a2[4], b2[4];
                ldsm4(a_addr(sDP, 0, ks, l), a);
                ldsm4(b_addr(sA, 0, ks, l), b);
                mma(x[0], a, b[0], b[1]);
                mma(x[1], a, b[2], b[3]);
                ldsm4(a_addr(sA, 0, ks, l), a2);
                ldsm4(b_addr(sDP, 0, ks, l), b2);
                mma(y[0], a2, b2[0], b2[1]);
                mma(y[1], a2, b2[2], b2[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int row = r + 8 * (q >> 1), col = 8 * nt + 2 * c + (q & 1);
                    x[nt][q] = col > row ? 0.f : -x[nt][q];   // dM: rows t, columns s <= t
                    y[nt][q] = row > col ? 0.f : -y[nt][q];   // dM^T: rows s, columns t >= s
                }
            acc_to_a(x, dmA);
            acc_to_a(y, dmtA);
        }
        // ---- dA = -(M^T dP + K GW) - Gc on this warp's features
        float da[2][4] = {};
        {
            uint32_t b[4];
            ldsm4t(bt_addr(sDP, f0, 0, l), b);
            mma(da[0], mtA, b[0], b[1]);
            mma(da[1], mtA, b[2], b[3]);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], bg[4];
                ldsm4(a_addr(sK, 0, ks, l), a);
                ldsm4t(bt_addr(sG, f0, ks, l), bg);
                mma(da[0], a, bg[0], bg[1]);
                mma(da[1], a, bg[2], bg[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) da[nt][q] = -da[nt][q] - gc[nt][q & 1];
        }
        // ---- dQ = dZ + dP W^T + dM K
        {
            uint32_t b[4];
            ldsm4t(bt_addr(sK, f0, 0, l), b);
            mma(z[0], dmA, b[0], b[1]);
            mma(z[1], dmA, b[2], b[3]);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], bw[4];
                ldsm4(a_addr(sDP, 0, ks, l), a);
                ldsm4(b_addr(sW, f0, ks, l), bw);
                mma(z[0], a, bw[0], bw[1]);
                mma(z[1], a, bw[2], bw[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<__nv_bfloat162*>(dQ + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c) =
                        __floats2bfloat162_rn(z[nt][2 * h], z[nt][2 * h + 1]);
        }
        // ---- deta, dDelta = eta dA, and the LN+residual backward of each row to de and dY
        float dy[2][4];
        {
            // [deta, dr = dDelta . U, sum dU, sum dU Xh] with dU = r dDelta
            float s4[4][2] = {};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int h = q >> 1;
                    const float u = u_of(nt, q);
                    const float dd = eta_r[h] * da[nt][q];
                    s4[0][h] += da[nt][q] * rr[h] * u;
                    s4[1][h] += dd * u;
                    s4[2][h] += rr[h] * dd;
                    s4[3][h] += rr[h] * dd * xh[nt][q];
                    da[nt][q] = dd;   // dDelta from here on
                }
            row_sums<4>(s4, red + 4 * kRedFloats, w, r, c);
            if (w == 0 && c == 0 && p.deta) {
                p.deta[(size_t)unit * p.T + t0 + r] = s4[0][0];
                p.deta[(size_t)unit * p.T + t0 + r + 8] = s4[0][1];
            }
            float sx[2][2] = {};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float dv[2];
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int q = 2 * h + k;
                        const float x = xh[nt][q];
                        const float du = rr[h] * da[nt][q];
                        const float dg = du - s4[2][h] * inv_d - x * s4[3][h] * inv_d;
                        const float de = gm[nt][k] * dg;
                        const float dx = -du * mgx[h] - gm[nt][k] * ev[nt][q] * s4[3][h] * inv_d + gm[nt][k] * de;
                        dgp[nt][k] += ev[nt][q] * dg + x * de;
                        dbp[nt][k] += de;
                        dv[k] = -de;
                        ev[nt][q] = de;   // de from here on
                        dy[nt][q] = dx;   // dXh for now
                        sx[0][h] += dx;
                        sx[1][h] += dx * x;
                    }
                    *reinterpret_cast<__nv_bfloat162*>(dV + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c) =
                        __floats2bfloat162_rn(dv[0], dv[1]);
                }
            row_sums<2>(sx, red + 5 * kRedFloats, w, r, c);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int h = q >> 1;
                    const float x = xh[nt][q];
                    dy[nt][q] = rr[h] * (dy[nt][q] - sx[0][h] * inv_d - x * sx[1][h] * inv_d) -
                                s4[1][h] * rr[h] * rr[h] * x * inv_d;
                }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<uint32_t*>(smem + kLBOffDY + toff(r + 8 * h, (f0 >> 3) + nt) + 4 * c) =
                        pk(dy[nt][2 * h], dy[nt][2 * h + 1]);
        }
        __syncthreads();   // dY complete
        // ---- dK = de + dM^T Q - A GW^T + dY W^T
        {
            float x[2][4], ag[2][4] = {};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) x[nt][q] = ev[nt][q];
            uint32_t b[4];
            ldsm4t(bt_addr(sQ, f0, 0, l), b);
            mma(x[0], dmtA, b[0], b[1]);
            mma(x[1], dmtA, b[2], b[3]);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], bg[4], ay[4], bw[4];
                ldsm4(a_addr(sA, 0, ks, l), a);
                ldsm4(b_addr(sG, f0, ks, l), bg);
                mma(ag[0], a, bg[0], bg[1]);
                mma(ag[1], a, bg[2], bg[3]);
                ldsm4(a_addr(sDY, 0, ks, l), ay);
                ldsm4(b_addr(sW, f0, ks, l), bw);
                mma(x[0], ay, bw[0], bw[1]);
                mma(x[1], ay, bw[2], bw[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<__nv_bfloat162*>(dK + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c) =
                        __floats2bfloat162_rn(x[nt][2 * h] - ag[nt][2 * h], x[nt][2 * h + 1] - ag[nt][2 * h + 1]);
        }
        // ---- GW += Q^T dP + K^T dY on this warp's state rows;  Gc += 1^T dP + 1^T dY
        {
            uint32_t aq[4], ak[4];
            ldsm4t(at_addr(sQ, f0, l), aq);
            ldsm4t(at_addr(sK, f0, l), ak);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b[4], bd[4];
                ldsm4t(bt_addr(sDP, 16 * np, 0, l), b);
                mma(g[2 * np], aq, b[0], b[1]);
                mma(g[2 * np + 1], aq, b[2], b[3]);
                ldsm4t(bt_addr(sDY, 16 * np, 0, l), bd);
                mma(g[2 * np], ak, bd[0], bd[1]);
                mma(g[2 * np + 1], ak, bd[2], bd[3]);
            }
            float cs[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int k = 0; k < 2; ++k) cs[nt][k] = dp[nt][k] + dp[nt][2 + k] + dy[nt][k] + dy[nt][2 + k];
            col_sums(cs);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int k = 0; k < 2; ++k) gc[nt][k] += cs[nt][k];
        }
        __syncthreads();   // every read of this mini-batch's tiles is done
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<float2*>(p.dW0 + (size_t)unit * kD * kD + (size_t)(f0 + r + 8 * h) * kD + 8 * nt + 2 * c) =
                make_float2(g[nt][2 * h], g[nt][2 * h + 1]);
    col_sums(dgp);
    col_sums(dbp);
    if (r == 0)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const size_t j = (size_t)unit * kD + f0 + 8 * nt + 2 * c + k;
                p.dc0[j] = gc[nt][k];
                p.dgamma[j] = dgp[nt][k];
                p.dbeta[j] = dbp[nt][k];
            }
}

}  // namespace mbk
}  // namespace ttt
