// Tensor-core (mma.sync, bf16 operands, fp32 accumulation) kernel of the
// TTT-Linear backward for d = 64, b = 16 with bf16 inputs and outputs.  It
// computes the same reverse step as the fp32 CUDA-core kernel
// (simt_backward.cuh; paper digest "论文速览 | TTT", sections 3.4, 3.6 and
// 6.12), with W the batch-start state, A = diag(eta) E, M = tril(Q K^T),
// G = dL/d(state after the mini-batch):
//     E = K W - V
//     P = mask(dZ A^T),  P^T = mask(A dZ^T),  M^T = triu(K Q^T)
//     dA = -M^T dZ - K G,   dE = diag(eta) dA,   deta_t = dA_t . E_t
//     dQ = dZ W^T - P K,    dK = -P^T Q - A G^T + dE W^T,   dV = -dE
//     G <- G + Q^T dZ + K^T dE
// Products take bf16 copies of W, G, A, dE and of the 16 x 16 causal
// matrices (the tensor-core forward rounds W the same way); G itself is
// accumulated in fp32 registers for the whole reverse sweep.
//
// One CTA of four warps per (sequence, head) unit.  Warp w owns the features
// 16 w .. 16 w + 15 of every 16 x 64 product (dA, dQ, dK, E) and the state
// rows 16 w .. 16 w + 15 of G; the 16 x 16 causal matrices are computed by
// every warp.  Operand tiles are bf16 in shared memory with 128-byte rows
// and the 16-byte chunks XOR-swizzled by the row (conflict-free ldmatrix).
#pragma once
#include "common.cuh"
#include "simt_backward.cuh"

namespace ttt {
namespace mbk {

constexpr int kD = 64, kB = 16, kThreads = 128;
// shared memory (bytes): W and G (bf16 64 x 64), tiles K, Q, dZ, A, dE (bf16 16 x 64),
// eta (16 floats), per-warp deta partials (4 x 16 floats)
constexpr int kOffW = 0, kOffG = 8192, kOffK = 16384, kOffQ = kOffK + 2048, kOffDZ = kOffQ + 2048;
constexpr int kOffA = kOffDZ + 2048, kOffDE = kOffA + 2048, kOffEta = kOffDE + 2048, kOffDP = kOffEta + 64;
constexpr int kSmemBytes = kOffDP + 256;

__device__ __forceinline__ uint32_t toff(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

// The three warp-collective operations (ldmatrix x4, its transposing form, and
// the m16n8k16 bf16 MMA).  The CPU test suite's host emulation of these
// kernels supplies its own definitions, written from the same documented
// fragment layouts, and defines TTT_HOST_EMULATION.
#ifndef TTT_HOST_EMULATION
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
#endif
__device__ __forceinline__ uint32_t pk(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
// A fragment (rows m, k = 16 columns) from a 16 x 16 accumulator pair
__device__ __forceinline__ void acc_to_a(const float (&x)[2][4], uint32_t* a) {
    a[0] = pk(x[0][0], x[0][1]);
    a[1] = pk(x[0][2], x[0][3]);
    a[2] = pk(x[1][0], x[1][1]);
    a[3] = pk(x[1][2], x[1][3]);
}

// ldmatrix lane addresses (l = lane) on a tile with 128-byte rows:
// A operand, rows m0.., k-step ks, tile stored [m][k]
__device__ __forceinline__ uint32_t a_addr(uint32_t t, int m0, int ks, int l) {
    return t + toff(m0 + (l & 15), 2 * ks + (l >> 4));
}
// A operand = X^T, X stored [k][m] (16 k rows), columns m0.. (ldmatrix .trans)
__device__ __forceinline__ uint32_t at_addr(uint32_t t, int m0, int l) {
    return t + toff((l & 7) + 8 * (l >> 4), (m0 >> 3) + ((l >> 3) & 1));
}
// B operand for two n-tiles n0.., n0 + 8.., k-step ks, tile stored [n][k]
__device__ __forceinline__ uint32_t b_addr(uint32_t t, int n0, int ks, int l) {
    return t + toff(n0 + (l & 7) + 8 * (l >> 4), 2 * ks + ((l >> 3) & 1));
}
// B operand for two n-tiles, k-step ks, tile stored [k][n] (ldmatrix .trans)
__device__ __forceinline__ uint32_t bt_addr(uint32_t t, int n0, int ks, int l) {
    return t + toff(16 * ks + (l & 7) + 8 * ((l >> 3) & 1), (n0 >> 3) + (l >> 4));
}

__global__ void __launch_bounds__(kThreads) mma_linear_backward_kernel(SimtBackwardParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sW = smem_u32(smem + kOffW), sG = smem_u32(smem + kOffG), sK = smem_u32(smem + kOffK);
    const uint32_t sQ = smem_u32(smem + kOffQ), sDZ = smem_u32(smem + kOffDZ), sA = smem_u32(smem + kOffA);
    const uint32_t sDE = smem_u32(smem + kOffDE);
    float* s_eta = reinterpret_cast<float*>(smem + kOffEta);
    float* s_dp = reinterpret_cast<float*>(smem + kOffDP);
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, r = l >> 2, c = l & 3;
    const int unit = blockIdx.x;
    const int nb = p.T / kB;
    const size_t tok = (size_t)unit * p.T * kD;
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.Q) + tok;
    const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(p.K) + tok;
    const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(p.V) + tok;
    const __nv_bfloat16* dZ = p.dZ ? static_cast<const __nv_bfloat16*>(p.dZ) + tok : nullptr;
    __nv_bfloat16* dQ = static_cast<__nv_bfloat16*>(p.dQ) + tok;
    __nv_bfloat16* dK = static_cast<__nv_bfloat16*>(p.dK) + tok;
    __nv_bfloat16* dV = static_cast<__nv_bfloat16*>(p.dV) + tok;
    const int f0 = 16 * w;   // this warp's features / state rows

    // G (fp32): rows f0 + r (+8), columns 8 nt + 2c (+1)
    float g[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            g[nt][e] = p.dW_out ? p.dW_out[(size_t)unit * kD * kD + (size_t)(f0 + r + 8 * (e >> 1)) * kD +
                                           8 * nt + 2 * c + (e & 1)]
                                : 0.f;
    // the next mini-batch's operands are loaded into registers while the current one computes
    float4 pw[8];
    uint4 pkq[3];
    uint32_t pv[2][2];
    float pe = 0.f;
    auto prefetch = [&](int i) {
        const float4* Ws = reinterpret_cast<const float4*>(p.W_states + ((size_t)unit * nb + i) * kD * kD);
#pragma unroll
        for (int q = 0; q < 8; ++q) pw[q] = Ws[tid + kThreads * q];
        const int t0 = i * kB, row = tid >> 3, ch = tid & 7;
        const size_t gi = (size_t)(t0 + row) * kD + 8 * ch;
        pkq[0] = *reinterpret_cast<const uint4*>(K + gi);
        pkq[1] = *reinterpret_cast<const uint4*>(Q + gi);
        pkq[2] = dZ ? *reinterpret_cast<const uint4*>(dZ + gi) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                pv[nt][h] = *reinterpret_cast<const uint32_t*>(V + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c);
        if (tid < kB) pe = p.eta ? p.eta[(size_t)unit * p.T + t0 + tid] : p.eta_const;
    };
    if (nb > 0) prefetch(nb - 1);
    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * kB;
        // ---- this mini-batch's operands to shared memory: batch-start state (bf16), G (bf16), K, Q, dZ, eta
        uint32_t vcur[2][2];
        {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int idx = tid + kThreads * q;   // float4 index: row idx / 16, columns 4 (idx % 16) ..
                const float4 v = pw[q];
                const int row = idx >> 4, c4 = idx & 15;
                *reinterpret_cast<uint2*>(smem + kOffW + toff(row, c4 >> 1) + 8 * (c4 & 1)) =
                    make_uint2(pk(v.x, v.y), pk(v.z, v.w));
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<uint32_t*>(smem + kOffG + toff(f0 + r + 8 * h, nt) + 4 * c) =
                        pk(g[nt][2 * h], g[nt][2 * h + 1]);
            const int row = tid >> 3, ch = tid & 7;
            *reinterpret_cast<uint4*>(smem + kOffK + toff(row, ch)) = pkq[0];
            *reinterpret_cast<uint4*>(smem + kOffQ + toff(row, ch)) = pkq[1];
            *reinterpret_cast<uint4*>(smem + kOffDZ + toff(row, ch)) = pkq[2];
            if (tid < kB) s_eta[tid] = pe;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) vcur[nt][h] = pv[nt][h];
        }
        if (i > 0) prefetch(i - 1);
        __syncthreads();
        const float eta_r[2] = {s_eta[r], s_eta[r + 8]};
        // ---- E = K W - V on features f0..f0+15 (rows t = r, r + 8)
        float e[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&vcur[nt][h]);
                e[nt][2 * h] = -__bfloat162float(v2.x);
                e[nt][2 * h + 1] = -__bfloat162float(v2.y);
            }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4], b[4];
            ldsm4(a_addr(sK, 0, ks, l), a);
            ldsm4t(bt_addr(sW, f0, ks, l), b);
            mma(e[0], a, b[0], b[1]);
            mma(e[1], a, b[2], b[3]);
        }
        // A = diag(eta) E -> shared (bf16)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint32_t*>(smem + kOffA + toff(r + 8 * h, (f0 >> 3) + nt) + 4 * c) =
                    pk(eta_r[h] * e[nt][2 * h], eta_r[h] * e[nt][2 * h + 1]);
        // M^T = triu(K Q^T): rows s, columns t, kept where s <= t
        uint32_t mtA[4];
        {
            float x[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4];
                ldsm4(a_addr(sK, 0, ks, l), a);
                ldsm4(b_addr(sQ, 0, ks, l), b);
                mma(x[0], a, b[0], b[1]);
                mma(x[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (r + 8 * (q >> 1) > 8 * nt + 2 * c + (q & 1)) x[nt][q] = 0.f;
            acc_to_a(x, mtA);
        }
        __syncthreads();   // A complete
        // P = mask(dZ A^T) (rows t, columns s, s <= t) and P^T = mask(A dZ^T) (rows s, columns t)
        uint32_t pA[4], ptA[4];
        {
            float x[2][4] = {}, y[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4], a2[4], b2[4];
                ldsm4(a_addr(sDZ, 0, ks, l), a);
                ldsm4(b_addr(sA, 0, ks, l), b);
                mma(x[0], a, b[0], b[1]);
                mma(x[1], a, b[2], b[3]);
                ldsm4(a_addr(sA, 0, ks, l), a2);
                ldsm4(b_addr(sDZ, 0, ks, l), b2);
                mma(y[0], a2, b2[0], b2[1]);
                mma(y[1], a2, b2[2], b2[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int row = r + 8 * (q >> 1), col = 8 * nt + 2 * c + (q & 1);
                    if (col > row) x[nt][q] = 0.f;   // P: keep s <= t
                    if (row > col) y[nt][q] = 0.f;   // P^T: keep s <= t
                }
            acc_to_a(x, pA);
            acc_to_a(y, ptA);
        }
        // dA = -(M^T dZ + K G) on this warp's features
        float da[2][4] = {};
        {
            uint32_t b[4];
            ldsm4t(bt_addr(sDZ, f0, 0, l), b);
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
        }
        // deta partials, dE = diag(eta) dA -> shared (bf16), dV = -dE
        {
            float part[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    da[nt][q] = -da[nt][q];
                    part[q >> 1] += da[nt][q] * e[nt][q];
                }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                part[h] += __shfl_xor_sync(0xffffffffu, part[h], 1);
                part[h] += __shfl_xor_sync(0xffffffffu, part[h], 2);
            }
            if (c == 0) {
                s_dp[w * kB + r] = part[0];
                s_dp[w * kB + r + 8] = part[1];
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float d0 = eta_r[h] * da[nt][2 * h], d1 = eta_r[h] * da[nt][2 * h + 1];
                    da[nt][2 * h] = d0;
                    da[nt][2 * h + 1] = d1;
                    *reinterpret_cast<uint32_t*>(smem + kOffDE + toff(r + 8 * h, (f0 >> 3) + nt) + 4 * c) = pk(d0, d1);
                    *reinterpret_cast<__nv_bfloat162*>(dV + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c) =
                        __floats2bfloat162_rn(-d0, -d1);
                }
        }
        // dQ = dZ W^T - P K on this warp's features
        {
            float x[2][4] = {}, y[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4];
                ldsm4(a_addr(sDZ, 0, ks, l), a);
                ldsm4(b_addr(sW, f0, ks, l), b);
                mma(x[0], a, b[0], b[1]);
                mma(x[1], a, b[2], b[3]);
            }
            uint32_t b[4];
            ldsm4t(bt_addr(sK, f0, 0, l), b);
            mma(y[0], pA, b[0], b[1]);
            mma(y[1], pA, b[2], b[3]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<__nv_bfloat162*>(dQ + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c) =
                        __floats2bfloat162_rn(x[nt][2 * h] - y[nt][2 * h], x[nt][2 * h + 1] - y[nt][2 * h + 1]);
        }
        __syncthreads();   // dE and the deta partials complete
        if (tid < kB && p.deta)
            p.deta[(size_t)unit * p.T + t0 + tid] = s_dp[tid] + s_dp[kB + tid] + s_dp[2 * kB + tid] + s_dp[3 * kB + tid];
        // dK = dE W^T - P^T Q - A G^T on this warp's features
        {
            float x[2][4] = {};
            {
                uint32_t b[4];
                ldsm4t(bt_addr(sQ, f0, 0, l), b);
                mma(x[0], ptA, b[0], b[1]);
                mma(x[1], ptA, b[2], b[3]);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4];
                ldsm4(a_addr(sA, 0, ks, l), a);
                ldsm4(b_addr(sG, f0, ks, l), b);
                mma(x[0], a, b[0], b[1]);
                mma(x[1], a, b[2], b[3]);
            }
            float y[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4];
                ldsm4(a_addr(sDE, 0, ks, l), a);
                ldsm4(b_addr(sW, f0, ks, l), b);
                mma(y[0], a, b[0], b[1]);
                mma(y[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<__nv_bfloat162*>(dK + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c) =
                        __floats2bfloat162_rn(y[nt][2 * h] - x[nt][2 * h], y[nt][2 * h + 1] - x[nt][2 * h + 1]);
        }
        // G += Q^T dZ + K^T dE on this warp's state rows
        {
            uint32_t aq[4], ak[4];
            ldsm4t(at_addr(sQ, f0, l), aq);
            ldsm4t(at_addr(sK, f0, l), ak);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b[4], bd[4];
                ldsm4t(bt_addr(sDZ, 16 * np, 0, l), b);
                mma(g[2 * np], aq, b[0], b[1]);
                mma(g[2 * np + 1], aq, b[2], b[3]);
                ldsm4t(bt_addr(sDE, 16 * np, 0, l), bd);
                mma(g[2 * np], ak, bd[0], bd[1]);
                mma(g[2 * np + 1], ak, bd[2], bd[3]);
            }
        }
        __syncthreads();   // every read of this mini-batch's tiles is done
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<float2*>(p.dW0 + (size_t)unit * kD * kD + (size_t)(f0 + r + 8 * h) * kD + 8 * nt + 2 * c) =
                make_float2(g[nt][2 * h], g[nt][2 * h + 1]);
}

}  // namespace mbk
}  // namespace ttt
