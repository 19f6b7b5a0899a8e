// Tensor-core (mma.sync, bf16 operands, fp32 accumulation) TTT-Linear
// prefill for d = 64, b = 16, bf16 inputs and outputs, that also writes the
// state at the start of every mini-batch (the checkpoints the backward
// reads; paper digest "论文速览 | TTT", section 6.12).  Per mini-batch, in
// the dual form of section 3.6, with W the batch-start state and
// A = diag(eta) (K W - V):
//     Z = Q W - tril(Q K^T) A,     W <- W - K^T A.
// The fp32 state stays in registers as the accumulator of the update; the
// products read a bf16 copy of it (as the tcgen05 forward does).
//
// One CTA of four warps per (sequence, head) unit.  Warp w owns the features
// 16 w .. 16 w + 15 of E and Z and the state rows 16 w .. 16 w + 15 of W.
// Tiles are bf16 in shared memory with 128-byte rows and row-swizzled
// 16-byte chunks, as in the tensor-core backward.
#pragma once
#include "mma_backward.cuh"

namespace ttt {
namespace mbk {

struct FwdStatesParams {
    int H, T;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W0;
    long long W0_bstride;
    void* Z;
    float* W_out;
    float* W_states;   // [units, T/16, 64, 64]
};

// shared memory (bytes): W (bf16 64 x 64), tiles K, Q, A (bf16 16 x 64), eta
constexpr int kFOffW = 0, kFOffK = 8192, kFOffQ = kFOffK + 2048, kFOffA = kFOffQ + 2048, kFOffEta = kFOffA + 2048;
constexpr int kFSmemBytes = kFOffEta + 64;

__global__ void __launch_bounds__(kThreads) mma_linear_forward_states_kernel(FwdStatesParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sW = smem_u32(smem + kFOffW), sK = smem_u32(smem + kFOffK), sQ = smem_u32(smem + kFOffQ);
    const uint32_t sA = smem_u32(smem + kFOffA);
    float* s_eta = reinterpret_cast<float*>(smem + kFOffEta);
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, r = l >> 2, c = l & 3;
    const int unit = blockIdx.x;
    const int n = unit / p.H, hd = unit % p.H;
    const int nb = p.T / kB;
    const size_t tok = (size_t)unit * p.T * kD;
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.Q) + tok;
    const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(p.K) + tok;
    const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(p.V) + tok;
    __nv_bfloat16* Z = static_cast<__nv_bfloat16*>(p.Z) + tok;
    const int f0 = 16 * w;

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
    // the next mini-batch's tiles are loaded into registers while the current one computes
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
        // ---- batch-start state: fp32 to the checkpoints, bf16 to shared memory; the tiles
        float* Ws = p.W_states + ((size_t)unit * nb + i) * kD * kD;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = f0 + r + 8 * h;
                *reinterpret_cast<float2*>(Ws + (size_t)row * kD + 8 * nt + 2 * c) =
                    make_float2(wr[nt][2 * h], wr[nt][2 * h + 1]);
                *reinterpret_cast<uint32_t*>(smem + kFOffW + toff(row, nt) + 4 * c) =
                    pk(wr[nt][2 * h], wr[nt][2 * h + 1]);
            }
        uint32_t vcur[2][2];
        {
            const int row = tid >> 3, ch = tid & 7;
            *reinterpret_cast<uint4*>(smem + kFOffK + toff(row, ch)) = pkq[0];
            *reinterpret_cast<uint4*>(smem + kFOffQ + toff(row, ch)) = pkq[1];
            if (tid < kB) s_eta[tid] = pe;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) vcur[nt][h] = pv[nt][h];
        }
        if (i + 1 < nb) prefetch(i + 1);
        __syncthreads();
        const float eta_r[2] = {s_eta[r], s_eta[r + 8]};
        // ---- E = K W - V on this warp's features; A = diag(eta) E -> shared
        float e[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&vcur[nt][h]);
                e[nt][2 * h] = -__bfloat162float(v2.x);
                e[nt][2 * h + 1] = -__bfloat162float(v2.y);
            }
        float z[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4], aq[4], b[4];
            ldsm4(a_addr(sK, 0, ks, l), a);
            ldsm4(a_addr(sQ, 0, ks, l), aq);
            ldsm4t(bt_addr(sW, f0, ks, l), b);
            mma(e[0], a, b[0], b[1]);
            mma(e[1], a, b[2], b[3]);
            mma(z[0], aq, b[0], b[1]);   // Q W on the same operand
            mma(z[1], aq, b[2], b[3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint32_t*>(smem + kFOffA + toff(r + 8 * h, (f0 >> 3) + nt) + 4 * c) =
                    pk(eta_r[h] * e[nt][2 * h], eta_r[h] * e[nt][2 * h + 1]);
        // ---- M = tril(Q K^T): rows t, columns s, kept where s <= t; negated for Z = Q W - M A
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
                    x[nt][q] = (8 * nt + 2 * c + (q & 1) > r + 8 * (q >> 1)) ? 0.f : -x[nt][q];
            acc_to_a(x, mA);
        }
        __syncthreads();   // A complete (every feature: the state update reads all of it)
        // ---- Z = Q W - M A on this warp's features
        {
            uint32_t b[4];
            ldsm4t(bt_addr(sA, f0, 0, l), b);
            mma(z[0], mA, b[0], b[1]);
            mma(z[1], mA, b[2], b[3]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<__nv_bfloat162*>(Z + (size_t)(t0 + r + 8 * h) * kD + f0 + 8 * nt + 2 * c) =
                        __floats2bfloat162_rn(z[nt][2 * h], z[nt][2 * h + 1]);
        }
        // ---- W <- W - K^T A on this warp's state rows (the K^T fragment negated)
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
        __syncthreads();   // every read of this mini-batch's shared tiles is done
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<float2*>(p.W_out + (size_t)unit * kD * kD + (size_t)(f0 + r + 8 * h) * kD + 8 * nt + 2 * c) =
                make_float2(wr[nt][2 * h], wr[nt][2 * h + 1]);
}

}  // namespace mbk
}  // namespace ttt
