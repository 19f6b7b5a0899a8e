// Tensor-core (mma.sync, bf16 operands, fp32 accumulation) outer-loop backward
// of the TTT-MLP prefill, f(x) = GELU(x W1 + c1) W2 + c2 with m = 4 d, for
// d = 64, b = 16 and bf16 inputs and outputs: the same reverse steps as the
// fp32 CUDA-core kernel (simt_mlp_backward.cuh; paper digest "论文速览 | TTT",
// sections 3.4, 3.7 and 6.12), from the batch-start states the forward writes.
//
// One CTA of eight warps per (sequence, head) unit.  Warp w owns the hidden
// units 32 w .. 32 w + 31 of every 16 x 256 product and the features
// 8 w .. 8 w + 7 of every 16 x 64 product (each 16 x 64 product contracts
// over all 256 hidden units).  Per mini-batch the shared memory holds bf16
// copies of the batch-start state (W1, W2) and of the end-state adjoint
// (GW1, GW2), the token tiles and the mini-batch's 16 x 256 intermediates;
// the 16 x 16 causal matrices are fp32 in shared memory, so a warp builds
// either orientation's mma fragments from them.  The running adjoint is fp32
// in the gradient outputs dW1, dc1, dW2, dc2 (global memory, L2-resident):
// each warp adds its block of this mini-batch's terms after every product
// with the end-state adjoint has read the bf16 copy.
//
// Layouts in shared memory (bf16, 128-byte rows, 16-byte chunks XOR-swizzled
// by the row as in mma_backward.cuh):
//   W1, GW1  [64 a][256 p]: four 64 x 64 tiles, one per 64 hidden units
//   W2, GW2  [256 p][64 j]: one tile of 256 rows
//   16 x 256 intermediates: four 16 x 64 tiles
//   16 x 64 token tiles: one tile
#pragma once
#include "mma_backward.cuh"
#include "simt_mlp_backward.cuh"

namespace ttt {
namespace mmb {

using mbk::acc_to_a;
using mbk::at_addr;
using mbk::a_addr;
using mbk::b_addr;
using mbk::bt_addr;
using mbk::ldsm4;
using mbk::ldsm4t;
using mbk::mma;
using mbk::pk;
using mbk::toff;

constexpr int kD = 64, kM = 256, kB = 16, kThreads = 256;
constexpr int kTileMM = 8192;   // 16 x 256 bf16
constexpr int kTileBD = 2048;   // 16 x 64 bf16
// shared memory (bytes)
constexpr int kOffW1 = 0, kOffW2 = 32768, kOffG1 = 65536, kOffG2 = 98304;
constexpr int kOffHk = 131072, kOffD1 = kOffHk + kTileMM, kOffHq = kOffD1 + kTileMM, kOffDAq = kOffHq + kTileMM;
constexpr int kOffDM = kOffDAq + kTileMM, kOffDA = kOffDM + kTileMM;
constexpr int kOffK = kOffDA + kTileMM, kOffQ = kOffK + kTileBD, kOffDZ = kOffQ + kTileBD, kOffE = kOffDZ + kTileBD;
constexpr int kOffDE = kOffE + kTileBD;
constexpr int kOffP1 = kOffDE + kTileBD;         // fp32 16 x 16: tril(Q K^T + 1)
constexpr int kOffP2 = kOffP1 + 1024;            // tril(Hq Hk^T + 1)
constexpr int kOffL2 = kOffP2 + 1024;            // tril(-dZ E^T)
constexpr int kOffL1 = kOffL2 + 1024;            // tril(-dAq D1^T)
constexpr int kOffPart = kOffL1 + 1024;          // split-K partials: 8 warps x 16 x 16 fp32
constexpr int kOffRow = kOffPart + 8 * 1024;     // per-warp row partials: 8 x 16 fp32
constexpr int kOffEta = kOffRow + 512;
constexpr int kOffX = kOffEta + 64;              // LN row sums: two areas of 8 warps x 16 rows x 4 fp32
constexpr int kSmemBytes = kOffX + 2 * 2048;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// element (row, col) of a [rows][256] bf16 matrix stored as four [rows][64] tiles of `tile` bytes
__device__ __forceinline__ uint32_t mm_off(int tile, int row, int col) {
    return (col >> 6) * tile + toff(row, (col & 63) >> 3) + 2 * (col & 7);
}
// the bf16 pair (row, col .. col + 1) of a swizzled 16 x 64 tile at byte offset `off`, as floats
__device__ __forceinline__ float2 tile_pair_bf16(const uint8_t* smem, int off, int row, int col) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(smem + off + toff(row, col >> 3) + 2 * (col & 7));
    return make_float2(__bfloat162float(v.x), __bfloat162float(v.y));
}
// A fragment of a 16 x 16 fp32 matrix S (row-major in shared memory): rows m, columns k, or the
// transpose (rows m of S^T = columns of S); each column k is scaled by colscale[k] when given
__device__ __forceinline__ void frag_from_f32(const float* S, bool transpose, const float* colscale, int l,
                                              uint32_t* a) {
    const int g = l >> 2, c = l & 3;
    auto el = [&](int row, int col) {
        const float v = transpose ? S[col * 16 + row] : S[row * 16 + col];
        return colscale ? v * colscale[col] : v;
    };
    a[0] = pk(el(g, 2 * c), el(g, 2 * c + 1));
    a[1] = pk(el(g + 8, 2 * c), el(g + 8, 2 * c + 1));
    a[2] = pk(el(g, 2 * c + 8), el(g, 2 * c + 9));
    a[3] = pk(el(g + 8, 2 * c + 8), el(g + 8, 2 * c + 9));
}

// A lane's place in the kernels' layout (warp w, lane l = 4 r + c; hidden units p0 .. p0 + 31; features
// j0 .. j0 + 7 = half jh of the 16-column window jn0) and the products and exchanges built on it
struct Ops {
    uint8_t* smem;
    float* part;
    float* rowp;
    int tid, w, l, r, c, p0, jn0, jh, j0;

    // the per-lane columns of a 16 x 256 product: hidden unit p0 + 8 nt + 2 c + k
    __device__ __forceinline__ int hid(int nt, int k) const { return p0 + 8 * nt + 2 * c + k; }
    // store a warp's 16 x 32 block (four n-tiles) of a 16 x 256 intermediate as bf16
    __device__ __forceinline__ void store_mm(int off, const float (&x)[4][4]) const {
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint32_t*>(smem + off + mm_off(kTileBD, r + 8 * h, hid(nt, 0))) =
                    pk(x[nt][2 * h], x[nt][2 * h + 1]);
    }
    // store a warp's 16 x 8 block of a 16 x 64 product as bf16
    __device__ __forceinline__ void store_bd(int off, const float (&x)[4]) const {
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<uint32_t*>(smem + off + toff(r + 8 * h, j0 >> 3) + 4 * c) = pk(x[2 * h], x[2 * h + 1]);
    }
    // 16 x 32 block (this warp's hidden units) of A (16 x K, [m][k] tile at ta, K = 16 kst) times
    // B[k][p] stored [k][n] in 64-column tiles of `btile` bytes at tb (rows k)
    __device__ __forceinline__ void mm_AB_kn(float (&x)[4][4], uint32_t ta, int a_is_mm, int kst, uint32_t tb, int btile) const {
#pragma unroll 1
        for (int ks = 0; ks < kst; ++ks) {
            uint32_t a[4];
            if (a_is_mm)
                ldsm4(a_addr(ta + (ks >> 2) * kTileBD, 0, ks & 3, l), a);
            else
                ldsm4(a_addr(ta, 0, ks, l), a);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4];
                const int n0 = p0 + 16 * np;
                ldsm4t(bt_addr(tb + (n0 >> 6) * btile, n0 & 63, ks, l), b);
                mma(x[2 * np], a, b[0], b[1]);
                mma(x[2 * np + 1], a, b[2], b[3]);
            }
        }
    }
    // 16 x 32 block of A (16 x 64 token tile at ta) times B[k=j][n=p] = X[p][j], X stored [256 p][64 j] at tb
    __device__ __forceinline__ void mm_A_Xt(float (&x)[4][4], uint32_t ta, uint32_t tb) const {
#pragma unroll 1
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4];
            ldsm4(a_addr(ta, 0, ks, l), a);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4];
                ldsm4(b_addr(tb, p0 + 16 * np, ks, l), b);
                mma(x[2 * np], a, b[0], b[1]);
                mma(x[2 * np + 1], a, b[2], b[3]);
            }
        }
    }
    // 16 x 8 block (this warp's features) of A (16 x 256 intermediate at ta) times
    // B[k=p][n=j] = X[p][j], X stored [256 p][64 j] at tb
    __device__ __forceinline__ void bd_A_X(float (&y)[4], uint32_t ta, uint32_t tb) const {
#pragma unroll 2
        for (int ks = 0; ks < 16; ++ks) {
            uint32_t a[4], b[4];
            ldsm4(a_addr(ta + (ks >> 2) * kTileBD, 0, ks & 3, l), a);
            ldsm4t(bt_addr(tb, jn0, ks, l), b);
            mma(y, a, jh ? b[2] : b[0], jh ? b[3] : b[1]);
        }
    }
    // 16 x 8 block of A (16 x 256 intermediate at ta) times B[k=p][n=a] = X[a][p], X stored [64 a][256 p]
    __device__ __forceinline__ void bd_A_Yt(float (&y)[4], uint32_t ta, uint32_t tb) const {
#pragma unroll 2
        for (int ks = 0; ks < 16; ++ks) {
            uint32_t a[4], b[4];
            ldsm4(a_addr(ta + (ks >> 2) * kTileBD, 0, ks & 3, l), a);
            ldsm4(b_addr(tb + (ks >> 2) * 8192, jn0, ks & 3, l), b);
            mma(y, a, jh ? b[2] : b[0], jh ? b[3] : b[1]);
        }
    }
    // per-row sums over the CTA of the lane's partials v[h] (rows r + 8 h): quad shuffle, per-warp
    // partials in shared memory, one barrier
    __device__ __forceinline__ void row_total(float (&v)[2]) const {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            v[h] += __shfl_xor_sync(0xffffffffu, v[h], 1);
            v[h] += __shfl_xor_sync(0xffffffffu, v[h], 2);
        }
        if (c == 0) {
            rowp[w * kB + r] = v[0];
            rowp[w * kB + r + 8] = v[1];
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float s = 0.f;
#pragma unroll
            for (int ww = 0; ww < 8; ++ww) s += rowp[ww * kB + r + 8 * h];
            v[h] = s;
        }
    }
    // split-K 16 x 16 product over the hidden units: sum over warps of A[:, p0..] B[:, p0..]^T into dst,
    // masked to s <= t and with `add` on the kept entries, scaled by `scale`
    // sums over the CTA's 64 features of rows r and r + 8 for NQ quantities v[k][h], through exchange area
    // `xa` (two areas used in turn, so consecutive calls never overwrite values still being read)
    template <int NQ>
    __device__ __forceinline__ void rows(float (&v)[NQ][2], float* xa) const {
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
                for (int h = 0; h < 2; ++h) xa[(w * kB + r + 8 * h) * 4 + k] = v[k][h];
        __syncthreads();
#pragma unroll
        for (int k = 0; k < NQ; ++k)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float sum = 0.f;
#pragma unroll
                for (int ww = 0; ww < 8; ++ww) sum += xa[(ww * kB + r + 8 * h) * 4 + k];
                v[k][h] = sum;
            }
    }
    __device__ __forceinline__ void tt_split(uint32_t ta, uint32_t tb, float* dst, float add, float scale) const {
        float x[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int ks = 2 * w + kk;   // 16-unit step of this warp's 32 hidden units
            uint32_t a[4], b[4];
            ldsm4(a_addr(ta + (ks >> 2) * kTileBD, 0, ks & 3, l), a);
            ldsm4(b_addr(tb + (ks >> 2) * kTileBD, 0, ks & 3, l), b);
            mma(x[0], a, b[0], b[1]);
            mma(x[1], a, b[2], b[3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) part[w * 256 + (r + 8 * (q >> 1)) * 16 + 8 * nt + 2 * c + (q & 1)] = x[nt][q];
        __syncthreads();
        {
            const int t = tid >> 4, s = tid & 15;
            float v = 0.f;
#pragma unroll
            for (int ww = 0; ww < 8; ++ww) v += part[ww * 256 + tid];
            dst[tid] = s <= t ? scale * (v + add) : 0.f;
        }
        __syncthreads();
    }

};

// LN = true: LN+residual on the output layer (the steps of simt_mlp_backward_kernel<D, IO, true>): Delta2
// takes E's place, dP takes dZ's (the dZ tile is overwritten by dP), and the complete adjoint of Delta2
// goes through each row's LN+residual backward to dY (written to the dE tile) and de.
template <bool LN = false>
__global__ void __launch_bounds__(kThreads, 1) mma_mlp_backward_kernel(SimtMlpBackwardParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t s0 = smem_u32(smem);
    const uint32_t sW1 = s0 + kOffW1, sW2 = s0 + kOffW2, sG1 = s0 + kOffG1, sG2 = s0 + kOffG2;
    const uint32_t sHk = s0 + kOffHk, sD1 = s0 + kOffD1, sHq = s0 + kOffHq, sDAq = s0 + kOffDAq;
    const uint32_t sDM = s0 + kOffDM, sDA = s0 + kOffDA;
    const uint32_t sK = s0 + kOffK, sQ = s0 + kOffQ, sDZ = s0 + kOffDZ, sE = s0 + kOffE, sDE = s0 + kOffDE;
    float* P1 = reinterpret_cast<float*>(smem + kOffP1);
    float* P2 = reinterpret_cast<float*>(smem + kOffP2);
    float* L2 = reinterpret_cast<float*>(smem + kOffL2);
    float* L1 = reinterpret_cast<float*>(smem + kOffL1);
    float* part = reinterpret_cast<float*>(smem + kOffPart);
    float* rowp = reinterpret_cast<float*>(smem + kOffRow);
    float* s_eta = reinterpret_cast<float*>(smem + kOffEta);
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, r = l >> 2, c = l & 3;
    const int unit = blockIdx.x;
    const int T = p.T, nb = T / kB;
    const size_t tok = (size_t)unit * T * kD;
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.Q) + tok;
    const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(p.K) + tok;
    const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(p.V) + tok;
    const __nv_bfloat16* dZ = p.dZ ? static_cast<const __nv_bfloat16*>(p.dZ) + tok : nullptr;
    __nv_bfloat16* dQ = static_cast<__nv_bfloat16*>(p.dQ) + tok;
    __nv_bfloat16* dK = static_cast<__nv_bfloat16*>(p.dK) + tok;
    __nv_bfloat16* dV = static_cast<__nv_bfloat16*>(p.dV) + tok;
    float* gW1 = p.dW1 + (size_t)unit * kD * kM;
    float* gc1 = p.dc1 + (size_t)unit * kM;
    float* gW2 = p.dW2 + (size_t)unit * kM * kD;
    float* gc2 = p.dc2 + (size_t)unit * kD;
    const int p0 = 32 * w;                  // this warp's hidden units
    const int jn0 = 16 * (w >> 1), jh = w & 1;   // its features: half jh of the 16-column window jn0
    const int j0 = jn0 + 8 * jh;
    constexpr size_t SZ = 2 * (size_t)kD * kM + kM + kD;
    const Ops ops{smem, part, rowp, tid, w, l, r, c, p0, jn0, jh, j0};
    float* xa0 = reinterpret_cast<float*>(smem + kOffX);
    float* xa1 = xa0 + 512;
    const float inv_d = 1.f / kD;
    // LN: gamma, beta of this lane's two features j0 + 2c + k, and the lane's partial dgamma, dbeta
    float gm[2] = {0.f, 0.f}, bt[2] = {0.f, 0.f}, dgp[2] = {0.f, 0.f}, dbp[2] = {0.f, 0.f};
    if (LN)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            gm[k] = p.gamma[(size_t)(unit % p.H) * kD + j0 + 2 * c + k];
            bt[k] = p.beta[(size_t)(unit % p.H) * kD + j0 + 2 * c + k];
        }

    // the adjoint of the final state: the upstream gradients, or zero
    for (int e = tid; e < kD * kM; e += kThreads) {
        gW1[e] = p.dW1_out ? p.dW1_out[(size_t)unit * kD * kM + e] : 0.f;
        gW2[e] = p.dW2_out ? p.dW2_out[(size_t)unit * kM * kD + e] : 0.f;
    }
    for (int e = tid; e < kM; e += kThreads) gc1[e] = p.dc1_out ? p.dc1_out[(size_t)unit * kM + e] : 0.f;
    for (int e = tid; e < kD; e += kThreads) gc2[e] = p.dc2_out ? p.dc2_out[(size_t)unit * kD + e] : 0.f;
    __syncthreads();

    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * kB;
        const float* S = p.W_states + ((size_t)unit * nb + i) * SZ;
        const float* W1s = S;
        const float* c1s = S + kD * kM;
        const float* W2s = c1s + kM;
        const float* c2s = W2s + kM * kD;
        // ---- bf16 copies: state (W1, W2) and end-state adjoint (GW1, GW2); token tiles; eta
        for (int e = tid; e < kD * kM / 4; e += kThreads) {
            const int a = (4 * e) / kM, pp = (4 * e) % kM;   // W1 / GW1 [a][p]
            const float4 v = reinterpret_cast<const float4*>(W1s)[e];
            const float4 g = reinterpret_cast<const float4*>(gW1)[e];
            *reinterpret_cast<uint2*>(smem + kOffW1 + mm_off(8192, a, pp)) = make_uint2(pk(v.x, v.y), pk(v.z, v.w));
            *reinterpret_cast<uint2*>(smem + kOffG1 + mm_off(8192, a, pp)) = make_uint2(pk(g.x, g.y), pk(g.z, g.w));
            const int q = (4 * e) / kD, j = (4 * e) % kD;   // W2 / GW2 [p][j]
            const float4 v2 = reinterpret_cast<const float4*>(W2s)[e];
            const float4 g2 = reinterpret_cast<const float4*>(gW2)[e];
            *reinterpret_cast<uint2*>(smem + kOffW2 + toff(q, j >> 3) + 2 * (j & 7)) =
                make_uint2(pk(v2.x, v2.y), pk(v2.z, v2.w));
            *reinterpret_cast<uint2*>(smem + kOffG2 + toff(q, j >> 3) + 2 * (j & 7)) =
                make_uint2(pk(g2.x, g2.y), pk(g2.z, g2.w));
        }
        if (tid < 128) {
            const int row = tid >> 3, ch = tid & 7;
            const size_t gi = (size_t)(t0 + row) * kD + 8 * ch;
            *reinterpret_cast<uint4*>(smem + kOffK + toff(row, ch)) = *reinterpret_cast<const uint4*>(K + gi);
            *reinterpret_cast<uint4*>(smem + kOffQ + toff(row, ch)) = *reinterpret_cast<const uint4*>(Q + gi);
            *reinterpret_cast<uint4*>(smem + kOffDZ + toff(row, ch)) =
                dZ ? *reinterpret_cast<const uint4*>(dZ + gi) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (tid < kB) s_eta[tid] = p.eta ? p.eta[(size_t)unit * T + t0 + tid] : p.eta_const;
        __syncthreads();
        const float eta_r[2] = {s_eta[r], s_eta[r + 8]};
        // ---- forward: A = K W1 + c1 and Aq0 = Q W1 + c1 on this warp's hidden units; Hk = GELU(A)
        float A_[4][4], Aq[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) A_[nt][q] = Aq[nt][q] = c1s[ops.hid(nt, q & 1)];
        ops.mm_AB_kn(A_, sK, 0, 4, sW1, 8192);
        ops.mm_AB_kn(Aq, sQ, 0, 4, sW1, 8192);
        {
            float hk[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) hk[nt][q] = gelu_f(A_[nt][q]);
            ops.store_mm(kOffHk, hk);
        }
        // P1 = tril(Q K^T + 1) (warp 0)
        if (w == 0) {
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
                for (int q = 0; q < 4; ++q) {
                    const int t = r + 8 * (q >> 1), s = 8 * nt + 2 * c + (q & 1);
                    P1[t * 16 + s] = s <= t ? x[nt][q] + 1.f : 0.f;
                }
        }
        __syncthreads();   // Hk, P1
        // E = Hk W2 + c2 - V on this warp's features
        float E_[4];
        {
            const float2 cc = *reinterpret_cast<const float2*>(c2s + j0 + 2 * c);
            E_[0] = E_[2] = cc.x;
            E_[1] = E_[3] = cc.y;
            ops.bd_A_X(E_, sHk, sW2);
            if (!LN) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const __nv_bfloat162 v2 =
                        *reinterpret_cast<const __nv_bfloat162*>(V + (size_t)(t0 + r + 8 * h) * kD + j0 + 2 * c);
                    E_[2 * h] -= __bfloat162float(v2.x);
                    E_[2 * h + 1] -= __bfloat162float(v2.y);
                }
            }
        }
        // LN: E_ holds Y = Hk W2 + c2; per row, Xh = LN(Y) (r), E = K + gamma Xh + beta - V,
        // Delta2 = r (G - mean(G) - Xh mean(G Xh)) with G = gamma E, which takes E's place
        float xh[4] = {}, rY[2] = {}, mg[2] = {}, mgx[2] = {};
        auto e_of = [&](int q) {   // E at (row r + 8 (q >> 1), feature j0 + 2c + (q & 1))
            const int row = r + 8 * (q >> 1), j = j0 + 2 * c + (q & 1);
            const float kv = __bfloat162float(
                *reinterpret_cast<const __nv_bfloat16*>(smem + kOffK + toff(row, j >> 3) + 2 * (j & 7)));
            const float vv = __bfloat162float(V[(size_t)(t0 + row) * kD + j]);
            return kv + gm[q & 1] * xh[q] + bt[q & 1] - vv;
        };
        if (LN) {
            float sy[2][2] = {};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                sy[0][q >> 1] += E_[q];
                sy[1][q >> 1] += E_[q] * E_[q];
            }
            ops.rows<2>(sy, xa0);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float mu = sy[0][h] * inv_d;
                rY[h] = rsqrtf(fmaxf(sy[1][h] * inv_d - mu * mu, 0.f) + p.eps);
                xh[2 * h] = (E_[2 * h] - mu) * rY[h];
                xh[2 * h + 1] = (E_[2 * h + 1] - mu) * rY[h];
            }
            float sg[2][2] = {};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float g = gm[q & 1] * e_of(q);
                sg[0][q >> 1] += g;
                sg[1][q >> 1] += g * xh[q];
            }
            ops.rows<2>(sg, xa1);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mg[h] = sg[0][h] * inv_d;
                mgx[h] = sg[1][h] * inv_d;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                E_[q] = rY[q >> 1] * (gm[q & 1] * e_of(q) - mg[q >> 1] - xh[q] * mgx[q >> 1]);
        }
        ops.store_bd(kOffE, E_);
        __syncthreads();   // E (LN: Delta2)
        // M = E W2^T, D1 = M GELU'(A) on this warp's hidden units
        float M_[4][4] = {};
        ops.mm_A_Xt(M_, sE, sW2);
        {
            float d1[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) d1[nt][q] = M_[nt][q] * gelu_grad_f(A_[nt][q]);
            ops.store_mm(kOffD1, d1);
        }
        __syncthreads();   // D1
        // Aq = Aq0 - L1 D1 with L1 = P1 diag(eta); Hq = GELU(Aq)
        {
            uint32_t a[4];
            frag_from_f32(P1, false, s_eta, l, a);
#pragma unroll
            for (int q = 0; q < 4; ++q) a[q] ^= 0x80008000u;   // -L1
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4];
                const int n0 = p0 + 16 * np;
                ldsm4t(bt_addr(sD1 + (n0 >> 6) * kTileBD, n0 & 63, 0, l), b);
                mma(Aq[2 * np], a, b[0], b[1]);
                mma(Aq[2 * np + 1], a, b[2], b[3]);
            }
            float hq[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) hq[nt][q] = gelu_f(Aq[nt][q]);
            ops.store_mm(kOffHq, hq);
        }
        __syncthreads();   // Hq
        // P2 = tril(Hq Hk^T + 1)
        ops.tt_split(sHq, sHk, P2, 1.f, 1.f);
        if (LN) {
            // the outputs' pre-LN P = Hq W2 + c2 - P2 diag(eta) Delta2 on this warp's features, its LN, and
            // dP = the LN adjoint of gamma dZ, written over the dZ tile (dZ itself is read again from global
            // memory for dQ); the outputs' dgamma, dbeta terms
            float pz[4];
            const float2 cc = *reinterpret_cast<const float2*>(c2s + j0 + 2 * c);
            pz[0] = pz[2] = cc.x;
            pz[1] = pz[3] = cc.y;
            ops.bd_A_X(pz, sHq, sW2);
            uint32_t a[4], b[4];
            frag_from_f32(P2, false, s_eta, l, a);
#pragma unroll
            for (int q = 0; q < 4; ++q) a[q] ^= 0x80008000u;
            ldsm4t(bt_addr(sE, jn0, 0, l), b);
            mma(pz, a, jh ? b[2] : b[0], jh ? b[3] : b[1]);
            float sp[2][2] = {};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                sp[0][q >> 1] += pz[q];
                sp[1][q >> 1] += pz[q] * pz[q];
            }
            ops.rows<2>(sp, xa0);
            float ro[2], dz[4], sd[2][2] = {};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float mu = sp[0][h] * inv_d;
                ro[h] = rsqrtf(fmaxf(sp[1][h] * inv_d - mu * mu, 0.f) + p.eps);
                const float2 zz = tile_pair_bf16(smem, kOffDZ, r + 8 * h, j0 + 2 * c);
                dz[2 * h] = zz.x;
                dz[2 * h + 1] = zz.y;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int q = 2 * h + k;
                    pz[q] = (pz[q] - mu) * ro[h];   // Xo
                    const float gd = gm[k] * dz[q];
                    sd[0][h] += gd;
                    sd[1][h] += gd * pz[q];
                    dgp[k] += dz[q] * pz[q];
                    dbp[k] += dz[q];
                }
            }
            ops.rows<2>(sd, xa1);
            float dpv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                dpv[q] = ro[q >> 1] * (gm[q & 1] * dz[q] - sd[0][q >> 1] * inv_d - pz[q] * sd[1][q >> 1] * inv_d);
            ops.store_bd(kOffDZ, dpv);
            __syncthreads();   // dP over the dZ tile
        }
        // ---- backward.  Products with the end-state adjoint (GW1, GW2 copies), dHq = dZ W2^T,
        // dL2 = tril(-dZ E^T)
        float G2[4], dKx[4];
        {
            const float2 gg = *reinterpret_cast<const float2*>(gc2 + j0 + 2 * c);
            G2[0] = G2[2] = gg.x;
            G2[1] = G2[3] = gg.y;
            ops.bd_A_X(G2, sHk, sG2);   // dc2' + Hk dW2'
            float x[4] = {};
            // D1 dW1'^T: B[k=p][n=a] = GW1[a][p]
            ops.bd_A_Yt(x, sD1, sG1);
#pragma unroll
            for (int q = 0; q < 4; ++q) dKx[q] = -eta_r[q >> 1] * x[q];
        }
        float G1[4][4], dHk[4][4], dHq[4][4] = {};
        {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    G1[nt][q] = gc1[ops.hid(nt, q & 1)];
                    dHk[nt][q] = 0.f;
                }
            ops.mm_AB_kn(G1, sK, 0, 4, sG1, 8192);   // dc1' + K dW1'
            ops.mm_A_Xt(dHk, sE, sG2);              // E dW2'^T
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) dHk[nt][q] *= -eta_r[q >> 1];
            ops.mm_A_Xt(dHq, sDZ, sW2);             // dZ W2^T
        }
        if (w == 1) {
            float x[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4], b[4];
                ldsm4(a_addr(sDZ, 0, ks, l), a);
                ldsm4(b_addr(sE, 0, ks, l), b);
                mma(x[0], a, b[0], b[1]);
                mma(x[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int t = r + 8 * (q >> 1), s = 8 * nt + 2 * c + (q & 1);
                    L2[t * 16 + s] = s <= t ? -x[nt][q] : 0.f;
                }
        }
        // deta from the state updates: -(G2 . E) - (G1 . D1) per row
        float det[2];
        {
            float v[2] = {0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q >> 1] -= G2[q] * E_[q];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    v[q >> 1] -= G1[nt][q] * M_[nt][q] * gelu_grad_f(A_[nt][q]);
            ops.row_total(v);   // (barrier: L2 complete too)
            det[0] = v[0];
            det[1] = v[1];
        }
        // + sum over t >= s of dL2[t][s] P2[t][s] (row s of deta)
        {
            float v0 = 0.f, v1 = 0.f;
            for (int t = r; t < 16; ++t) v0 += L2[t * 16 + r] * P2[t * 16 + r];
            for (int t = r + 8; t < 16; ++t) v1 += L2[t * 16 + r + 8] * P2[t * 16 + r + 8];
            det[0] += v0;
            det[1] += v1;
        }
        // dE = -eta (G2 + P2^T dZ) on this warp's features, kept in G2
        {
            uint32_t a[4], b[4];
            frag_from_f32(P2, true, nullptr, l, a);
            float x[4] = {};
            ldsm4t(bt_addr(sDZ, jn0, 0, l), b);
            mma(x, a, jh ? b[2] : b[0], jh ? b[3] : b[1]);
#pragma unroll
            for (int q = 0; q < 4; ++q) G2[q] = -eta_r[q >> 1] * (G2[q] + x[q]);
        }
        // dAq = (dHq + dP2 Hk) GELU'(Aq) and dHk += dP2^T Hq, with dP2 = dL2 diag(eta)
        {
            uint32_t a[4], at[4];
            frag_from_f32(L2, false, s_eta, l, a);
            frag_from_f32(L2, true, nullptr, l, at);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4], bq[4];
                const int n0 = p0 + 16 * np;
                ldsm4t(bt_addr(sHk + (n0 >> 6) * kTileBD, n0 & 63, 0, l), b);
                mma(dHq[2 * np], a, b[0], b[1]);
                mma(dHq[2 * np + 1], a, b[2], b[3]);
                ldsm4t(bt_addr(sHq + (n0 >> 6) * kTileBD, n0 & 63, 0, l), bq);
                float y[2][4] = {};
                mma(y[0], at, bq[0], bq[1]);
                mma(y[1], at, bq[2], bq[3]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    dHk[2 * np][q] += eta_r[q >> 1] * y[0][q];
                    dHk[2 * np + 1][q] += eta_r[q >> 1] * y[1][q];
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) dHq[nt][q] *= gelu_grad_f(Aq[nt][q]);   // dAq
            ops.store_mm(kOffDAq, dHq);
        }
        __syncthreads();   // dAq
        // dQ = dAq W1^T (this warp's features); dL1 = tril(-dAq D1^T); dD1 = -eta G1 - L1^T dAq
        float dQx[4] = {};
        ops.bd_A_Yt(dQx, sDAq, sW1);
        ops.tt_split(sDAq, sD1, L1, 0.f, -1.f);
        {
            uint32_t a[4];
            frag_from_f32(P1, true, nullptr, l, a);   // P1^T; L1^T = (P1 diag(eta))^T = diag(eta) P1^T
            float x[4][4] = {};
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4];
                const int n0 = p0 + 16 * np;
                ldsm4t(bt_addr(sDAq + (n0 >> 6) * kTileBD, n0 & 63, 0, l), b);
                mma(x[2 * np], a, b[0], b[1]);
                mma(x[2 * np + 1], a, b[2], b[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) G1[nt][q] = -eta_r[q >> 1] * (G1[nt][q] + x[nt][q]);   // dD1
        }
        // deta from the layer-1 outputs: sum over t >= s of dL1[t][s] P1[t][s]
        {
            float v0 = 0.f, v1 = 0.f;
            for (int t = r; t < 16; ++t) v0 += L1[t * 16 + r] * P1[t * 16 + r];
            for (int t = r + 8; t < 16; ++t) v1 += L1[t * 16 + r + 8] * P1[t * 16 + r + 8];
            det[0] += v0;
            det[1] += v1;
        }
        // dM = dD1 GELU'(A) -> shared; the first part of dA, dD1 M GELU''(A), in M_
        {
            float dm[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    dm[nt][q] = G1[nt][q] * gelu_grad_f(A_[nt][q]);
                    M_[nt][q] = G1[nt][q] * M_[nt][q] * gelu_grad2_f(A_[nt][q]);
                }
            ops.store_mm(kOffDM, dm);
        }
        __syncthreads();   // dM
        // with dP1 = dL1 diag(eta): dQ += dP1 K;  dK += dP1^T Q;  dE += dM W2
        {
            uint32_t a[4], at[4], b[4];
            frag_from_f32(L1, false, s_eta, l, a);
            frag_from_f32(L1, true, nullptr, l, at);
            ldsm4t(bt_addr(sK, jn0, 0, l), b);
            mma(dQx, a, jh ? b[2] : b[0], jh ? b[3] : b[1]);
            float y[4] = {};
            ldsm4t(bt_addr(sQ, jn0, 0, l), b);
            mma(y, at, jh ? b[2] : b[0], jh ? b[3] : b[1]);
#pragma unroll
            for (int q = 0; q < 4; ++q) dKx[q] += eta_r[q >> 1] * y[q];
            ops.bd_A_X(G2, sDM, sW2);   // dE += dM W2
            float dev_[4];               // the adjoint that reaches K and V (de with LN)
#pragma unroll
            for (int q = 0; q < 4; ++q) dev_[q] = G2[q];
            if (LN) {
                // G2 holds dDelta2: each row's LN+residual backward to de and dY (dY into G2)
                float s3[3][2] = {};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int h = q >> 1;
                    const float u = gm[q & 1] * e_of(q) - mg[h] - xh[q] * mgx[h];
                    const float du = rY[h] * G2[q];
                    s3[0][h] += G2[q] * u;
                    s3[1][h] += du;
                    s3[2][h] += du * xh[q];
                }
                ops.rows<3>(s3, xa0);
                float s2[2][2] = {}, dx[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int h = q >> 1, k = q & 1;
                    const float ev = e_of(q);
                    const float du = rY[h] * G2[q];
                    const float dg = du - s3[1][h] * inv_d - xh[q] * s3[2][h] * inv_d;
                    const float de = gm[k] * dg;
                    dx[q] = -du * mgx[h] - gm[k] * ev * s3[2][h] * inv_d + gm[k] * de;
                    dgp[k] += ev * dg + xh[q] * de;
                    dbp[k] += de;
                    dev_[q] = de;
                    s2[0][h] += dx[q];
                    s2[1][h] += dx[q] * xh[q];
                }
                ops.rows<2>(s2, xa1);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int h = q >> 1;
                    G2[q] = rY[h] * (dx[q] - s2[0][h] * inv_d - xh[q] * s2[1][h] * inv_d) -
                            s3[0][h] * rY[h] * rY[h] * xh[q] * inv_d;   // dY
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    dKx[q] += dev_[q];
                    // dQ also has the output residual's dZ (read again from global memory)
                    dQx[q] += dZ ? __bfloat162float(dZ[(size_t)(t0 + r + 8 * (q >> 1)) * kD + j0 + 2 * c + (q & 1)])
                                 : 0.f;
                }
            }
            ops.store_bd(kOffDE, G2);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                *reinterpret_cast<__nv_bfloat162*>(dV + (size_t)(t0 + r + 8 * h) * kD + j0 + 2 * c) =
                    __floats2bfloat162_rn(-dev_[2 * h], -dev_[2 * h + 1]);
                *reinterpret_cast<__nv_bfloat162*>(dQ + (size_t)(t0 + r + 8 * h) * kD + j0 + 2 * c) =
                    __floats2bfloat162_rn(dQx[2 * h], dQx[2 * h + 1]);
            }
        }
        __syncthreads();   // dE
        // dHk += dE W2^T;  dA = dD1 M GELU''(A) + dHk GELU'(A) -> shared
        {
            ops.mm_A_Xt(dHk, sDE, sW2);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) M_[nt][q] += dHk[nt][q] * gelu_grad_f(A_[nt][q]);
            ops.store_mm(kOffDA, M_);
        }
        __syncthreads();   // dA
        // dK += dA W1^T (this warp's features)
        ops.bd_A_Yt(dKx, sDA, sW1);
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<__nv_bfloat162*>(dK + (size_t)(t0 + r + 8 * h) * kD + j0 + 2 * c) =
                __floats2bfloat162_rn(dKx[2 * h], dKx[2 * h + 1]);
        if (w == 0 && c == 0 && p.deta) {
            p.deta[(size_t)unit * T + t0 + r] = det[0];
            p.deta[(size_t)unit * T + t0 + r + 8] = det[1];
        }
        // ---- this mini-batch's terms of the start-state adjoint (fp32, global)
        // GW1[a][p] += (Q^T dAq + K^T dA)[a][p] on this warp's hidden units (four 16-row blocks of a)
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
            float x[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    x[nt][q] = gW1[(size_t)(16 * mt + r + 8 * (q >> 1)) * kM + ops.hid(nt, q & 1)];
            uint32_t aq[4], ak[4];
            ldsm4t(at_addr(sQ, 16 * mt, l), aq);
            ldsm4t(at_addr(sK, 16 * mt, l), ak);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4], bd[4];
                const int n0 = p0 + 16 * np;
                ldsm4t(bt_addr(sDAq + (n0 >> 6) * kTileBD, n0 & 63, 0, l), b);
                mma(x[2 * np], aq, b[0], b[1]);
                mma(x[2 * np + 1], aq, b[2], b[3]);
                ldsm4t(bt_addr(sDA + (n0 >> 6) * kTileBD, n0 & 63, 0, l), bd);
                mma(x[2 * np], ak, bd[0], bd[1]);
                mma(x[2 * np + 1], ak, bd[2], bd[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<float2*>(gW1 + (size_t)(16 * mt + r + 8 * h) * kM + ops.hid(nt, 0)) =
                        make_float2(x[nt][2 * h], x[nt][2 * h + 1]);
        }
        // GW2[p][j] += (Hq^T dZ + dM^T E + Hk^T dE)[p][j] on this warp's hidden units (two 16-row blocks)
#pragma unroll 1
        for (int mt = 0; mt < 2; ++mt) {
            const int pr = p0 + 16 * mt;
            const uint32_t ch = (pr >> 6) * kTileBD;
            uint32_t ah[4], am[4], ak[4];
            ldsm4t(at_addr(sHq + ch, pr & 63, l), ah);
            ldsm4t(at_addr(sDM + ch, pr & 63, l), am);
            ldsm4t(at_addr(sHk + ch, pr & 63, l), ak);
#pragma unroll 1
            for (int np = 0; np < 4; ++np) {
                float x[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        x[nt][q] = gW2[(size_t)(pr + r + 8 * (q >> 1)) * kD + 16 * np + 8 * nt + 2 * c + (q & 1)];
                uint32_t b[4];
                ldsm4t(bt_addr(sDZ, 16 * np, 0, l), b);
                mma(x[0], ah, b[0], b[1]);
                mma(x[1], ah, b[2], b[3]);
                ldsm4t(bt_addr(sE, 16 * np, 0, l), b);
                mma(x[0], am, b[0], b[1]);
                mma(x[1], am, b[2], b[3]);
                ldsm4t(bt_addr(sDE, 16 * np, 0, l), b);
                mma(x[0], ak, b[0], b[1]);
                mma(x[1], ak, b[2], b[3]);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        *reinterpret_cast<float2*>(gW2 + (size_t)(pr + r + 8 * h) * kD + 16 * np + 8 * nt + 2 * c) =
                            make_float2(x[nt][2 * h], x[nt][2 * h + 1]);
            }
        }
        // dc1 += column sums of dAq + dA (this warp's hidden units); dc2 += of dZ + dE (its features)
        {
            float s1[4][2];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    s1[nt][k] = dHq[nt][k] + dHq[nt][2 + k] + M_[nt][k] + M_[nt][2 + k];
                    s1[nt][k] += __shfl_xor_sync(0xffffffffu, s1[nt][k], 4);
                    s1[nt][k] += __shfl_xor_sync(0xffffffffu, s1[nt][k], 8);
                    s1[nt][k] += __shfl_xor_sync(0xffffffffu, s1[nt][k], 16);
                }
            if (r == 0)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int k = 0; k < 2; ++k) gc1[ops.hid(nt, k)] += s1[nt][k];
            float s2[2];
            const float2 z0 = tile_pair_bf16(smem, kOffDZ, r, j0 + 2 * c);
            const float2 z1 = tile_pair_bf16(smem, kOffDZ, r + 8, j0 + 2 * c);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float zz = k == 0 ? z0.x + z1.x : z0.y + z1.y;
                s2[k] = zz + G2[k] + G2[2 + k];
                s2[k] += __shfl_xor_sync(0xffffffffu, s2[k], 4);
                s2[k] += __shfl_xor_sync(0xffffffffu, s2[k], 8);
                s2[k] += __shfl_xor_sync(0xffffffffu, s2[k], 16);
            }
            if (r == 0) {
                gc2[j0 + 2 * c] += s2[0];
                gc2[j0 + 2 * c + 1] += s2[1];
            }
        }
        __syncthreads();   // every read of this mini-batch's shared data and of the adjoint is done
    }
    if (LN) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            dgp[k] += __shfl_xor_sync(0xffffffffu, dgp[k], 4);
            dgp[k] += __shfl_xor_sync(0xffffffffu, dgp[k], 8);
            dgp[k] += __shfl_xor_sync(0xffffffffu, dgp[k], 16);
            dbp[k] += __shfl_xor_sync(0xffffffffu, dbp[k], 4);
            dbp[k] += __shfl_xor_sync(0xffffffffu, dbp[k], 8);
            dbp[k] += __shfl_xor_sync(0xffffffffu, dbp[k], 16);
        }
        if (r == 0)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                p.dgamma[(size_t)unit * kD + j0 + 2 * c + k] = dgp[k];
                p.dbeta[(size_t)unit * kD + j0 + 2 * c + k] = dbp[k];
            }
    }
}

// The TTT-MLP forward that writes the batch-start states, on mma.sync (bf16, d = 64, b = 16): the dual
// form of section 3.7 per mini-batch, in the layout of the backward above.  The state is not kept in
// registers: mini-batch i reads S_i from its checkpoint W_states[i] (S_0 = the initial state, copied
// there first) and each warp writes its block of S_{i+1} = S_i + (update) to W_states[i + 1], or to the
// final-state outputs after the last mini-batch.
struct MlpFwdStatesParams {
    int H, T;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W1;   // initial state, [H, ...] or [B, H, ...] (per_seq)
    const float* c1;   // or null
    const float* W2;
    const float* c2;   // or null
    int per_seq;
    void* Z;           // or null (state only)
    float* W1_out;
    float* c1_out;     // or null
    float* W2_out;
    float* c2_out;     // or null
    float* W_states;   // [units, T/16, 2 d m + m + d]
    const float* gamma;   // LN+residual on the output layer (the LN instance): [H, 64]
    const float* beta;
    float eps;
};

// LN = true: f(x) = x + gamma LN(GELU(x W1 + c1) W2 + c2) + beta: Delta2 (the LN+residual backward at
// Y = Hk W2 + c2) takes E's place, and Z = Q + gamma LN(P) + beta with P the plain model's output.
template <bool LN = false>
__global__ void __launch_bounds__(kThreads, 1) mma_mlp_forward_states_kernel(MlpFwdStatesParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t s0 = smem_u32(smem);
    const uint32_t sW1 = s0 + kOffW1, sW2 = s0 + kOffW2;
    const uint32_t sHk = s0 + kOffHk, sD1 = s0 + kOffD1, sHq = s0 + kOffHq;
    const uint32_t sK = s0 + kOffK, sQ = s0 + kOffQ, sE = s0 + kOffE, sEE = s0 + kOffDE;
    float* P1 = reinterpret_cast<float*>(smem + kOffP1);
    float* P2 = reinterpret_cast<float*>(smem + kOffP2);
    float* part = reinterpret_cast<float*>(smem + kOffPart);
    float* rowp = reinterpret_cast<float*>(smem + kOffRow);
    float* s_eta = reinterpret_cast<float*>(smem + kOffEta);
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, r = l >> 2, c = l & 3;
    const int unit = blockIdx.x;
    const int T = p.T, nb = T / kB;
    const int pu = p.per_seq ? unit : unit % p.H;
    const size_t tok = (size_t)unit * T * kD;
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.Q) + tok;
    const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(p.K) + tok;
    const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(p.V) + tok;
    __nv_bfloat16* Z = p.Z ? static_cast<__nv_bfloat16*>(p.Z) + tok : nullptr;
    const int p0 = 32 * w;
    const int jn0 = 16 * (w >> 1), jh = w & 1;
    const int j0 = jn0 + 8 * jh;
    constexpr size_t SZ = 2 * (size_t)kD * kM + kM + kD;
    const Ops ops{smem, part, rowp, tid, w, l, r, c, p0, jn0, jh, j0};
    float* states = p.W_states + (size_t)unit * nb * SZ;
    float* xa0 = reinterpret_cast<float*>(smem + kOffX);
    float* xa1 = xa0 + 512;
    const float inv_d = 1.f / kD;
    float gm[2] = {0.f, 0.f}, bt[2] = {0.f, 0.f};
    if (LN)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            gm[k] = p.gamma[(size_t)(unit % p.H) * kD + j0 + 2 * c + k];
            bt[k] = p.beta[(size_t)(unit % p.H) * kD + j0 + 2 * c + k];
        }

    // S_0: the initial state, to the first checkpoint
    if (nb > 0) {
        for (int e = tid; e < kD * kM; e += kThreads) {
            states[e] = p.W1[(size_t)pu * kD * kM + e];
            states[kD * kM + kM + e] = p.W2[(size_t)pu * kM * kD + e];
        }
        for (int e = tid; e < kM; e += kThreads) states[kD * kM + e] = p.c1 ? p.c1[(size_t)pu * kM + e] : 0.f;
        for (int e = tid; e < kD; e += kThreads) states[2 * kD * kM + kM + e] = p.c2 ? p.c2[(size_t)pu * kD + e] : 0.f;
    }
    __syncthreads();
    for (int i = 0; i < nb; ++i) {
        const int t0 = i * kB;
        const float* S = states + (size_t)i * SZ;
        const float* W1s = S;
        const float* c1s = S + kD * kM;
        const float* W2s = c1s + kM;
        const float* c2s = W2s + kM * kD;
        const bool last = i + 1 == nb;
        float* N = last ? nullptr : states + (size_t)(i + 1) * SZ;
        // where S_{i+1} goes: the next checkpoint, or the final-state outputs (c1_out, c2_out may be null)
        float* nW1 = last ? p.W1_out + (size_t)unit * kD * kM : N;
        float* nW2 = last ? p.W2_out + (size_t)unit * kM * kD : N + kD * kM + kM;
        float* nc1 = !last ? N + kD * kM : p.c1_out ? p.c1_out + (size_t)unit * kM : nullptr;
        float* nc2 = !last ? N + 2 * kD * kM + kM : p.c2_out ? p.c2_out + (size_t)unit * kD : nullptr;
        // ---- bf16 copies of the state, token tiles, eta
        for (int e = tid; e < kD * kM / 4; e += kThreads) {
            const int a = (4 * e) / kM, pp = (4 * e) % kM;
            const float4 v = reinterpret_cast<const float4*>(W1s)[e];
            *reinterpret_cast<uint2*>(smem + kOffW1 + mm_off(8192, a, pp)) = make_uint2(pk(v.x, v.y), pk(v.z, v.w));
            const int q = (4 * e) / kD, j = (4 * e) % kD;
            const float4 v2 = reinterpret_cast<const float4*>(W2s)[e];
            *reinterpret_cast<uint2*>(smem + kOffW2 + toff(q, j >> 3) + 2 * (j & 7)) =
                make_uint2(pk(v2.x, v2.y), pk(v2.z, v2.w));
        }
        if (tid < 128) {
            const int row = tid >> 3, ch = tid & 7;
            const size_t gi = (size_t)(t0 + row) * kD + 8 * ch;
            *reinterpret_cast<uint4*>(smem + kOffK + toff(row, ch)) = *reinterpret_cast<const uint4*>(K + gi);
            *reinterpret_cast<uint4*>(smem + kOffQ + toff(row, ch)) = *reinterpret_cast<const uint4*>(Q + gi);
        }
        if (tid < kB) s_eta[tid] = p.eta ? p.eta[(size_t)unit * T + t0 + tid] : p.eta_const;
        __syncthreads();
        const float eta_r[2] = {s_eta[r], s_eta[r + 8]};
        // ---- A = K W1 + c1, Aq0 = Q W1 + c1 on this warp's hidden units; Hk = GELU(A); P1 (warp 0)
        float A_[4][4], Aq[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) A_[nt][q] = Aq[nt][q] = c1s[ops.hid(nt, q & 1)];
        ops.mm_AB_kn(A_, sK, 0, 4, sW1, 8192);
        ops.mm_AB_kn(Aq, sQ, 0, 4, sW1, 8192);
        {
            float hk[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) hk[nt][q] = gelu_f(A_[nt][q]);
            ops.store_mm(kOffHk, hk);
        }
        if (w == 0) {
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
                for (int q = 0; q < 4; ++q) {
                    const int t = r + 8 * (q >> 1), s_ = 8 * nt + 2 * c + (q & 1);
                    P1[t * 16 + s_] = s_ <= t ? x[nt][q] + 1.f : 0.f;
                }
        }
        __syncthreads();   // Hk, P1
        // ---- E = Hk W2 + c2 - V on this warp's features -> E and diag(eta) E (bf16); c2 update
        float E_[4];
        {
            const float2 cc = *reinterpret_cast<const float2*>(c2s + j0 + 2 * c);
            E_[0] = E_[2] = cc.x;
            E_[1] = E_[3] = cc.y;
            ops.bd_A_X(E_, sHk, sW2);
            float vv[4], kk[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __nv_bfloat162 v2 =
                    *reinterpret_cast<const __nv_bfloat162*>(V + (size_t)(t0 + r + 8 * h) * kD + j0 + 2 * c);
                vv[2 * h] = __bfloat162float(v2.x);
                vv[2 * h + 1] = __bfloat162float(v2.y);
                const float2 k2 = tile_pair_bf16(smem, kOffK, r + 8 * h, j0 + 2 * c);
                kk[2 * h] = k2.x;
                kk[2 * h + 1] = k2.y;
            }
            if (!LN) {
#pragma unroll
                for (int q = 0; q < 4; ++q) E_[q] -= vv[q];
            } else {
                // E_ holds Y: per row Xh = LN(Y), E = K + gamma Xh + beta - V, Delta2 = r (G - mean(G) - Xh
                // mean(G Xh)), G = gamma E, which takes E's place
                float sy[2][2] = {};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sy[0][q >> 1] += E_[q];
                    sy[1][q >> 1] += E_[q] * E_[q];
                }
                ops.rows<2>(sy, xa0);
                float rY[2], xh[4], g[4], sg[2][2] = {};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float mu = sy[0][h] * inv_d;
                    rY[h] = rsqrtf(fmaxf(sy[1][h] * inv_d - mu * mu, 0.f) + p.eps);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int h = q >> 1;
                    xh[q] = (E_[q] - sy[0][h] * inv_d) * rY[h];
                    g[q] = gm[q & 1] * (kk[q] + gm[q & 1] * xh[q] + bt[q & 1] - vv[q]);
                    sg[0][h] += g[q];
                    sg[1][h] += g[q] * xh[q];
                }
                ops.rows<2>(sg, xa1);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int h = q >> 1;
                    E_[q] = rY[h] * (g[q] - sg[0][h] * inv_d - xh[q] * sg[1][h] * inv_d);
                }
            }
            ops.store_bd(kOffE, E_);
            float ee[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) ee[q] = eta_r[q >> 1] * E_[q];
            ops.store_bd(kOffDE, ee);
            float s2[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                s2[k] = ee[k] + ee[2 + k];
                s2[k] += __shfl_xor_sync(0xffffffffu, s2[k], 4);
                s2[k] += __shfl_xor_sync(0xffffffffu, s2[k], 8);
                s2[k] += __shfl_xor_sync(0xffffffffu, s2[k], 16);
            }
            if (r == 0 && nc2) {
                nc2[j0 + 2 * c] = c2s[j0 + 2 * c] - s2[0];
                nc2[j0 + 2 * c + 1] = c2s[j0 + 2 * c + 1] - s2[1];
            }
        }
        __syncthreads();   // E, diag(eta) E
        // ---- M = E W2^T, D1 = M GELU'(A) -> diag(eta) D1 (bf16); c1 update
        {
            float M_[4][4] = {};
            ops.mm_A_Xt(M_, sE, sW2);
            float s1[4][2];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) M_[nt][q] = eta_r[q >> 1] * M_[nt][q] * gelu_grad_f(A_[nt][q]);
            ops.store_mm(kOffD1, M_);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    s1[nt][k] = M_[nt][k] + M_[nt][2 + k];
                    s1[nt][k] += __shfl_xor_sync(0xffffffffu, s1[nt][k], 4);
                    s1[nt][k] += __shfl_xor_sync(0xffffffffu, s1[nt][k], 8);
                    s1[nt][k] += __shfl_xor_sync(0xffffffffu, s1[nt][k], 16);
                }
            if (r == 0 && nc1)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int k = 0; k < 2; ++k) nc1[ops.hid(nt, k)] = c1s[ops.hid(nt, k)] - s1[nt][k];
        }
        __syncthreads();   // diag(eta) D1
        // ---- Aq = Aq0 - P1 (diag(eta) D1); Hq = GELU(Aq)
        {
            uint32_t a[4];
            frag_from_f32(P1, false, nullptr, l, a);
#pragma unroll
            for (int q = 0; q < 4; ++q) a[q] ^= 0x80008000u;
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4];
                const int n0 = p0 + 16 * np;
                ldsm4t(bt_addr(sD1 + (n0 >> 6) * kTileBD, n0 & 63, 0, l), b);
                mma(Aq[2 * np], a, b[0], b[1]);
                mma(Aq[2 * np + 1], a, b[2], b[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) Aq[nt][q] = gelu_f(Aq[nt][q]);
            ops.store_mm(kOffHq, Aq);
        }
        __syncthreads();   // Hq
        // ---- P2 = tril(Hq Hk^T + 1);  Z = Hq W2 + c2 - P2 (diag(eta) E) on this warp's features
        ops.tt_split(sHq, sHk, P2, 1.f, 1.f);
        if (Z) {
            float z[4];
            const float2 cc = *reinterpret_cast<const float2*>(c2s + j0 + 2 * c);
            z[0] = z[2] = cc.x;
            z[1] = z[3] = cc.y;
            ops.bd_A_X(z, sHq, sW2);
            uint32_t a[4], b[4];
            frag_from_f32(P2, false, nullptr, l, a);
#pragma unroll
            for (int q = 0; q < 4; ++q) a[q] ^= 0x80008000u;
            ldsm4t(bt_addr(sEE, jn0, 0, l), b);
            mma(z, a, jh ? b[2] : b[0], jh ? b[3] : b[1]);
            if (LN) {
                // Z = Q + gamma LN(P) + beta
                float sz[2][2] = {};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sz[0][q >> 1] += z[q];
                    sz[1][q >> 1] += z[q] * z[q];
                }
                ops.rows<2>(sz, xa0);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float mu = sz[0][h] * inv_d;
                    const float ro = rsqrtf(fmaxf(sz[1][h] * inv_d - mu * mu, 0.f) + p.eps);
                    const float2 qv = tile_pair_bf16(smem, kOffQ, r + 8 * h, j0 + 2 * c);
                    z[2 * h] = qv.x + gm[0] * (z[2 * h] - mu) * ro + bt[0];
                    z[2 * h + 1] = qv.y + gm[1] * (z[2 * h + 1] - mu) * ro + bt[1];
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<__nv_bfloat162*>(Z + (size_t)(t0 + r + 8 * h) * kD + j0 + 2 * c) =
                    __floats2bfloat162_rn(z[2 * h], z[2 * h + 1]);
        }
        // ---- S_{i+1}: W1 - K^T diag(eta) D1 and W2 - Hk^T diag(eta) E, this warp's blocks
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
            float x[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    x[nt][q] = W1s[(size_t)(16 * mt + r + 8 * (q >> 1)) * kM + ops.hid(nt, q & 1)];
            uint32_t ak[4];
            ldsm4t(at_addr(sK, 16 * mt, l), ak);
#pragma unroll
            for (int q = 0; q < 4; ++q) ak[q] ^= 0x80008000u;
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b[4];
                const int n0 = p0 + 16 * np;
                ldsm4t(bt_addr(sD1 + (n0 >> 6) * kTileBD, n0 & 63, 0, l), b);
                mma(x[2 * np], ak, b[0], b[1]);
                mma(x[2 * np + 1], ak, b[2], b[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    *reinterpret_cast<float2*>(nW1 + (size_t)(16 * mt + r + 8 * h) * kM + ops.hid(nt, 0)) =
                        make_float2(x[nt][2 * h], x[nt][2 * h + 1]);
        }
#pragma unroll 1
        for (int mt = 0; mt < 2; ++mt) {
            const int pr = p0 + 16 * mt;
            uint32_t ak[4];
            ldsm4t(at_addr(sHk + (pr >> 6) * kTileBD, pr & 63, l), ak);
#pragma unroll
            for (int q = 0; q < 4; ++q) ak[q] ^= 0x80008000u;
#pragma unroll 1
            for (int np = 0; np < 4; ++np) {
                float x[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        x[nt][q] = W2s[(size_t)(pr + r + 8 * (q >> 1)) * kD + 16 * np + 8 * nt + 2 * c + (q & 1)];
                uint32_t b[4];
                ldsm4t(bt_addr(sEE, 16 * np, 0, l), b);
                mma(x[0], ak, b[0], b[1]);
                mma(x[1], ak, b[2], b[3]);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        *reinterpret_cast<float2*>(nW2 + (size_t)(pr + r + 8 * h) * kD + 16 * np + 8 * nt + 2 * c) =
                            make_float2(x[nt][2 * h], x[nt][2 * h + 1]);
            }
        }
        __syncthreads();   // S_{i+1} written; every read of this mini-batch's shared data is done
    }
    if (nb == 0) {
        // no mini-batch: the final state is the initial one
        for (int e = tid; e < kD * kM; e += kThreads) {
            p.W1_out[(size_t)unit * kD * kM + e] = p.W1[(size_t)pu * kD * kM + e];
            p.W2_out[(size_t)unit * kM * kD + e] = p.W2[(size_t)pu * kM * kD + e];
        }
        if (p.c1_out)
            for (int e = tid; e < kM; e += kThreads) p.c1_out[(size_t)unit * kM + e] = p.c1 ? p.c1[(size_t)pu * kM + e] : 0.f;
        if (p.c2_out)
            for (int e = tid; e < kD; e += kThreads) p.c2_out[(size_t)unit * kD + e] = p.c2 ? p.c2[(size_t)pu * kD + e] : 0.f;
    }
}

}  // namespace mmb
}  // namespace ttt
