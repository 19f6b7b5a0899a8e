// Tensor-core (tcgen05) persistent kernel of the TTT-Linear prefill, plain
// and LN+residual inner models, d = 64, mini-batch b = 16, bf16 Q/K/V/Z,
// fp32 state.
//
// Method (paper digest "论文速览 | TTT", section 3.6, half-loss convention):
// per (sequence, head) unit and mini-batch of 16 tokens with batch-start
// state W0,
//     E  = K W0 - V                                  (key-side residual)
//     Z  = Q W0 - (tril(Q K^T) * eta_s) E            (outputs)
//     W  = W0 - K^T diag(eta) E                      (end-of-batch state)
// and for f(x) = x + LN(x W + c) (section 4.4) E is replaced by the LN
// backward Delta, the bias enters the causal matrix as tril(Q K^T + 1), and
// Z = Q + LN(Q W0 + c - (tril(Q K^T + 1) * eta_s) Delta).
//
// Mapping onto sm_100a.  b = 16 is below the smallest tcgen05 M (64), so the
// contractions are computed transposed with the head dim d = 64 in M:
//     MMA1   [E^T | Zq^T] (64 x 32) = W0^T (64 x 64) . [K^T | Q^T] (64 x 32)
//     MMA2   W^T (64 x 64) += A^T (64 x 16) . K (16 x 64)   with A = -eta * E
//     MMA3   Zq^T (64 x 16) += A^T (64 x 16) . tril(Q K^T)^T (16 x 16)
//     (LN)   Zq^T += A^T . tril(ones)^T                      (the "+1" term)
// The fp32 state W^T stays in tensor memory for the whole sequence and is
// updated in place by MMA2; each mini-batch the epilogue warps read it back,
// round it to bf16 and write it to shared memory as MMA1's A operand.  The
// K tile loaded by TMA serves as the K-major B operand of MMA1 and as the
// MN-major B operand of MMA2 (no transposed copy).
//
// Each CTA owns two units ("pair") that share every instruction: their
// accumulators sit at different TMEM columns and the .16x32bx2 TMEM loads
// give threads 0-15 of a warp one unit and threads 16-31 the other.
//
// Warp roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// computes S = tril(Q K^T) with mma.sync (16x16x64, below tcgen05's shape
// range) into the B operand of MMA3, warps 4-7 are the epilogue (TMEM <->
// registers, the residual, LN statistics and backward, eta scaling, the Z
// store and the bf16 copy of W).
//
// Every wait is bounded; on expiry the kernel records kStatusTimeout, stops
// issuing new asynchronous work, drains what it issued and returns.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace ttt {
namespace ltc {

constexpr int kD = 64;          // head dim
constexpr int kTok = 16;        // tokens per mini-batch
constexpr int kStages = 4;      // input pipeline depth
constexpr int kThreads = 256;

// stage layout (bytes, from a 1024-aligned stage base)
constexpr int kTile = kTok * kD * 2;                 // 2048: one 16 x 64 bf16 tile
constexpr int kOffKQ0 = 0;                           // unit 0: K tile then Q tile
constexpr int kOffKQ1 = 2 * kTile;                   // unit 1
constexpr int kOffV0 = 4 * kTile;
constexpr int kOffV1 = 5 * kTile;
constexpr int kOffS0 = 6 * kTile;                    // 512 B each
constexpr int kOffS1 = kOffS0 + 512;
constexpr int kOffEta0 = kOffS1 + 512;               // 64 B each
constexpr int kOffEta1 = kOffEta0 + 64;
constexpr int kStageBytes = 14336;                   // 14 KB, multiple of 1024

constexpr int kOffStages = 0;
constexpr int kOffA1 = kStages * kStageBytes;        // 2 x 8 KB bf16 W^T (K-major, 128B swizzle)
constexpr int kOffAt = kOffA1 + 2 * 8192;            // 2 x 2 KB bf16 A^T (K-major, no swizzle)
constexpr int kOffOnes = kOffAt + 2 * 2048;          // 512 B tril(ones) (LN)
constexpr int kOffZst = kOffOnes + 1024;             // 2 buffers x 2 units x 2 KB
constexpr int kOffRed = kOffZst + 2 * 2 * kTile;     // 2 x [4 warps][2 units][16] float2
constexpr int kOffBar = kOffRed + 2 * 4 * 2 * 16 * 8;
constexpr int kNumBars = 3 * kStages + 6;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;     // + alignment slack

// TMEM columns
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColW = 0;      // unit 0 W^T [0,64), unit 1 [64,128)
constexpr uint32_t kColE = 128;    // unit 0 [128,144) E^T, [144,160) Zq^T; unit 1 at +32
constexpr uint32_t kColZ = 144;

struct Params {
    int U, H, T;
    int nsteps;
    const float* eta;
    float eta_const;
    const float* W0;
    long long W0_bstride;
    const float* c0;
    long long c0_bstride;
    const float* gamma;
    const float* beta;
    float eps;
    float* W_out;
    float* c_out;
    int* status;
    unsigned long long wait_ns;
    unsigned flags;
};

// K-major, no-swizzle canonical layout of a (rows x 16) bf16 operand:
// 8-row x 16-byte core matrices, K-chunk stride 128 B, row-group stride 256 B.
__device__ __forceinline__ uint32_t nosw_off(int row, int k) {
    return (row >> 3) * 256 + (row & 7) * 16 + (k >> 3) * 128 + (k & 7) * 2;
}
// byte offset of element (row, col) in a 128B-swizzled tile of 128-byte rows
__device__ __forceinline__ uint32_t sw128_off(int row, int col) {
    return row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + (col & 7) * 2;
}

__device__ __forceinline__ float ld_bf16(const uint8_t* base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}

// ldmatrix x4 (four 8x8 b16 matrices)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// S = tril(Q K^T) for one unit, written as the K-major (no swizzle) B operand
// of MMA3: element (n = t, k = s) holds q_t . k_s for s <= t, else 0.
__device__ __forceinline__ void compute_S(const uint8_t* kq, uint8_t* sdst, int lane) {
    const uint32_t kbase = smem_u32(kq), qbase = kbase + kTile;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        {   // A = Q rows 0..15, k chunk 2ks + (lane/16)
            const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
            const int ch = 2 * ks + (lane >> 4);
            ldsm_x4(qbase + row * 128 + ((ch ^ (row & 7)) << 4), a0, a1, a2, a3);
        }
        {   // B = K rows: matrices (keys 0-7, chunk 2ks), (keys 0-7, 2ks+1), (keys 8-15, 2ks), (keys 8-15, 2ks+1)
            const int mi = lane >> 3;
            const int row = 8 * (mi >> 1) + (lane & 7);
            const int ch = 2 * ks + (mi & 1);
            ldsm_x4(kbase + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
        }
        mma_16816(acc[0], a0, a1, a2, a3, b0, b1);
        mma_16816(acc[1], a0, a1, a2, a3, b2, b3);
    }
    const int r0 = lane >> 2, c0 = 2 * (lane & 3);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int t = r0 + 8 * hh;
            const int s = 8 * nt + c0;
            const float x0 = (s <= t) ? acc[nt][2 * hh + 0] : 0.f;
            const float x1 = (s + 1 <= t) ? acc[nt][2 * hh + 1] : 0.f;
            *reinterpret_cast<uint32_t*>(sdst + nosw_off(t, s)) = pack_bf16x2(x0, x1);
        }
    }
}

// Butterfly reduce-scatter of two 16-vectors over the 16 lanes of a
// half-warp: afterwards a[0], b[0] hold the half-warp sums for token
// t = lane & 15.
__device__ __forceinline__ void halfwarp_reduce2(float* a, float* b, int lane) {
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1) {
        const bool up = (lane & w) != 0;
#pragma unroll
        for (int k = 0; k < w; ++k) {
            const float sa = up ? a[k] : a[k + w], ka = up ? a[k + w] : a[k];
            const float sb = up ? b[k] : b[k + w], kb = up ? b[k + w] : b[k];
            a[k] = ka + __shfl_xor_sync(0xffffffffu, sa, w);
            b[k] = kb + __shfl_xor_sync(0xffffffffu, sb, w);
        }
    }
}

// Sums over the 64 features (16 lanes x 4 epilogue warps) of two per-token
// quantities; every thread of the unit half gets all 16 token sums.
__device__ __forceinline__ void feature_sum2(float* a, float* b, float2* red, int ew, int lane) {
    halfwarp_reduce2(a, b, lane);
    const int u = lane >> 4, t = lane & 15;
    red[(ew * 2 + u) * 16 + t] = make_float2(a[0], b[0]);
    named_bar_sync(2, 128);
    float sa = 0.f, sb = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const float2 v = red[(w * 2 + u) * 16 + t];
        sa += v.x;
        sb += v.y;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        a[k] = __shfl_sync(0xffffffffu, sa, (lane & 16) | k);
        b[k] = __shfl_sync(0xffffffffu, sb, (lane & 16) | k);
    }
}

template <bool LN>
__global__ void __launch_bounds__(kThreads, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmZ, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;                    // [kStages] TMA landed
    uint64_t* empty = bars + kStages;         // [kStages] stage free (MMA commit + epilogue)
    uint64_t* sready = bars + 2 * kStages;    // [kStages] S tile written
    uint64_t* a1_ready = bars + 3 * kStages;  // bf16 W^T written
    uint64_t* a2_ready = a1_ready + 1;        // A^T written
    uint64_t* d1_full = a1_ready + 2;         // MMA1 done
    uint64_t* d2_full = a1_ready + 3;         // MMA2/3 done
    uint64_t* drain = a1_ready + 4;           // final MMA drain
    uint64_t* stall = a1_ready + 5;           // never arrived on (test hook)
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit0 = 2 * blockIdx.x;
    const bool has1 = unit0 + 1 < p.U;
    const int unit1 = has1 ? unit0 + 1 : unit0;
    const int nsteps = p.nsteps;
    const uint64_t lim = p.wait_ns;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 2);
            mbar_init(&sready[s], 1);
        }
        mbar_init(a1_ready, 1);
        mbar_init(a2_ready, 1);
        mbar_init(d1_full, 1);
        mbar_init(d2_full, 1);
        mbar_init(drain, 1);
        mbar_init(stall, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (LN) {   // constant tril(ones) operand (n = t, k = s): 1 for s <= t
        for (int e = tid; e < 256; e += kThreads) {
            const int t = e >> 4, s = e & 15;
            *reinterpret_cast<__nv_bfloat16*>(smem + kOffOnes + nosw_off(t, s)) =
                __float2bfloat16_rn(s <= t ? 1.f : 0.f);
        }
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;

    auto fail = [&]() {
        *s_abort = 1;
        atomicOr(p.status, kStatusTimeout);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int issued_last = -1;
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            const uint32_t bytes = 6 * kTile + (p.eta ? 128 : 0);
            for (int i = 0; i < nsteps; ++i) {
                const int s = i % kStages;
                if (i >= kStages && !wait_bounded(&empty[s], ((i / kStages) - 1) & 1, lim, s_abort)) {
                    fail();
                    break;
                }
                if (*s_abort) break;
                uint8_t* st = smem + kOffStages + s * kStageBytes;
                mbar_arrive_expect_tx(&full[s], bytes);
                const int y0 = unit0 * p.T + i * kTok, y1 = unit1 * p.T + i * kTok;
                tma_load_2d(st + kOffKQ0, &tmK, 0, y0, &full[s]);
                tma_load_2d(st + kOffKQ0 + kTile, &tmQ, 0, y0, &full[s]);
                tma_load_2d(st + kOffKQ1, &tmK, 0, y1, &full[s]);
                tma_load_2d(st + kOffKQ1 + kTile, &tmQ, 0, y1, &full[s]);
                tma_load_2d(st + kOffV0, &tmV, 0, y0, &full[s]);
                tma_load_2d(st + kOffV1, &tmV, 0, y1, &full[s]);
                if (p.eta) {
                    bulk_load(st + kOffEta0, p.eta + (size_t)y0, 64, &full[s]);
                    bulk_load(st + kOffEta1, p.eta + (size_t)y1, 64, &full[s]);
                }
                issued_last = i;
            }
            // drain: every issued load must land before the CTA exits (these
            // waits ignore the abort flag; a TMA load always completes)
            for (int i = issued_last - kStages + 1; i <= issued_last; ++i) {
                if (i < 0) continue;
                if (!wait_bounded(&full[i % kStages], (i / kStages) & 1, lim, nullptr)) fail();
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t id1 = make_idesc_bf16(64, 32, 0, 0);
            const uint32_t id2 = make_idesc_bf16(64, 64, 0, 1);
            const uint32_t id3 = make_idesc_bf16(64, 16, 0, 0);
            const uint32_t a1 = smem_u32(smem + kOffA1), at = smem_u32(smem + kOffAt);
            const uint32_t ones = smem_u32(smem + kOffOnes);
            bool ok = true;
            if (p.flags & TTT_FLAG_TEST_STALL) {
                // test hook: wait on a barrier nothing arrives on
                if (!wait_bounded(stall, 0, lim, s_abort)) fail();
                ok = false;
            }
            for (int i = 0; ok && i < nsteps; ++i) {
                const int s = i % kStages;
                const uint32_t par = (i / kStages) & 1;
                const uint32_t st = smem_u32(smem + kOffStages + s * kStageBytes);
                if (!wait_bounded(a1_ready, i & 1, lim, s_abort) || !wait_bounded(&full[s], par, lim, s_abort)) {
                    fail();
                    break;
                }
                tc_fence_after();
                for (int u = 0; u < 2; ++u) {
                    const uint32_t kq = st + (u ? kOffKQ1 : kOffKQ0);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t ad = make_sdesc(a1 + u * 8192 + 32 * ks, 16, 1024, kSwizzle128B);
                        const uint64_t bd = make_sdesc(kq + 32 * ks, 16, 1024, kSwizzle128B);
                        umma_bf16(tbase + kColE + 32 * u, ad, bd, id1, ks > 0);
                    }
                }
                umma_commit(d1_full);
                if (!wait_bounded(a2_ready, i & 1, lim, s_abort) || !wait_bounded(&sready[s], par, lim, s_abort)) {
                    fail();
                    break;
                }
                tc_fence_after();
                for (int u = 0; u < 2; ++u) {
                    const uint32_t kq = st + (u ? kOffKQ1 : kOffKQ0);
                    const uint64_t ad = make_sdesc(at + u * 2048, 128, 256, kSwizzleNone);
                    const uint64_t bk = make_sdesc(kq, 1024, 1024, kSwizzle128B);
                    umma_bf16(tbase + kColW + 64 * u, ad, bk, id2, 1);
                    const uint64_t bs = make_sdesc(st + (u ? kOffS1 : kOffS0), 128, 256, kSwizzleNone);
                    umma_bf16(tbase + kColZ + 32 * u, ad, bs, id3, 1);
                    if (LN) umma_bf16(tbase + kColZ + 32 * u, ad, make_sdesc(ones, 128, 256, kSwizzleNone), id3, 1);
                }
                umma_commit(d2_full);
                umma_commit(&empty[s]);
            }
            // drain every MMA issued so far before TMEM is released
            umma_commit(drain);
            if (!wait_bounded(drain, 0, lim, nullptr)) fail();
        }
    } else if (warp == 2) {
        // --------------------------------------------------------- S = QK^T
        for (int i = 0; i < nsteps; ++i) {
            const int s = i % kStages;
            if (!wait_bounded(&full[s], (i / kStages) & 1, lim, s_abort)) {
                if (lane == 0) fail();
                break;
            }
            uint8_t* st = smem + kOffStages + s * kStageBytes;
            compute_S(st + kOffKQ0, st + kOffS0, lane);
            compute_S(st + kOffKQ1, st + kOffS1, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sready[s]);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 4, u = lane >> 4, r16 = lane & 15;
        const int j = 16 * ew + r16;
        const int unit = u ? unit1 : unit0;
        const bool store_unit = (u == 0) || has1;
        const int n = unit / p.H, h = unit % p.H;
        const uint32_t tl = tbase + ((uint32_t)(32 * ew) << 16);
        uint8_t* a1row = smem + kOffA1 + u * 8192;
        uint8_t* atu = smem + kOffAt + u * 2048;
        float2* red0 = reinterpret_cast<float2*>(smem + kOffRed);
        float2* red1 = red0 + 4 * 2 * 16;
        const bool leader = (ew == 0 && lane == 0);
        float gam = 0.f, bet = 0.f, cj = 0.f;
        if (LN) {
            gam = p.gamma[(size_t)h * kD + j];
            bet = p.beta[(size_t)h * kD + j];
            cj = p.c0 ? p.c0[(size_t)n * p.c0_bstride + (size_t)h * kD + j] : 0.f;
        }
        // initial state: column j of W0 -> TMEM (fp32) and bf16 A operand
        uint32_t w[64];   // fp32 bits of column j of W (row j of W^T)
        {
            const float* W0u = p.W0 + (size_t)n * p.W0_bstride + (size_t)h * kD * kD;
#pragma unroll
            for (int i = 0; i < 64; ++i) w[i] = __float_as_uint(W0u[i * kD + j]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_st_16x32bx2_x16<64>(tl + kColW + 16 * c, w + 16 * c);
            tmem_wait_st();
        }
        auto write_a1 = [&]() {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(w[8 * c + 0]), __uint_as_float(w[8 * c + 1]));
                v.y = pack_bf16x2(__uint_as_float(w[8 * c + 2]), __uint_as_float(w[8 * c + 3]));
                v.z = pack_bf16x2(__uint_as_float(w[8 * c + 4]), __uint_as_float(w[8 * c + 5]));
                v.w = pack_bf16x2(__uint_as_float(w[8 * c + 6]), __uint_as_float(w[8 * c + 7]));
                *reinterpret_cast<uint4*>(a1row + (j >> 3) * 1024 + (j & 7) * 128 + ((c ^ (j & 7)) << 4)) = v;
            }
        };
        write_a1();
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(1, 128);
        if (leader) mbar_arrive(a1_ready);

        bool dead = false;   // set when a wait expired: run the loop without waiting
        for (int i = 0; i < nsteps; ++i) {
            const int s = i % kStages;
            const uint8_t* st = smem + kOffStages + s * kStageBytes;
            const uint8_t* ktile = st + (u ? kOffKQ1 : kOffKQ0);
            const uint8_t* qtile = ktile + kTile;
            const uint8_t* vtile = st + (u ? kOffV1 : kOffV0);
            const float* etas = reinterpret_cast<const float*>(st + (u ? kOffEta1 : kOffEta0));
            if (!dead && (!wait_bounded(&full[s], (i / kStages) & 1, lim, s_abort) ||
                          !wait_bounded(d1_full, i & 1, lim, s_abort))) {
                dead = true;
                fail();
            }
            tc_fence_after();
            float x[16];
            {
                uint32_t xr[16];
                tmem_ld_16x32bx2_x16<32>(tl + kColE, xr);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 16; ++t) x[t] = __uint_as_float(xr[t]);
            }
            float et[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) et[t] = p.eta ? etas[t] : p.eta_const;
            float av[16];   // A^T row j: -eta_t * delta_t
            float c_old = cj;
            if (!LN) {
#pragma unroll
                for (int t = 0; t < 16; ++t) av[t] = -et[t] * (x[t] - ld_bf16(vtile, sw128_off(t, j)));
            } else {
                float y[16], y2[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    y[t] = x[t] + cj;
                    x[t] = y[t];
                    y2[t] = y[t] * y[t];
                }
                feature_sum2(y, y2, red0, ew, lane);
                float r[16], xh[16], g[16], gx[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float mu = y[t] * (1.f / kD);
                    const float var = fmaxf(y2[t] * (1.f / kD) - mu * mu, 0.f);
                    r[t] = rsqrtf(var + p.eps);
                    xh[t] = (x[t] - mu) * r[t];
                    const float e = ld_bf16(ktile, sw128_off(t, j)) + gam * xh[t] + bet -
                                    ld_bf16(vtile, sw128_off(t, j));
                    g[t] = gam * e;
                    gx[t] = g[t] * xh[t];
                }
                float gs[16], gxs[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    gs[t] = g[t];
                    gxs[t] = gx[t];
                }
                feature_sum2(gs, gxs, red1, ew, lane);
                float csum = 0.f;
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float delta = r[t] * (g[t] - gs[t] * (1.f / kD) - xh[t] * gxs[t] * (1.f / kD));
                    av[t] = -et[t] * delta;
                    csum += av[t];
                }
                cj += csum;
            }
            {   // A^T row j, K-major no-swizzle: two 16-byte chunks
                uint4 v0, v1;
                v0.x = pack_bf16x2(av[0], av[1]);
                v0.y = pack_bf16x2(av[2], av[3]);
                v0.z = pack_bf16x2(av[4], av[5]);
                v0.w = pack_bf16x2(av[6], av[7]);
                v1.x = pack_bf16x2(av[8], av[9]);
                v1.y = pack_bf16x2(av[10], av[11]);
                v1.z = pack_bf16x2(av[12], av[13]);
                v1.w = pack_bf16x2(av[14], av[15]);
                *reinterpret_cast<uint4*>(atu + nosw_off(j, 0)) = v0;
                *reinterpret_cast<uint4*>(atu + nosw_off(j, 8)) = v1;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (leader) bulk_wait_read<1>();   // Z staging buffer i%2 is free again
            named_bar_sync(1, 128);
            if (leader) mbar_arrive(a2_ready);

            if (!dead && !wait_bounded(d2_full, i & 1, lim, s_abort)) {
                dead = true;
                fail();
            }
            tc_fence_after();
            float z[16];
            {
                uint32_t zr[16];
                tmem_ld_16x32bx2_x16<32>(tl + kColZ, zr);
                tmem_ld_16x32bx2_x32<64>(tl + kColW, w);
                tmem_ld_16x32bx2_x32<64>(tl + kColW + 32, w + 32);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 16; ++t) z[t] = __uint_as_float(zr[t]);
            }
            if (LN) {
                float y[16], y2[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    z[t] += c_old;
                    y[t] = z[t];
                    y2[t] = z[t] * z[t];
                }
                feature_sum2(y, y2, red0, ew, lane);
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float mu = y[t] * (1.f / kD);
                    const float var = fmaxf(y2[t] * (1.f / kD) - mu * mu, 0.f);
                    const float rr = rsqrtf(var + p.eps);
                    z[t] = ld_bf16(qtile, sw128_off(t, j)) + gam * (z[t] - mu) * rr + bet;
                }
            }
            uint8_t* zst = smem + kOffZst + ((i & 1) * 2 + u) * kTile;
#pragma unroll
            for (int t = 0; t < 16; ++t)
                *reinterpret_cast<__nv_bfloat16*>(zst + t * 128 + j * 2) = __float2bfloat16_rn(z[t]);
            if (i + 1 < nsteps) write_a1();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, 128);
            if (leader) {
                if (!dead) {
                    tma_store_2d(&tmZ, smem + kOffZst + ((i & 1) * 2 + 0) * kTile, 0, unit0 * p.T + i * kTok);
                    if (has1)
                        tma_store_2d(&tmZ, smem + kOffZst + ((i & 1) * 2 + 1) * kTile, 0, unit1 * p.T + i * kTok);
                    bulk_commit();
                }
                mbar_arrive(&empty[s]);
                if (i + 1 < nsteps) mbar_arrive(a1_ready);
            }
        }
        // final state
        if (store_unit) {
            float* Wo = p.W_out + (size_t)unit * kD * kD;
#pragma unroll
            for (int i = 0; i < 64; ++i) Wo[i * kD + j] = __uint_as_float(w[i]);
            if (LN && p.c_out) p.c_out[(size_t)unit * kD + j] = cj;
        }
        if (leader) bulk_wait<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

}  // namespace ltc
}  // namespace ttt
