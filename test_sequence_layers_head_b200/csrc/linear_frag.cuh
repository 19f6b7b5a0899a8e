// Tensor-core persistent kernel of the TTT-Linear prefill, plain (f(x) = x W)
// and LN+residual (f(x) = x + LN(x W + c)), d = 64, mini-batch b = 16, bf16
// Q/K/V/Z, fp32 state.  Mini-batches are processed in pairs, so that every
// tensor-core round trip serves two of them.
//
// Method (paper digest "论文速览 | TTT", section 3.6, half-loss convention):
// per (sequence, head) unit and mini-batch i of 16 tokens with batch-start
// state W_i, and A_i = -(eta_i * E_i)^T (64 x 16, [j][s]):
//     E_i = K_i W_i - V_i
//     Z_i = Q_i W_i + tril(Q_i K_i^T) A_i^T             (causal mask s <= t)
//     W_{i+1}^T = W_i^T + A_i K_i
// For a pair of mini-batches a = 2g, b = 2g+1 with W = W_a:
//     E_a^T = W^T K_a^T - V_a^T                     Zq_a^T = W^T Q_a^T
//     E_b^T = W^T K_b^T + A_a (K_a K_b^T) - V_b^T   Zq_b^T = W^T Q_b^T + A_a (K_a Q_b^T)
//     W_{2g+2}^T = W^T + A_a K_a + A_b K_b
// (W_b = W_a + A_a K_a substituted into E_b and Zq_b: an identity, not an
// approximation.)
// LN+residual (section 4.4): the pre-activation x = k W + c replaces k W, E
// is replaced by the LN backward Delta (gamma, beta frozen, biased variance),
// the bias c is state (c += sum_s A[., s]) and enters every token product as
// "+1": with c = c_a,
//     X_b^T = W^T K_b^T + c + A_a (K_a K_b^T + 1)
//     pre_a^T = W^T Q_a^T + c + A_a tril(Q_a K_a^T + 1)^T
//     pre_b^T = W^T Q_b^T + c + A_a (K_a Q_b^T + 1) + A_b tril(Q_b K_b^T + 1)^T
// and Z = Q + LN(pre).  The per-token reductions over the 64 features are
// in-thread sums over 4 rows, three shuffle levels and one exchange between
// the unit's two warps.
//
// Mapping onto sm_100a.  Two units share a CTA and are stacked in M = 128
// (unit 0 in TMEM lanes 0-63, unit 1 in 64-127).  Per pair:
//   MMA_P  P = bf16(W)^T [K0a Q0a K1a Q1a K0b Q0b K1b Q1b]^T   (N = 128, 4 k-steps)
//   MMA_W  W^T += Ablk [K0a; K0b; K1a; K1b]                    (4 k-steps)
// with the fp32 state W^T resident in TMEM for the whole sequence, bf16 W^T
// rewritten into TMEM once per pair (A operand of MMA_P), and Ablk the
// block-diagonal [A0a A0b 0 0; 0 0 A1a A1b] in shared memory.  The rest of a
// pair runs on the epilogue warps' registers: tcgen05.ld.16x256b returns a
// TMEM tile in the m16n8 mma.sync accumulator layout, and an accumulator
// tile of A_a packed to bf16 pairs is the A-operand fragment of the
// correction A_a (K_a K_b^T) (mma.sync) and of the causal products.  The
// 16 x 16 token products tril(Q K^T), K_b K_a^T and Q_b K_a^T come from two
// helper warps (mma.sync) through shared memory.  Z goes out through a
// shared staging tile (stmatrix) and a TMA store.
//
// Warps 0-3: epilogue (warp q: unit q >> 1, state rows 32 (q & 1) .. +31 as
// two m16 tiles); warp 4 TMA producer; warp 5 MMA issuer; warps 6-7 helpers
// (one per unit).  Every wait is bounded; on expiry the kernel records
// kStatusTimeout, stops issuing new asynchronous work, drains what it issued
// and returns.
#pragma once
#include "common.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace ttt {
namespace lfr {

using tcc::ldsm_x4;
using tcc::load_a_frags;
using tcc::load_b_frags;
using Params = tcc::LinearParams;
using tcc::tmem_st_32x32b_x32;
using tcc::umma_ts;

constexpr int kD = 64;
constexpr int kTok = 16;
constexpr int kThreads = 256;
constexpr long long kOneUnitMaxUnits = 148;   // one unit per CTA up to this many units (the SM count)
constexpr int kStages = 3;       // input pipeline depth, in pairs of mini-batches
constexpr int kHring = 2;        // helper product slots, in pairs

// input stage (bytes from a 1024-aligned base), one pair of mini-batches:
// eight 16 x 64 bf16 tiles [K0a Q0a K1a Q1a K0b Q0b K1b Q1b] (the N = 128 B
// operand of MMA_P), then V and eta
constexpr int kTile = kTok * kD * 2;   // 2048
__host__ __device__ constexpr int off_k(int u, int hb) { return hb * 4 * kTile + u * 2 * kTile; }
__host__ __device__ constexpr int off_q(int u, int hb) { return off_k(u, hb) + kTile; }
__host__ __device__ constexpr int off_v(int u, int hb) { return 8 * kTile + (2 * hb + u) * kTile; }
__host__ __device__ constexpr int off_eta(int u, int hb) { return 12 * kTile + (2 * hb + u) * 64; }
constexpr int kStageBytes = 25600;   // 24832 used

// helper slot: per unit four bf16 16 x 16 products [t][s], 32-byte rows with
// the two 16-byte halves swapped on rows 4-7 and 12-15 (conflict-free
// ldmatrix and stores): S_a = tril(Q_a K_a^T), S_b = tril(Q_b K_b^T),
// M1 = K_b K_a^T, M2 = Q_b K_a^T
constexpr int kMat = 512;
constexpr int kHslot = 8 * kMat;   // 4096
__host__ __device__ constexpr int mat_off(int t, int half) { return t * 32 + ((half ^ ((t >> 2) & 1)) << 4); }

constexpr int kOffStages = 0;
constexpr int kOffH = kStages * kStageBytes;              // 76800
constexpr int kOffAblk = kOffH + kHring * kHslot;         // 84992 (1024-aligned)
constexpr int kAblkBytes = 16384;                         // bf16 [128 rows][64 k], K-major, no swizzle
constexpr int kOffZs = kOffAblk + kAblkBytes;             // Z staging: [4 warps] 32 tokens x 32 j, 64B swizzle
constexpr int kZsBytes = 2048;
constexpr int kOffRed = kOffZs + 4 * kZsBytes;           // LN: 2 buffers x [4 warps][4 c][8] float
constexpr int kOffBar = kOffRed + 2 * 4 * 16 * 8;
constexpr int kNumBars = 2 * kStages + 2 * kHring + 6;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64;
static_assert(kOffAblk % 1024 == 0 && kOffZs % 1024 == 0, "alignment");

// TMEM columns (unit 0 in lanes 0-63, unit 1 in lanes 64-127)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColW = 0;      // fp32 W^T (64 columns)
constexpr uint32_t kColP = 64;     // fp32 P (128 columns): unit u, batch hb at 64 hb + 32 u: [E (16) | Zq (16)]
constexpr uint32_t kColAW = 192;   // bf16 W^T (A operand of MMA_P), 32 columns

// byte offset of element (m, k) of the block-diagonal A operand of MMA_W:
// K-major, no swizzle, 8 x 16-byte core matrices, K-chunk stride 128 B,
// row-group stride 1024 B
__device__ __forceinline__ uint32_t ablk_off(int m, int k) {
    return (m >> 3) * 1024 + (k >> 3) * 128 + (m & 7) * 16 + (k & 7) * 2;
}

#ifndef TTT_HOST_EMULATION   // the host emulation supplies these four
__device__ __forceinline__ void tmem_ld_16x256b_x2(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
// stmatrix x4 with transpose: register fragment (row, col) -> shared (col, row)
__device__ __forceinline__ void stsm_x4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
}
// ldmatrix x4 with transpose
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// mma.sync m16n8k16 bf16 -> fp32 without the volatile qualifier, so that the
// compiler may interleave independent products
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
#endif

// Helper: the 16 x 16 product X Y^T + add of two 16 x 64 tiles (fragments
// given), masked to s <= t if `causal`, stored in bf16 at `dst` (layout of
// mat_off).
__device__ __forceinline__ void product_store(const uint32_t (*fa)[4], const uint32_t (*fb)[4], bool causal,
                                              float add, uint8_t* dst, int lane) {
    float acc[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        mma16816(acc[0], fa[ks], fb[ks][0], fb[ks][1]);
        mma16816(acc[1], fa[ks], fb[ks][2], fb[ks][3]);
    }
    const int r0 = lane >> 2, c0 = 2 * (lane & 3);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int t = r0 + 8 * hh, s = 8 * nt + c0;
            float lo = acc[nt][2 * hh] + add, hi = acc[nt][2 * hh + 1] + add;
            if (causal) {
                lo = s <= t ? lo : 0.f;
                hi = s + 1 <= t ? hi : 0.f;
            }
            *reinterpret_cast<uint32_t*>(dst + mat_off(t, nt) + c0 * 2) = pack_bf16x2(lo, hi);
        }
}

// LN: sums over the unit's 64 features of two per-token quantities sa[k],
// sb[k] (the thread's tokens k = 2 nt + e1 -> t = 8 nt + 2 c + e1).  The eight
// lanes of a warp that hold the same tokens (same c) reduce the eight values
// by recursive halving: at each of three levels a lane keeps one half of its
// list and adds the partner's copy of that half (4 + 2 + 1 shuffles), so lane
// r = lane / 4 ends with the warp's sum of entry r.  The entries go to shared
// memory as [warp][c][8]; after a named barrier over the unit's NW warps (2:
// warps q, q ^ 1; 4: warps 0-3) every thread adds up the NW lists of its c.
// (Measured: merging two of these into one reduction of more values, or the
// forward and backward sums of a mini-batch into one, is slower.)
template <int NW>
__device__ __forceinline__ void tok_sum2(float* sa, float* sb, float* red, int q, int lane) {
    const float l0[8] = {sa[0], sa[1], sa[2], sa[3], sb[0], sb[1], sb[2], sb[3]};
    float l1[4], l2[2];
    {
        const bool up = (lane & 16) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float keep = up ? l0[4 + i] : l0[i], send = up ? l0[i] : l0[4 + i];
            l1[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
    }
    {
        const bool up = (lane & 8) != 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float keep = up ? l1[2 + i] : l1[i], send = up ? l1[i] : l1[2 + i];
            l2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
    }
    const bool up = (lane & 4) != 0;
    const float l3 = (up ? l2[1] : l2[0]) + __shfl_xor_sync(0xffffffffu, up ? l2[0] : l2[1], 4);
    const int c = lane & 3;
    red[(q * 4 + c) * 8 + (lane >> 2)] = l3;
    if (NW == 2)
        named_bar_sync(1 + (q >> 1), 64);
    else
        named_bar_sync(1, 128);
    float tot[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int ww = NW == 2 ? (q & 2) + w : w;
        const float4* src = reinterpret_cast<const float4*>(red + (ww * 4 + c) * 8);
        const float4 x0 = src[0], x1 = src[1];
        tot[0] += x0.x; tot[1] += x0.y; tot[2] += x0.z; tot[3] += x0.w;
        tot[4] += x1.x; tot[5] += x1.y; tot[6] += x1.z; tot[7] += x1.w;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        sa[k] = tot[k];
        sb[k] = tot[4 + k];
    }
}

// bf16 element e (0..3, accumulator order) of an ldmatrix.trans fragment pair
__device__ __forceinline__ float frag_val(const uint32_t* f, int nt, int e) {
    const uint32_t x = f[2 * nt + (e >> 1)];
    return (e & 1) ? bf16_hi(x) : bf16_lo(x);
}

// UPC = units per CTA.  2: two units stacked in M = 128, each epilogue warp
// owns 32 state rows (two m16 tiles).  1: the CTA's unit is loaded into both
// halves of M = 128 and each epilogue warp owns 16 of its rows, one m16 tile
// on its own lane quadrant (rows 0-15, 32-47 from the first half, 16-31,
// 48-63 from the second); the other lanes carry unused copies.  1 is for
// workloads with fewer units than SMs: half the serial work per warp.
template <bool LN, int UPC>
__global__ void __launch_bounds__(kThreads, LN ? 1 : 2)
    linear_frag_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmZ,
                       const __grid_constant__ CUtensorMap tmZ1, Params p) {
    // the dynamic buffer starts at the CTA's shared window (1024-aligned)
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(p.status, kStatusBadSmem);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;                   // [kStages] TMA landed
    uint64_t* empty = bars + kStages;        // [kStages] stage free: 4 epilogue warps
    uint64_t* haux = bars + 2 * kStages;     // [kHring] helper products written: 2 helpers
    uint64_t* hfree = haux + kHring;         // [kHring] helper slot consumed: 4 epilogue warps
    uint64_t* aw_ready = hfree + kHring;     // bf16 W^T in TMEM: 4 epilogue warps
    uint64_t* a_ready = aw_ready + 1;        // A of the pair in the A block: 4 epilogue warps
    uint64_t* p_ready = aw_ready + 2;        // MMA_P complete
    uint64_t* w_done = aw_ready + 3;         // MMA_W complete
    uint64_t* drain = aw_ready + 4;          // final MMA drain
    uint64_t* stall = aw_ready + 5;          // never arrived on (test hook)
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit0 = UPC * blockIdx.x;
    const bool has1 = UPC == 2 && unit0 + 1 < p.U;
    const int unit1 = has1 ? unit0 + 1 : unit0;
    const int nsteps = p.nsteps;
    const int npairs = (nsteps + 1) / 2;
    const uint64_t lim = p.wait_ns;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        for (int s = 0; s < kHring; ++s) {
            mbar_init(&haux[s], 2);
            mbar_init(&hfree[s], 4);
        }
        mbar_init(aw_ready, 4);
        mbar_init(a_ready, 4);
        mbar_init(p_ready, 1);
        mbar_init(w_done, 1);
        mbar_init(drain, 1);
        mbar_init(stall, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
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
    auto stage_ptr = [&](int g) { return smem + kOffStages + (g % kStages) * kStageBytes; };
    auto hslot_ptr = [&](int g) { return smem + kOffH + (g % kHring) * kHslot; };

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued_last = -1;
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            for (int g = 0; g < npairs; ++g) {
                const int s = g % kStages;
                if (g >= kStages && !wait_bounded(&empty[s], ((g / kStages) - 1) & 1, lim, s_abort)) {
                    fail();
                    break;
                }
                if (*s_abort) break;
                const int nb = (2 * g + 1 < nsteps) ? 2 : 1;   // mini-batches in this pair
                uint8_t* st = stage_ptr(g);
                mbar_arrive_expect_tx(&full[s], nb * (6 * kTile + (p.eta ? 128 : 0)));
                for (int hb = 0; hb < nb; ++hb) {
                    const int y0 = unit0 * p.T + (2 * g + hb) * kTok, y1 = unit1 * p.T + (2 * g + hb) * kTok;
                    tma_load_2d(st + off_k(0, hb), &tmK, 0, y0, &full[s]);
                    tma_load_2d(st + off_q(0, hb), &tmQ, 0, y0, &full[s]);
                    tma_load_2d(st + off_k(1, hb), &tmK, 0, y1, &full[s]);
                    tma_load_2d(st + off_q(1, hb), &tmQ, 0, y1, &full[s]);
                    tma_load_2d(st + off_v(0, hb), &tmV, 0, y0, &full[s]);
                    tma_load_2d(st + off_v(1, hb), &tmV, 0, y1, &full[s]);
                    if (p.eta) {
                        bulk_load(st + off_eta(0, hb), p.eta + (size_t)y0, 64, &full[s]);
                        bulk_load(st + off_eta(1, hb), p.eta + (size_t)y1, 64, &full[s]);
                    }
                }
                issued_last = g;
            }
            // every issued load must land before the CTA exits (a TMA load
            // always completes, so these waits ignore the abort flag)
            for (int g = issued_last - kStages + 1; g <= issued_last; ++g) {
                if (g < 0) continue;
                if (!wait_bounded(&full[g % kStages], (g / kStages) & 1, lim, nullptr)) fail();
            }
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------- MMA issuer
        //   per pair g, once bf16 W_{2g} is in TMEM:  MMA_P  P = bf16(W)^T [K|Q]^T  (N = 128)
        //   once A of the pair is in the A block:     MMA_W  W^T += Ablk [K0a; K0b; K1a; K1b]
        if (lane == 0) {
            const uint32_t idP = make_idesc_bf16(128, 128, 0, 0);
            const uint32_t idW = make_idesc_bf16(128, 64, 0, 1);
            const uint32_t ablk = smem_u32(smem + kOffAblk);
            bool ok = true;
            auto W = [&](uint64_t* b, uint32_t par) {
                if (ok && !wait_bounded(b, par, lim, s_abort)) {
                    fail();
                    ok = false;
                }
                return ok;
            };
            if (p.flags & TTT_FLAG_TEST_STALL) {
                // test hook: wait on a barrier nothing arrives on
                if (!wait_bounded(stall, 0, lim, s_abort)) fail();
                ok = false;
            }
            for (int g = 0; ok && g < npairs; ++g) {
                const uint32_t st = smem_u32(stage_ptr(g));
                if (!W(aw_ready, g & 1) || !W(&full[g % kStages], (g / kStages) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ts(tbase + kColP, tbase + kColAW + 8 * ks, make_sdesc(st + 32 * ks, 16, 1024, kSwizzle128B),
                            idP, ks > 0);
                umma_commit(p_ready);
                if (!W(a_ready, g & 1)) break;
                tc_fence_after();
                const bool hasb = 2 * g + 1 < nsteps;
                // k-step 2u + hb: rows of unit u hold A_{u,hb}, the other unit's rows zero
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const int u = ks >> 1, hb = ks & 1;
                    if (hb && !hasb) continue;
                    umma_bf16(tbase + kColW, make_sdesc(ablk + 256 * ks, 128, 1024, kSwizzleNone),
                              make_sdesc(st + off_k(u, hb), 1024, 1024, kSwizzle128B), idW, 1);
                }
                umma_commit(w_done);
            }
            // drain every MMA issued so far before TMEM is released
            umma_commit(drain);
            if (!wait_bounded(drain, 0, lim, nullptr)) fail();
        }
    } else if (warp >= 6) {
        // -------------------------------- helpers: 16 x 16 token products, one unit each
        const int u = warp - 6;
        for (int g = 0; g < npairs; ++g) {
            if (!wait_bounded(&full[g % kStages], (g / kStages) & 1, lim, s_abort) ||
                (g >= kHring && !wait_bounded(&hfree[g % kHring], ((g / kHring) - 1) & 1, lim, s_abort))) {
                if (lane == 0) fail();
                break;
            }
            const uint32_t st = smem_u32(stage_ptr(g));
            uint8_t* hs = hslot_ptr(g) + u * 4 * kMat;
            const bool hasb = 2 * g + 1 < nsteps;
            uint32_t fka[4][4], fx[4][4], fy[4][4];
            load_b_frags(st + off_k(u, 0), lane, fka);      // K_a as B
            load_a_frags(st + off_q(u, 0), lane, fx);       // Q_a as A
            // LN: "+1" for the bias term of every token product
            const float one = LN ? 1.f : 0.f;
            product_store(fx, fka, true, one, hs, lane);         // S_a
            if (hasb) {
                load_a_frags(st + off_q(u, 1), lane, fx);   // Q_b as A
                product_store(fx, fka, false, one, hs + 3 * kMat, lane);   // M2 = Q_b K_a^T (+1)
                load_b_frags(st + off_k(u, 1), lane, fy);   // K_b as B
                product_store(fx, fy, true, one, hs + kMat, lane);         // S_b
                load_a_frags(st + off_k(u, 1), lane, fx);   // K_b as A
                product_store(fx, fka, false, one, hs + 2 * kMat, lane);   // M1 = K_b K_a^T (+1)
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&haux[g % kHring]);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp, u = q >> 1;
        const int jb = 32 * (q & 1) + (UPC == 1 ? 16 * u : 0);   // first state row (feature) of this warp
        constexpr int NMT = UPC == 2 ? 2 : 1;                     // m16 tiles per warp
        // TMEM lane of the first row of m-tile mt (rows and lanes coincide within a unit half)
        auto lane0 = [&](int mt) { return 64 * u + jb + 16 * mt; };
        const int r = lane >> 2, c = lane & 3;
        const int unit = u ? unit1 : unit0;
        const bool store_unit = (u == 0) || has1 || UPC == 1;
        const int n = unit / p.H, h = unit % p.H;
        const uint32_t tl = tbase + ((uint32_t)(32 * q) << 16);
        uint8_t* zs = smem + kOffZs + q * kZsBytes;   // this warp's Z staging tile
        // LN: gamma, beta and the bias state c of this thread's rows jb + 16 mt + r + 8 h
        float gam[2][2] = {}, bet[2][2] = {}, cst[2][2] = {};
        float* red = reinterpret_cast<float*>(smem + kOffRed);
        int nred = 0;   // reductions so far (two alternating buffers)
        if (LN) {
#pragma unroll
            for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int j = jb + 16 * mt + r + 8 * hh;
                    gam[mt][hh] = p.gamma[(size_t)h * kD + j];
                    bet[mt][hh] = p.beta[(size_t)h * kD + j];
                    cst[mt][hh] = p.c0 ? p.c0[(size_t)n * p.c0_bstride + (size_t)h * kD + j] : 0.f;
                }
        }
        auto rsum = [&](float* sa, float* sb) {
            tok_sum2<4 / NMT>(sa, sb, red + (nred & 1) * 128, q, lane);
            ++nred;
        };
        // W_0^T row j = column j of W_0, in fp32 and bf16; the other unit's
        // half of this warp's rows in the block-diagonal A stays zero
        {
            const int j = 32 * (q & 1) + lane;   // row held by this lane of the quadrant
            const float* W0u = p.W0 + (size_t)n * p.W0_bstride + (size_t)h * kD * kD;
            uint32_t w[64], pk[32];
#pragma unroll
            for (int i = 0; i < 64; ++i) w[i] = __float_as_uint(W0u[i * kD + j]);
            tmem_st_32x32b_x32(tl + kColW, w);
            tmem_st_32x32b_x32(tl + kColW + 32, w + 32);
#pragma unroll
            for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
            tmem_st_32x32b_x32(tl + kColAW, pk);
            const int m = 64 * u + j;
            const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
            if (UPC == 2) {
#pragma unroll
                for (int k = 0; k < 32; k += 8)
                    *reinterpret_cast<uint4*>(smem + kOffAblk + ablk_off(m, 32 * (1 - u) + k)) = z4;
            } else {
                // rows not owned by an epilogue warp keep an all-zero A
#pragma unroll
                for (int k = 0; k < 64; k += 8)
                    *reinterpret_cast<uint4*>(smem + kOffAblk + ablk_off(m, k)) = z4;
            }
        }
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(aw_ready);

        bool dead = false;   // set when a wait expired: run the loop without waiting
        auto WT = [&](uint64_t* b, uint32_t par) {
            if (!dead && !wait_bounded(b, par, lim, s_abort)) {
                dead = true;
                fail();
            }
        };
        const int mi = lane >> 3;   // ldmatrix / stmatrix: matrix served by this lane's address
        // Z of a pair (bf16 pairs of tokens 2c, 2c+1: [hb][mt][nt][rows r / r+8]) is
        // staged and stored while the next pair's MMA_P runs
        uint32_t zp[2][2][2][2];
        auto store_z = [&](int g1) {
            if (lane == 0) bulk_wait_read<0>();   // the previous store has read the staging tile
            __syncwarp();
            const int t8 = 8 * (mi >> 1) + (lane & 7);
#pragma unroll
            for (int hb = 0; hb < 2; ++hb)
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt) {
                    const int t = 16 * hb + t8, chunk = 2 * mt + (mi & 1);
                    const uint32_t off = UPC == 2 ? t * 64 + ((chunk ^ ((t >> 1) & 3)) << 4)    // 64B swizzle
                                                  : t * 32 + ((chunk ^ ((t >> 2) & 1)) << 4);   // 32B swizzle
                    stsm_x4_t(smem_u32(zs) + off, zp[hb][mt][0][0], zp[hb][mt][0][1], zp[hb][mt][1][0],
                              zp[hb][mt][1][1]);
                }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && !dead && store_unit) {
                tma_store_2d(2 * g1 + 1 < nsteps ? &tmZ : &tmZ1, zs, jb, unit * p.T + 2 * g1 * kTok);
                bulk_commit();
            }
        };
        for (int g = 0; g < npairs; ++g) {
            const uint8_t* st = stage_ptr(g);
            const uint32_t hs = smem_u32(hslot_ptr(g) + u * 4 * kMat);
            const bool hasb = 2 * g + 1 < nsteps;
            // 0. W_{2g} (MMA_W of the previous pair) -> bf16 in TMEM, the A operand of MMA_P
            if (g >= 1) {
                WT(w_done, (g - 1) & 1);
                tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t w[32], pk[16];
                    tmem_ld_32x32b_x32(tl + kColW + 32 * half, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        pk[k] = pack_bf16x2(__uint_as_float(w[2 * k]), __uint_as_float(w[2 * k + 1]));
                    tmem_st_32x32b_x16(tl + kColAW + 16 * half, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(aw_ready);
                    mbar_arrive(&empty[(g - 1) % kStages]);   // MMA_W of pair g-1 was its last reader
                }
                if (UPC == 2) store_z(g - 1);
            }
            // 1. inputs: eta, eta * V (accumulator layout), the token products
            WT(&full[g % kStages], (g / kStages) & 1);
            WT(&haux[g % kHring], (g / kHring) & 1);
            float et[2][4];          // [hb]: eta of tokens 2c, 2c+1, 8+2c, 9+2c
            float ev[2][2][2][4];    // plain: [hb][mt][nt][e]: eta_t * V[t][j]
            uint32_t vf[2][2][4], kf[2][2][4], qf[2][2][4];   // LN: [hb][mt] bf16 fragments of V, K, Q
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                if (p.eta) {
                    const float* etas = reinterpret_cast<const float*>(st + off_eta(u, hb));
                    const float2 e0 = *reinterpret_cast<const float2*>(etas + 2 * c);
                    const float2 e1 = *reinterpret_cast<const float2*>(etas + 8 + 2 * c);
                    et[hb][0] = e0.x;
                    et[hb][1] = e0.y;
                    et[hb][2] = e1.x;
                    et[hb][3] = e1.y;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) et[hb][e] = p.eta_const;
                }
                const uint32_t vt = smem_u32(st + off_v(u, hb));
                const int t = 8 * (mi >> 1) + (lane & 7);
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt) {
                    const int jblk = (jb >> 3) + 2 * mt + (mi & 1);
                    const uint32_t off = t * 128 + ((jblk ^ (t & 7)) << 4);
                    if (LN) {
                        ldsm_x4_t(vt + off, vf[hb][mt]);
                        ldsm_x4_t(smem_u32(st + off_k(u, hb)) + off, kf[hb][mt]);
                        ldsm_x4_t(smem_u32(st + off_q(u, hb)) + off, qf[hb][mt]);
                    } else {
                        uint32_t v[4];
                        ldsm_x4_t(vt + off, v);
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) ev[hb][mt][nt][e] = et[hb][2 * nt + (e & 1)] * frag_val(v, nt, e);
                    }
                }
            }
            uint32_t msa[4], msb[4], m1[4], m2[4];
            {
                const int row = 8 * (mi >> 1) + (lane & 7);
                const uint32_t a = hs + mat_off(row, mi & 1);
                ldsm_x4(a, msa);
                ldsm_x4(a + kMat, msb);
                ldsm_x4(a + 2 * kMat, m1);
                ldsm_x4(a + 3 * kMat, m2);
            }
            // one unit per CTA: the previous pair's Z goes out while these loads are in
            // flight (measured faster there; with two units per CTA and two CTAs per SM
            // the other CTA hides the load latency and the earlier store is better)
            if (UPC == 1 && g >= 1) store_z(g - 1);
            // 2. P of the pair (E parts), accumulator layout
            WT(p_ready, g & 1);
            tc_fence_after();
            uint32_t pe[2][2][8];   // [hb][mt]
#pragma unroll
            for (int hb = 0; hb < 2; ++hb)
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt)
                    tmem_ld_16x256b_x2(tbase + ((uint32_t)lane0(mt) << 16) + kColP + 64 * hb + 32 * u, pe[hb][mt]);
            tmem_wait_ld();
            // 3. A_a = eta (V_a - E_a); E_b += A_a M1^T; A_b = eta (V_b - E_b)
            //    (LN: A = -eta Delta of the LN backward at X_a, X_b)
            uint32_t aa[2][4], ab[2][4];
            float c_old[2][2];
            if (LN) {
                // one mini-batch of the LN chain: x (pre-activation, accumulator
                // layout) -> A (fp32 in x, packed bf16 fragments in fr)
                auto ln_batch = [&](float (&x)[2][2][4], int hb, uint32_t (&fr)[2][4]) {
                    float s1[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float v = x[mt][nt][e];
                                s1[2 * nt + (e & 1)] += v;
                                s2[2 * nt + (e & 1)] += v * v;
                            }
                    rsum(s1, s2);
                    float rr[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float mu = s1[k] * (1.f / kD);
                        rr[k] = rsqrtf(fmaxf(s2[k] * (1.f / kD) - mu * mu, 0.f) + p.eps);
                        s1[k] = mu;
                    }
                    float gg[2][2][4], t1[4] = {0.f, 0.f, 0.f, 0.f}, t2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int k = 2 * nt + (e & 1), hh = e >> 1;
                                const float xh = (x[mt][nt][e] - s1[k]) * rr[k];   // x-hat
                                // e = k + gamma xhat + beta - v (residual of f), g = gamma e
                                const float res = frag_val(kf[hb][mt], nt, e) + gam[mt][hh] * xh + bet[mt][hh] -
                                                  frag_val(vf[hb][mt], nt, e);
                                const float g = gam[mt][hh] * res;
                                gg[mt][nt][e] = g;
                                x[mt][nt][e] = xh;
                                t1[k] += g;
                                t2[k] += g * xh;
                            }
                    rsum(t1, t2);
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int k = 2 * nt + (e & 1);
                                const float delta = rr[k] * (gg[mt][nt][e] - t1[k] * (1.f / kD) -
                                                             x[mt][nt][e] * t2[k] * (1.f / kD));
                                x[mt][nt][e] = -et[hb][k] * delta;
                            }
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt) {
                        fr[mt][0] = pack_bf16x2(x[mt][0][0], x[mt][0][1]);
                        fr[mt][1] = pack_bf16x2(x[mt][0][2], x[mt][0][3]);
                        fr[mt][2] = pack_bf16x2(x[mt][1][0], x[mt][1][1]);
                        fr[mt][3] = pack_bf16x2(x[mt][1][2], x[mt][1][3]);
                    }
                };
                float xa[2][2][4], xb[2][2][4];
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            xa[mt][nt][e] = __uint_as_float(pe[0][mt][4 * nt + e]) + cst[mt][e >> 1];
                            xb[mt][nt][e] = __uint_as_float(pe[1][mt][4 * nt + e]) + cst[mt][e >> 1];
                        }
                ln_batch(xa, 0, aa);
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) mma16816(xb[mt][nt], aa[mt], m1[2 * nt], m1[2 * nt + 1]);
                ln_batch(xb, 1, ab);
                // bias state: c += sum over the pair's tokens of A (fp32); a missing
                // second mini-batch contributes nothing
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float cs = 0.f;
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e1 = 0; e1 < 2; ++e1)
                                cs += xa[mt][nt][2 * hh + e1] + (hasb ? xb[mt][nt][2 * hh + e1] : 0.f);
                        cs += __shfl_xor_sync(0xffffffffu, cs, 1);
                        cs += __shfl_xor_sync(0xffffffffu, cs, 2);
                        c_old[mt][hh] = cst[mt][hh];
                        cst[mt][hh] += cs;
                    }
            } else {
#pragma unroll
            for (int mt = 0; mt < NMT; ++mt) {
                float a[2][4], b[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        a[nt][e] = fmaf(-et[0][2 * nt + (e & 1)], __uint_as_float(pe[0][mt][4 * nt + e]), ev[0][mt][nt][e]);
                aa[mt][0] = pack_bf16x2(a[0][0], a[0][1]);
                aa[mt][1] = pack_bf16x2(a[0][2], a[0][3]);
                aa[mt][2] = pack_bf16x2(a[1][0], a[1][1]);
                aa[mt][3] = pack_bf16x2(a[1][2], a[1][3]);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    float d[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) d[e] = __uint_as_float(pe[1][mt][4 * nt + e]);
                    mma16816(d, aa[mt], m1[2 * nt], m1[2 * nt + 1]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) b[nt][e] = fmaf(-et[1][2 * nt + (e & 1)], d[e], ev[1][mt][nt][e]);
                }
                ab[mt][0] = pack_bf16x2(b[0][0], b[0][1]);
                ab[mt][1] = pack_bf16x2(b[0][2], b[0][3]);
                ab[mt][2] = pack_bf16x2(b[1][0], b[1][1]);
                ab[mt][3] = pack_bf16x2(b[1][2], b[1][3]);
            }
            }
            // 4. A_a, A_b into the block-diagonal A operand of MMA_W (k = 32 u + 16 hb + s)
#pragma unroll
            for (int mt = 0; mt < NMT; ++mt) {
                const int m = 64 * u + jb + 16 * mt + r;
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const uint32_t* fr = hb ? ab[mt] : aa[mt];
                    const int k = 32 * u + 16 * hb + 2 * c;
                    *reinterpret_cast<uint32_t*>(smem + kOffAblk + ablk_off(m, k)) = fr[0];
                    *reinterpret_cast<uint32_t*>(smem + kOffAblk + ablk_off(m + 8, k)) = fr[1];
                    *reinterpret_cast<uint32_t*>(smem + kOffAblk + ablk_off(m, k + 8)) = fr[2];
                    *reinterpret_cast<uint32_t*>(smem + kOffAblk + ablk_off(m + 8, k + 8)) = fr[3];
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(a_ready);
            // 5. outputs while MMA_W runs:
            //    Z_a^T = P_Zqa + A_a S_a^T,  Z_b^T = P_Zqb + A_a M2^T + A_b S_b^T
            float zf[2][2][2][4];      // [hb][mt][nt][e]: pre-output (LN: then output) in fp32
            {
                uint32_t pq[2][2][8];
#pragma unroll
                for (int hb = 0; hb < 2; ++hb)
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt)
                        tmem_ld_16x256b_x2(tbase + ((uint32_t)lane0(mt) << 16) + kColP + 64 * hb + 32 * u + 16,
                                           pq[hb][mt]);
                tmem_wait_ld();
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        float* da = zf[0][mt][nt];
                        float* db = zf[1][mt][nt];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            da[e] = __uint_as_float(pq[0][mt][4 * nt + e]) + (LN ? c_old[mt][e >> 1] : 0.f);
                            db[e] = __uint_as_float(pq[1][mt][4 * nt + e]) + (LN ? c_old[mt][e >> 1] : 0.f);
                        }
                        mma16816(da, aa[mt], msa[2 * nt], msa[2 * nt + 1]);
                        mma16816(db, aa[mt], m2[2 * nt], m2[2 * nt + 1]);
                        mma16816(db, ab[mt], msb[2 * nt], msb[2 * nt + 1]);
                    }
            }
            if (LN) {
                // Z = Q + gamma LN(pre) + beta, per mini-batch of the pair
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    float s1[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float v = zf[hb][mt][nt][e];
                                s1[2 * nt + (e & 1)] += v;
                                s2[2 * nt + (e & 1)] += v * v;
                            }
                    rsum(s1, s2);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float mu = s1[k] * (1.f / kD);
                        s2[k] = rsqrtf(fmaxf(s2[k] * (1.f / kD) - mu * mu, 0.f) + p.eps);
                        s1[k] = mu;
                    }
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int k = 2 * nt + (e & 1), hh = e >> 1;
                                zf[hb][mt][nt][e] = frag_val(qf[hb][mt], nt, e) +
                                                    gam[mt][hh] * (zf[hb][mt][nt][e] - s1[k]) * s2[k] + bet[mt][hh];
                            }
                }
            }
#pragma unroll
            for (int hb = 0; hb < 2; ++hb)
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        zp[hb][mt][nt][0] = pack_bf16x2(zf[hb][mt][nt][0], zf[hb][mt][nt][1]);
                        zp[hb][mt][nt][1] = pack_bf16x2(zf[hb][mt][nt][2], zf[hb][mt][nt][3]);
                    }
            __syncwarp();
            if (lane == 0) mbar_arrive(&hfree[g % kHring]);
        }
        store_z(npairs - 1);
        // final state (MMA_W of the last pair)
        WT(w_done, (npairs - 1) & 1);
        tc_fence_after();
        if (lane == 0) bulk_wait<0>();   // Z stores complete before the CTA exits
        if (store_unit && !dead) {
            uint32_t w[32];
            // lane l of the quadrant holds row 32 (q & 1) + l of its unit half
            const bool own = UPC == 2 || (lane >> 4) == u;
            float* Wo = p.W_out + (size_t)unit * kD * kD + 32 * (q & 1) + lane;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld_32x32b_x32(tl + kColW + 32 * half, w);
                tmem_wait_ld();
                if (own) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) Wo[(32 * half + k) * kD] = __uint_as_float(w[k]);
                }
            }
            if (LN && p.c_out && c == 0) {
                // the four lanes of a row group hold the same bias rows; lane c = 0 writes them
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        p.c_out[(size_t)unit * kD + jb + 16 * mt + r + 8 * hh] = cst[mt][hh];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

}  // namespace lfr
}  // namespace ttt
