// Tensor-core (tcgen05) persistent kernel of the TTT-Linear prefill, plain
// and LN+residual inner models, d = 64, mini-batch b = 16, bf16 Q/K/V/Z,
// fp32 state.
//
// Method (paper digest "论文速览 | TTT", section 3.6, half-loss convention):
// per (sequence, head) unit and mini-batch i of 16 tokens with batch-start
// state W_i,
//     E_i = K_i W_i - V_i                              (key-side residual)
//     Z_i = Q_i W_i - (tril(Q_i K_i^T) * eta_s) E_i    (outputs)
//     W_{i+1} = W_i - K_i^T diag(eta) E_i             (end-of-batch state)
// and, for f(x) = x + LN(x W + c) (section 4.4), E_i is replaced by the LN
// backward Delta_i, the bias enters the causal matrix as tril(Q K^T + 1) and
// Z_i = Q_i + LN(Q_i W_i + c_i - (tril(Q_i K_i^T + 1) * eta_s) Delta_i).
//
// Transposed, with A_i = -eta_i * Delta_i^T (64 x 16):
//     W_{i+1}^T = W_i^T + A_i K_i
// and one step of look-ahead removes the serial dependence of E_i on W_i's
// bf16 copy:
//     E_i^T  = W_{i-1}^T K_i^T + A_{i-1} (K_{i-1} K_i^T) - V_i^T
//     Zq_i^T = W_{i-1}^T Q_i^T + A_{i-1} (K_{i-1} Q_i^T)      (= W_i^T Q_i^T)
// so one group of tensor-core MMAs per mini-batch produces W_i and the
// pre-residual of batch i from the epilogue's previous results:
//     MMA_P  P    = W_{i-1}^T [K_i^T | Q_i^T]          (4 x K16)
//     MMA_C  P   += A_{i-1} [K_{i-1} K_i^T | K_{i-1} Q_i^T]
//     MMA_W  W^T += A_{i-1} K_{i-1}
// and the epilogue adds the batch's own causal term
// sum_{s<=t} A_i[., s] S_i[t, s] in fp32 registers.
//
// Mapping onto sm_100a.  Each CTA owns two units stacked in M = 128 (unit 0
// in TMEM lanes 0-63, unit 1 in lanes 64-127), so one instruction serves
// both: their B operands are concatenated along N and each unit reads only
// its own columns (the cross products land in columns the other unit never
// reads).  The fp32 state W^T stays in TMEM for the whole sequence; the
// epilogue converts it to bf16 and writes it, together with A, back to TMEM
// as the A operand of the next group (tcgen05.mma with A in tensor memory),
// so no shared-memory operand needs a proxy fence.  b = 16 is below
// tcgen05's M range for the 16 x 16 products Q K^T, K_i K_{i-1}^T and
// Q_i K_{i-1}^T; two helper warps compute them with mma.sync.
//
// Warp roles (256 threads): warps 0-3 epilogue (warp q reads TMEM lanes
// 32q..32q+31: warps 0-1 unit 0, warps 2-3 unit 1; thread = one output
// feature j of one unit), warp 4 TMA producer, warp 5 MMA issuer, warps 6-7
// helpers (one per unit).  The epilogue warps hold the lowest warp ids, so
// on each SM sub-partition the scheduler favours them over the helper and
// waiting warps that share it.
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
constexpr int kStages = 5;      // input pipeline depth
constexpr int kThreads = 256;

// stage layout (bytes, from a 1024-aligned stage base)
constexpr int kTile = kTok * kD * 2;                 // 2048: one 16 x 64 bf16 tile
constexpr int kOffK0 = 0;                            // [K0 | Q0 | K1 | Q1]: B operand of MMA_P (N = 64)
constexpr int kOffQ0 = kTile;
constexpr int kOffK1 = 2 * kTile;
constexpr int kOffQ1 = 3 * kTile;
constexpr int kOffV0 = 4 * kTile;
constexpr int kOffV1 = 5 * kTile;
constexpr int kOffBS = 6 * kTile;                    // bf16 32 x 16 B operand of MMA_Z: tril(Q K^T) of both units
constexpr int kOffBC = kOffBS + 1024;                // bf16 64 x 16 B operand of MMA_C (K-major, no swizzle)
constexpr int kOffEta0 = kOffBC + 2048;              // 64 B per unit
constexpr int kOffEta1 = kOffEta0 + 64;
constexpr int kStageBytes = 16384;                   // 16 KB, multiple of 1024

constexpr int kOffStages = 0;
constexpr int kOffRed = kStages * kStageBytes;       // LN: 3 buffers x [4 warps][16] float2
constexpr int kOffBar = kOffRed + 3 * 4 * 16 * 8;
constexpr int kNumBars = 3 * kStages + 5;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64;

// TMEM columns (unit 0 in lanes 0-63, unit 1 in lanes 64-127)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColW = 0;       // fp32 W^T, 64 columns (both units)
constexpr uint32_t kColP = 64;      // fp32 P: unit 0 columns [64,96) = [E | Zq], unit 1 [96,128)
constexpr uint32_t kColZc = 128;    // fp32 causal term of the previous batch: unit 0 [128,144), unit 1 [144,160)
constexpr uint32_t kColAW = 160;    // bf16 W^T (A operand of MMA_P), 32 columns
constexpr uint32_t kColA = 192;     // bf16 A = -eta * Delta^T (A operand of MMA_C, MMA_Z), 8 columns
constexpr uint32_t kColAblk = 200;  // bf16 block-diagonal [A_0 0; 0 A_1] (A operand of MMA_W), 16 columns

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
    __nv_bfloat16* Z;
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
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragments (4 k-steps) of a 16 x 64 bf16 tile stored with the 128B swizzle
__device__ __forceinline__ void load_a_frags(uint32_t tile, int lane, uint32_t (*f)[4]) {
    const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        const int ch = 2 * ks + (lane >> 4);
        ldsm_x4(tile + row * 128 + ((ch ^ (row & 7)) << 4), f[ks]);
    }
}
// B fragments (4 k-steps, both 8-column n-tiles) of a 16 x 64 tile whose rows are the n index
__device__ __forceinline__ void load_b_frags(uint32_t tile, int lane, uint32_t (*f)[4]) {
    const int mi = lane >> 3;
    const int row = 8 * (mi >> 1) + (lane & 7);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        const int ch = 2 * ks + (mi & 1);
        ldsm_x4(tile + row * 128 + ((ch ^ (row & 7)) << 4), f[ks]);
    }
}
// Butterfly reduce-scatter of two 16-vectors over the 32 lanes of a warp:
// afterwards a[0], b[0] of lanes 2t and 2t+1 hold the warp sums of token t.
__device__ __forceinline__ void warp_reduce2(float* a, float* b, int lane) {
#pragma unroll
    for (int w = 16, n = 8; w >= 2; w >>= 1, n >>= 1) {
        const bool up = (lane & w) != 0;
#pragma unroll
        for (int k = 0; k < n; ++k) {
            const float sa = up ? a[k] : a[k + n], ka = up ? a[k + n] : a[k];
            const float sb = up ? b[k] : b[k + n], kb = up ? b[k + n] : b[k];
            a[k] = ka + __shfl_xor_sync(0xffffffffu, sa, w);
            b[k] = kb + __shfl_xor_sync(0xffffffffu, sb, w);
        }
    }
    a[0] += __shfl_xor_sync(0xffffffffu, a[0], 1);
    b[0] += __shfl_xor_sync(0xffffffffu, b[0], 1);
}

// Sums over the unit's 64 features (32 lanes x 2 warps) of two per-token
// quantities; every thread of the unit gets all 16 token sums.
__device__ __forceinline__ void feature_sum2(float* a, float* b, float2* red, int q, int lane) {
    warp_reduce2(a, b, lane);
    // the butterfly keeps the upper half of the remaining tokens on the lane
    // whose bit is set: lane bits 4,3,2,1 are token bits 3,2,1,0
    const int t = (lane >> 1) & 15;
    if ((lane & 1) == 0) red[q * 16 + t] = make_float2(a[0], b[0]);
    named_bar_sync(1 + (q >> 1), 64);
    const float2 mine = red[q * 16 + t], other = red[(q ^ 1) * 16 + t];
    const float sa = mine.x + other.x, sb = mine.y + other.y;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        a[k] = __shfl_sync(0xffffffffu, sa, 2 * k);
        b[k] = __shfl_sync(0xffffffffu, sb, 2 * k);
    }
}

__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), TTT_W8(r, 0)
                 : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        TTT_W8(r, 0), TTT_W8(r, 8), TTT_W8(r, 16), TTT_W8(r, 24)
        : "memory");
}

// tcgen05.mma with A in tensor memory
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// plain: two CTAs per SM (<= 128 registers); LN: one CTA per SM, no spills
template <bool LN>
__global__ void __launch_bounds__(kThreads, LN ? 1 : 2)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, Params p) {
    // No static shared memory: the dynamic buffer starts at the beginning of
    // the CTA's shared window (1024-byte aligned, as the 128B-swizzled tiles
    // need).  Addressing it directly keeps every access in the shared state
    // space (no generic-address loads).
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(p.status, kStatusBadSmem);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;                    // [kStages] TMA landed
    uint64_t* empty = bars + kStages;         // [kStages] stage free: MMA commit + 4 epilogue warps
    uint64_t* aux = bars + 2 * kStages;       // [kStages] helper products written (2 helper warps)
    uint64_t* op_ready = bars + 3 * kStages;  // A operands (bf16 W^T, A) written: 4 epilogue warps
    uint64_t* grp_done = op_ready + 1;        // one MMA group complete
    uint64_t* drain = op_ready + 2;           // final MMA drain
    uint64_t* stall = op_ready + 3;           // never arrived on (test hook)
    uint64_t* w_done = op_ready + 4;          // the group's state update (MMA_W) complete
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
            mbar_init(&empty[s], 5);
            mbar_init(&aux[s], 2);
        }
        mbar_init(op_ready, 4);
        mbar_init(grp_done, 1);
        mbar_init(drain, 1);
        mbar_init(stall, 1);
        mbar_init(w_done, 1);
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

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued_last = -1;
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
                tma_load_2d(st + kOffK0, &tmK, 0, y0, &full[s]);
                tma_load_2d(st + kOffQ0, &tmQ, 0, y0, &full[s]);
                tma_load_2d(st + kOffK1, &tmK, 0, y1, &full[s]);
                tma_load_2d(st + kOffQ1, &tmQ, 0, y1, &full[s]);
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
    } else if (warp == 5) {
        // ---------------------------------------------------------- MMA issuer
        // group g (0..nsteps) consumes A_{g-1} and bf16 W_{g-1}^T:
        //   MMA_W  W^T += A_{g-1} K_{g-1}           (block-diagonal A, two MMAs)
        //   MMA_Z  Zc   = A_{g-1} S_{g-1}^T         (causal term of batch g-1)
        //   MMA_P  P    = W_{g-1}^T [K_g | Q_g]^T    (four k-steps)
        //   MMA_C  P   += A_{g-1} [K_{g-1} K_g^T | K_{g-1} Q_g^T]
        if (lane == 0) {
            const uint32_t idP = make_idesc_bf16(128, 64, 0, 0);
            const uint32_t idW = make_idesc_bf16(128, 64, 0, 1);
            const uint32_t idZ = make_idesc_bf16(128, 32, 0, 0);
            bool ok = true;
            if (p.flags & TTT_FLAG_TEST_STALL) {
                // test hook: wait on a barrier nothing arrives on
                if (!wait_bounded(stall, 0, lim, s_abort)) fail();
                ok = false;
            }
            for (int g = 0; ok && g <= nsteps; ++g) {
                const int s = g % kStages;
                const uint32_t par = (g / kStages) & 1;
                const uint32_t st = smem_u32(smem + kOffStages + s * kStageBytes);
                const uint32_t sp = smem_u32(smem + kOffStages + ((g + kStages - 1) % kStages) * kStageBytes);
                uint64_t bdP[4];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) bdP[ks] = make_sdesc(st + kOffK0 + 32 * ks, 16, 1024, kSwizzle128B);
                const uint64_t bdC = make_sdesc(st + kOffBC, 128, 256, kSwizzleNone);
                // K tiles of the previous batch as MN-major B (one 64-wide atom each)
                const uint64_t bdW0 = make_sdesc(sp + kOffK0, 1024, 1024, kSwizzle128B);
                const uint64_t bdW1 = make_sdesc(sp + kOffK1, 1024, 1024, kSwizzle128B);
                const uint64_t bdZ = make_sdesc(sp + kOffBS, 128, 256, kSwizzleNone);
                if (g < nsteps && !wait_bounded(&full[s], par, lim, s_abort)) { fail(); break; }
                if (g >= 1 && g < nsteps && !wait_bounded(&aux[s], par, lim, s_abort)) { fail(); break; }
                if (!wait_bounded(op_ready, g & 1, lim, s_abort)) { fail(); break; }
                tc_fence_after();
                // the state update first, with its own commit, so that the
                // epilogue converts W_g while the rest of the group runs
                if (g >= 1) {
                    umma_ts(tbase + kColW, tbase + kColAblk, bdW0, idW, 1);
                    umma_ts(tbase + kColW, tbase + kColAblk + 8, bdW1, idW, 1);
                }
                umma_commit(w_done);
                if (g >= 1) umma_ts(tbase + kColZc, tbase + kColA, bdZ, idZ, 0);
                if (g < nsteps) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) umma_ts(tbase + kColP, tbase + kColAW + 8 * ks, bdP[ks], idP, ks > 0);
                    if (g >= 1) umma_ts(tbase + kColP, tbase + kColA, bdC, idP, 1);
                }
                umma_commit(grp_done);
                if (g >= 1) umma_commit(&empty[(g - 1) % kStages]);
            }
            // drain every MMA issued so far before TMEM is released
            umma_commit(drain);
            if (!wait_bounded(drain, 0, lim, nullptr)) fail();
        }
    } else if (warp >= 6) {
        // ------------------------------------- helpers: 16 x 16 products, one unit each
        const int u = warp - 6;
        const int r0 = lane >> 2, c0 = 2 * (lane & 3);
        for (int i = 0; i < nsteps; ++i) {
            const int s = i % kStages;
            if (!wait_bounded(&full[s], (i / kStages) & 1, lim, s_abort)) {
                if (lane == 0) fail();
                break;
            }
            uint8_t* st = smem + kOffStages + s * kStageBytes;
            const uint32_t kt = smem_u32(st + (u ? kOffK1 : kOffK0)), qt = smem_u32(st + (u ? kOffQ1 : kOffQ0));
            // fragments: Q_i and K_i as A (rows = tokens), K_i and K_{i-1} as B
            uint32_t fq[4][4], fka[4][4], fkb[4][4], fp[4][4];
            load_a_frags(qt, lane, fq);
            load_b_frags(kt, lane, fkb);
            const bool prev = i >= 1;
            if (prev) {
                const uint8_t* pst = smem + kOffStages + ((i - 1) % kStages) * kStageBytes;
                load_a_frags(kt, lane, fka);
                load_b_frags(smem_u32(pst + (u ? kOffK1 : kOffK0)), lane, fp);
            }
            // S = Q_i K_i^T, CQ = Q_i K_{i-1}^T, CK = K_i K_{i-1}^T, k-steps
            // interleaved across the six independent accumulators
            float aS[2][4] = {}, aQ[2][4] = {}, aK[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_16816(aS[0], fq[ks], fkb[ks][0], fkb[ks][1]);
                mma_16816(aS[1], fq[ks], fkb[ks][2], fkb[ks][3]);
                if (prev) {
                    mma_16816(aQ[0], fq[ks], fp[ks][0], fp[ks][1]);
                    mma_16816(aQ[1], fq[ks], fp[ks][2], fp[ks][3]);
                    mma_16816(aK[0], fka[ks], fp[ks][0], fp[ks][1]);
                    mma_16816(aK[1], fka[ks], fp[ks][2], fp[ks][3]);
                }
            }
            uint8_t* bs = st + kOffBS;
            uint8_t* bc = st + kOffBC;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int t = r0 + 8 * hh, ss = 8 * nt + c0;
                    // B_S rows (n = 16u + t): tril(Q_i K_i^T), strictly s <= t
                    *reinterpret_cast<uint32_t*>(bs + nosw_off(16 * u + t, ss)) =
                        pack_bf16x2(ss <= t ? aS[nt][2 * hh] : 0.f, ss + 1 <= t ? aS[nt][2 * hh + 1] : 0.f);
                    if (prev) {
                        // B_C rows (n = 32u + t): K_i K_{i-1}^T; rows 32u + 16 + t: Q_i K_{i-1}^T
                        *reinterpret_cast<uint32_t*>(bc + nosw_off(32 * u + t, ss)) =
                            pack_bf16x2(aK[nt][2 * hh], aK[nt][2 * hh + 1]);
                        *reinterpret_cast<uint32_t*>(bc + nosw_off(32 * u + 16 + t, ss)) =
                            pack_bf16x2(aQ[nt][2 * hh], aQ[nt][2 * hh + 1]);
                    }
                }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&aux[s]);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp, u = q >> 1;
        const int j = 32 * (q & 1) + lane;
        const int unit = u ? unit1 : unit0;
        const bool store_unit = (u == 0) || has1;
        const int n = unit / p.H, h = unit % p.H;
        const uint32_t tl = tbase + ((uint32_t)(32 * q) << 16);
        // three rotating reduction buffers: each reuse is two barriers apart
        float2* red0 = reinterpret_cast<float2*>(smem + kOffRed);
        float2* red1 = red0 + 4 * 16;
        float2* red2 = red1 + 4 * 16;
        float gam = 0.f, bet = 0.f, cj = 0.f;
        if (LN) {
            gam = p.gamma[(size_t)h * kD + j];
            bet = p.beta[(size_t)h * kD + j];
            cj = p.c0 ? p.c0[(size_t)n * p.c0_bstride + (size_t)h * kD + j] : 0.f;
        }
        uint32_t w[64];   // fp32 bits of column j of W (row j of W^T)
        {
            const float* W0u = p.W0 + (size_t)n * p.W0_bstride + (size_t)h * kD * kD;
#pragma unroll
            for (int i = 0; i < 64; ++i) w[i] = __float_as_uint(W0u[i * kD + j]);
            tmem_st_32x32b_x32(tl + kColW, w);
            tmem_st_32x32b_x32(tl + kColW + 32, w + 32);
            uint32_t pk[32], zero[8];
#pragma unroll
            for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(__uint_as_float(w[2 * c]), __uint_as_float(w[2 * c + 1]));
#pragma unroll
            for (int c = 0; c < 8; ++c) zero[c] = 0u;
            tmem_st_32x32b_x32(tl + kColAW, pk);
            // the other unit's half of the block-diagonal A stays zero
            tmem_st_32x32b_x8(tl + kColAblk + 8 * (1 - u), zero);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(op_ready);

        bool dead = false;   // set when a wait expired: run the loop without waiting
        __nv_bfloat16* Zu = p.Z + (size_t)unit * p.T * kD + j;
        float zb[16];        // previous batch: Zq (+ LN: c and the causal "+1" term)
        // Z of batch i-1 = zb + this group's causal term; the LN residual reads
        // Q of batch i-1, so its stage is released one step later.
        auto finish_z = [&](int i1, const float* zc, const uint8_t* pst) {
            float z[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) z[t] = zb[t] + zc[t];
            if (LN) {
                float y[16], y2[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    y[t] = z[t];
                    y2[t] = z[t] * z[t];
                }
                feature_sum2(y, y2, red2, q, lane);
                const uint8_t* qtile = pst + (u ? kOffQ1 : kOffQ0);
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float mu = y[t] * (1.f / kD);
                    const float r = rsqrtf(fmaxf(y2[t] * (1.f / kD) - mu * mu, 0.f) + p.eps);
                    z[t] = ld_bf16(qtile, sw128_off(t, j)) + gam * (z[t] - mu) * r + bet;
                }
            }
            if (!dead && store_unit) {
#pragma unroll
                for (int t = 0; t < 16; ++t) Zu[(size_t)(i1 * kTok + t) * kD] = __float2bfloat16_rn(z[t]);
            }
        };
        for (int i = 0; i < nsteps; ++i) {
            const int s = i % kStages;
            const uint32_t par = (i / kStages) & 1;
            const uint8_t* st = smem + kOffStages + s * kStageBytes;
            // 1. inputs of the batch (independent of the tensor cores): eta_t, eta_t v_t
            if (!dead && (!wait_bounded(&full[s], par, lim, s_abort) || !wait_bounded(&aux[s], par, lim, s_abort))) {
                dead = true;
                fail();
            }
            const uint8_t* vtile = st + (u ? kOffV1 : kOffV0);
            const float* etas = reinterpret_cast<const float*>(st + (u ? kOffEta1 : kOffEta0));
            float et[16], ev[16];
            if (p.eta) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 e4 = reinterpret_cast<const float4*>(etas)[c];
                    et[4 * c] = e4.x;
                    et[4 * c + 1] = e4.y;
                    et[4 * c + 2] = e4.z;
                    et[4 * c + 3] = e4.w;
                }
            } else {
#pragma unroll
                for (int t = 0; t < 16; ++t) et[t] = p.eta_const;
            }
            if (!LN) {
#pragma unroll
                for (int t = 0; t < 16; ++t) ev[t] = et[t] * ld_bf16(vtile, sw128_off(t, j));
            }
            // 2. W_i (after this group's MMA_W) -> bf16, held in registers
            if (!dead && !wait_bounded(w_done, i & 1, lim, s_abort)) {
                dead = true;
                fail();
            }
            tc_fence_after();
            tmem_ld_32x32b_x32(tl + kColW, w);
            tmem_ld_32x32b_x32(tl + kColW + 32, w + 32);
            tmem_wait_ld();
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(__uint_as_float(w[2 * c]), __uint_as_float(w[2 * c + 1]));
            // 3. P of this batch -> A row j; publish A and bf16 W^T for the next group
            if (!dead && !wait_bounded(grp_done, i & 1, lim, s_abort)) {
                dead = true;
                fail();
            }
            tc_fence_after();
            uint32_t pr[32], zr[16];
            tmem_ld_32x32b_x32(tl + kColP + 32 * u, pr);
            tmem_ld_32x32b_x16(tl + kColZc + 16 * u, zr);
            tmem_wait_ld();
            float av[16];   // A row j: -eta_t * delta_t
            const float c_old = cj;
            if (!LN) {
#pragma unroll
                for (int t = 0; t < 16; ++t) av[t] = fmaf(-et[t], __uint_as_float(pr[t]), ev[t]);
            } else {
                const uint8_t* ktile = st + (u ? kOffK1 : kOffK0);
                float y[16], y2[16], x[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    x[t] = __uint_as_float(pr[t]) + cj;
                    y[t] = x[t];
                    y2[t] = x[t] * x[t];
                }
                feature_sum2(y, y2, red0, q, lane);
                float g[16], gx[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float mu = y[t] * (1.f / kD);
                    const float r = rsqrtf(fmaxf(y2[t] * (1.f / kD) - mu * mu, 0.f) + p.eps);
                    x[t] = (x[t] - mu) * r;   // xhat
                    y[t] = r;
                    // e = k + gamma xhat + beta - v
                    const float e = ld_bf16(ktile, sw128_off(t, j)) + gam * x[t] + bet - ld_bf16(vtile, sw128_off(t, j));
                    g[t] = gam * e;
                    gx[t] = g[t] * x[t];
                    av[t] = g[t];
                }
                feature_sum2(g, gx, red1, q, lane);
                float csum = 0.f;
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float delta = y[t] * (av[t] - g[t] * (1.f / kD) - x[t] * gx[t] * (1.f / kD));
                    av[t] = -et[t] * delta;
                    csum += av[t];
                }
                cj += csum;
            }
            {
                uint32_t pa[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) pa[c] = pack_bf16x2(av[2 * c], av[2 * c + 1]);
                tmem_st_32x32b_x8(tl + kColA, pa);
                tmem_st_32x32b_x8(tl + kColAblk + 8 * u, pa);
                tmem_st_32x32b_x32(tl + kColAW, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(op_ready);

            // outputs of the previous batch, then keep this batch's pre-residual
            if (i >= 1) {
                float zc[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) zc[t] = __uint_as_float(zr[t]);
                const uint8_t* pst = smem + kOffStages + ((i - 1) % kStages) * kStageBytes;
                finish_z(i - 1, zc, pst);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[(i - 1) % kStages]);
            }
            float pre = LN ? c_old : 0.f;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                if (LN) pre += av[t];   // causal "+1" term: sum_{s<=t} A[s]
                zb[t] = __uint_as_float(pr[16 + t]) + pre;
            }
        }
        // final group: the last batch's causal term and the final state
        if (!dead && !wait_bounded(grp_done, nsteps & 1, lim, s_abort)) {
            dead = true;
            fail();
        }
        tc_fence_after();
        uint32_t zr[16];
        tmem_ld_32x32b_x16(tl + kColZc + 16 * u, zr);
        tmem_ld_32x32b_x32(tl + kColW, w);
        tmem_ld_32x32b_x32(tl + kColW + 32, w + 32);
        tmem_wait_ld();
        if (nsteps >= 1) {
            float zc[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) zc[t] = __uint_as_float(zr[t]);
            finish_z(nsteps - 1, zc, smem + kOffStages + ((nsteps - 1) % kStages) * kStageBytes);
        }
        if (store_unit && !dead) {
            float* Wo = p.W_out + (size_t)unit * kD * kD;
#pragma unroll
            for (int i = 0; i < 64; ++i) Wo[i * kD + j] = __uint_as_float(w[i]);
            if (LN && p.c_out) p.c_out[(size_t)unit * kD + j] = cj;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

}  // namespace ltc
}  // namespace ttt
