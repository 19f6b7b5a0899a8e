// Tensor-core (tcgen05) persistent kernel of the TTT-MLP prefill:
// f(x) = GELU(x W1 + c1) W2 + c2, d = 64, hidden m = 256, mini-batch b = 16,
// bf16 Q/K/V/Z, fp32 state.
//
// Method (paper digest "论文速览 | TTT", section 3.7, half-loss convention).
// Per (sequence, head) unit and mini-batch with batch-start parameters:
//   A  = K W1 + c1,  Hk = GELU(A),  E = Hk W2 + c2 - V
//   D1 = (E W2^T) * GELU'(A)
//   Aq = Q W1 + c1 - (tril(Q K^T + 1) * eta_s) D1,  Hq = GELU(Aq)
//   Z  = Hq W2 + c2 - (tril(Hq Hk^T + 1) * eta_s) E
//   W1 -= K^T diag(eta) D1,  c1 -= eta^T D1,  W2 -= Hk^T diag(eta) E,  c2 -= eta^T E
//
// Mapping onto sm_100a (everything transposed so that the hidden dim m = 256
// or the head dim d = 64 is the MMA's M):
//   S1  [A^T | Aq0^T] (m x 32)  = W1^T . [K^T | Q^T]           tcgen05, 2 tiles x 4 k-steps
//   S2  E0^T (d x 16)           = W2^T . Hk^T                  mma.sync on the epilogue warps
//   S3  G^T (m x 16)            = W2 . E^T                     mma.sync on the epilogue warps
//   S4  W1^T += (-eta D1)^T K,  Aq^T += (-eta D1)^T tril(Q K^T + 1)^T,
//       W2   += (-eta Hk)^T E                                  tcgen05, 6 MMAs
//   S5  Z0^T (d x 16)           = W2^T . Hq^T + (-eta E)^T tril(Hq Hk^T + 1)^T   tcgen05
// The fp32 accumulators W1^T (m x d) and W2 (m x d) stay in tensor memory for
// the whole sequence; bf16 W1^T is refreshed in tensor memory (A operand of
// S1) and bf16 W2 in shared memory (A operand of S5 as MN-major, of S2/S3 as
// ldmatrix fragments) once per mini-batch.  S2 and S3 have N = 16 tokens, too
// narrow for a tcgen05 round trip (issue, commit, wake-up) to pay, so the
// epilogue warps run them on mma.sync and keep E0, G and GELU'(A) in the
// accumulator fragment layout, which is also what tcgen05.ld.16x256b returns
// for A: D1 = G * GELU'(A) needs no exchange.  The "+1" bias terms of the
// causal matrices, the biases and GELU are applied in fp32 registers by the
// epilogue; the 16 x 16 products Q K^T and Hq Hk^T are computed by two helper
// warps with mma.sync.
//
// The output path of a mini-batch (Hq, S5, Z) is software-pipelined behind
// the next mini-batch's S1/E1: bf16 W2, Hk and Hq are double-buffered so S5
// of batch i reads the state of batch i while S2 of batch i+1 reads the next.
//
// One unit per CTA, 12 warps.  Epilogue warps 0-3 and 8-11: warp w reads TMEM
// lanes 32 (w & 3) .. + 31 (its quadrant) and covers the tokens 8 (w >> 3) .. + 7
// of the mini-batch; in the fragment layout lane (r, c) = (lane / 4, lane % 4)
// holds hidden rows 128 tt + 32 (w & 3) + 16 m + r (+ 8) and tokens 2c, 2c + 1
// of that half.  Warp 4 TMA producer; warp 5 MMA issuer; warps 6-7 helpers.
// Every wait is bounded; on expiry the kernel records kStatusTimeout, drains
// what it issued and returns.
#pragma once
#include "common.cuh"
#include "tc_common.cuh"
#include "ptx.cuh"

namespace ttt {
namespace mtc {

using tcc::ld_bf16;
using tcc::ldsm_x4;
using tcc::mma_16816;
using tcc::nosw_off;
using tcc::sw128_off;
using tcc::tmem_st_32x32b_x32;
using tcc::tmem_st_32x32b_x8;
using tcc::umma_ts;

constexpr int kD = 64, kM = 256, kTok = 16;
constexpr int kStages = 4;
constexpr int kThreads = 384;   // 8 epilogue warps (0-3, 8-11), producer 4, MMA 5, helpers 6-7
constexpr int kTile = kTok * kD * 2;   // 2048

// stage layout
constexpr int kOffK = 0;               // [K | Q]: B operand of S1 (N = 32)
constexpr int kOffQ = kTile;
constexpr int kOffV = 2 * kTile;
constexpr int kOffS1 = 3 * kTile;      // bf16 16 x 16 tril(Q K^T), K-major no swizzle
constexpr int kOffEta = kOffS1 + 512;
constexpr int kStageBytes = 7168;

constexpr int kOffStages = 0;
constexpr int kOffW2 = 28672;          // 2 x bf16 W2 [h][j], 128B swizzle, 256 rows (32 KB each)
constexpr int kOffHk = kOffW2 + 65536; // 2 x bf16 Hk [t][h]: 4 K-major sub-tiles of 16 x 64 (8 KB each)
constexpr int kOffHq = kOffHk + 16384; // 2 x bf16 Hq [t][h] (8 KB each)
constexpr int kOffE = kOffHq + 16384;  // bf16 E [t][j], 128B swizzle (2 KB)
constexpr int kOffAE = kOffE + 2048;   // 2 x bf16 (-eta E)^T [j][t], K-major no swizzle (2 KB each): S5 of
                                       // batch i reads it while E2 of batch i+1 writes the other one
constexpr int kOffS2 = kOffAE + 4096;  // bf16 tril(Hq Hk^T + 1), K-major no swizzle (512 B)
constexpr int kOffXch = kOffS2 + 512;  // two buffers x [2 halves][4 quadrants][4][32] float2 (partial sums)
constexpr int kOffBar = kOffXch + 2 * 1024 * 8;
constexpr int kNumBars = 3 * kStages + 14;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64;

// TMEM columns (M = 128 tiles: lane = hidden row mod 128; M = 64 stages use
// lanes 0-15 of each 32-lane quadrant)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t cW1 = 0;     // fp32 W1^T, tile t at 64 t
constexpr uint32_t cW2 = 128;   // fp32 W2, tile t at 128 + 64 t
constexpr uint32_t cA = 256;    // fp32 [A | Aq], tile t at 256 + 32 t
constexpr uint32_t cE = 352;    // fp32 E0^T (M = 64)
constexpr uint32_t cZ = 368;    // fp32 Z0^T (M = 64)
constexpr uint32_t cAW1 = 384;  // bf16 W1^T (A of S1), tile t at 384 + 32 t
constexpr uint32_t cAD1 = 448;  // bf16 (-eta D1)^T, tile t at 448 + 8 t
constexpr uint32_t cAHk = 464;  // bf16 (-eta Hk)^T, tile t at 464 + 8 t

struct Params {
    int H, T, nsteps, per_seq;
    const float* eta;
    float eta_const;
    const float* W1;
    const float* c1;
    const float* W2;
    const float* c2;
    __nv_bfloat16* Z;
    float* W1_out;
    float* c1_out;
    float* W2_out;
    float* c2_out;
    int* status;
    unsigned long long wait_ns;
    unsigned flags;
    // LN+residual on the output layer (template LN): gamma, beta [H, 64]
    const float* gamma;
    const float* beta;
    float eps;
};

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t* r) { tmem_ld_32x32b_x16(taddr, r); }

#ifndef TTT_HOST_EMULATION   // the host emulation supplies these nine
// ldmatrix / stmatrix x4 with transpose
__device__ __forceinline__ void ldsm_x4_tr(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void stsm_x4_tr(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_tr(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
__device__ __forceinline__ void stsm_x2_tr(uint32_t addr, uint32_t r0, uint32_t r1) {
    asm volatile("stmatrix.sync.aligned.m8n8.x2.trans.shared.b16 [%0], {%1,%2};" ::"r"(addr), "r"(r0), "r"(r1)
                 : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_16x256b_x1(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
// packed pair (row r, col c) and (row r + 8, col c): the accumulator layout's token pairs
__device__ __forceinline__ void tmem_st_16x128b_x1(uint32_t taddr, uint32_t r0, uint32_t r1) {
    asm volatile("tcgen05.st.sync.aligned.16x128b.x1.b32 [%0], {%1,%2};" ::"r"(taddr), "r"(r0), "r"(r1) : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
#endif
// element e (accumulator order) of an ldmatrix.trans fragment set: n-tile nt,
// rows r (e < 2) or r + 8, tokens 2c + (e & 1)
__device__ __forceinline__ float frag_at(const uint32_t* f, int nt, int e) {
    const uint32_t x = f[2 * nt + (e >> 1)];
    return (e & 1) ? bf16_hi(x) : bf16_lo(x);
}

// 16 x 16 tril(X Y^T) with X, Y stored as [t][k] K-major 128B-swizzled
// sub-tiles of 64 columns (nsub of them); n-tile nt (8 columns) only.
__device__ __forceinline__ void tril_product(uint32_t xbase, uint32_t ybase, int nsub, int nt, int lane,
                                             uint8_t* dst, float add = 0.f) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int arow = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int brow = 8 * nt + (lane & 7);
    for (int sub = 0; sub < nsub; ++sub) {
        const uint32_t xs = xbase + 2048 * sub, ys = ybase + 2048 * sub;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4], b[4];
            const int ach = 2 * ks + (lane >> 4);
            ldsm_x4(xs + arow * 128 + ((ach ^ (arow & 7)) << 4), a);
            // matrices: (rows 8nt.., chunk 2ks), (.., 2ks+1) twice (x4 keeps the code uniform)
            const int bch = 2 * ks + ((lane >> 3) & 1);
            ldsm_x4(ys + brow * 128 + ((bch ^ (brow & 7)) << 4), b);
            mma_16816(acc, a, b[0], b[1]);
        }
    }
    const int r0 = lane >> 2, c0 = 2 * (lane & 3);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int t = r0 + 8 * hh, s = 8 * nt + c0;
        *reinterpret_cast<uint32_t*>(dst + nosw_off(t, s)) =
            pack_bf16x2(s <= t ? acc[2 * hh] + add : 0.f, s + 1 <= t ? acc[2 * hh + 1] + add : 0.f);
    }
}

template <bool LN>
__global__ void __launch_bounds__(kThreads, 1)
    mlp_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(p.status, kStatusBadSmem);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;                    // [kStages] TMA landed
    uint64_t* empty = bars + kStages;         // [kStages] MMA (after S4) + 4 epilogue warps (after E2)
    uint64_t* aux1 = bars + 2 * kStages;      // [kStages] tril(Q K^T) written (helper warp 6)
    uint64_t* d_a = bars + 3 * kStages;       // S1 done
    uint64_t* d_e = d_a + 1;                  // S2 done
    // d_a + 2 unused
    uint64_t* d_u = d_a + 3;                  // S4 done
    uint64_t* d_z = d_a + 4;                  // S5 done
    uint64_t* hk_rdy = d_a + 5;               // Hk^T, (-eta Hk)^T written (4 epilogue warps)
    // d_a + 6 unused
    uint64_t* d1_rdy = d_a + 7;               // (-eta D1)^T written
    uint64_t* hq_rdy = d_a + 8;               // Hq^T written
    uint64_t* aux2 = d_a + 9;                 // tril(Hq Hk^T) written (2 helper warps)
    uint64_t* aw1_rdy = d_a + 10;             // bf16 W1^T refreshed
    uint64_t* w2_rdy = d_a + 11;              // bf16 W2 refreshed
    uint64_t* drain = d_a + 12;
    uint64_t* stall = d_a + 13;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x;
    const int nsteps = p.nsteps;
    const uint64_t lim = p.wait_ns;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 9);
            mbar_init(&aux1[s], 1);
        }
        for (uint64_t* b = d_a; b <= d_z; ++b) mbar_init(b, 1);
        mbar_init(hk_rdy, 8);
        mbar_init(d1_rdy, 8);
        mbar_init(hq_rdy, 8);
        mbar_init(aux2, 2);
        mbar_init(aw1_rdy, 8);
        mbar_init(w2_rdy, 8);
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

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued_last = -1;
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            const uint32_t bytes = 3 * kTile + (p.eta ? 64 : 0);
            for (int i = 0; i < nsteps; ++i) {
                const int s = i % kStages;
                if (i >= kStages && !wait_bounded(&empty[s], ((i / kStages) - 1) & 1, lim, s_abort)) {
                    fail();
                    break;
                }
                if (*s_abort) break;
                uint8_t* st = smem + kOffStages + s * kStageBytes;
                mbar_arrive_expect_tx(&full[s], bytes);
                const int y = unit * p.T + i * kTok;
                tma_load_2d(st + kOffK, &tmK, 0, y, &full[s]);
                tma_load_2d(st + kOffQ, &tmQ, 0, y, &full[s]);
                tma_load_2d(st + kOffV, &tmV, 0, y, &full[s]);
                if (p.eta) bulk_load(st + kOffEta, p.eta + (size_t)y, 64, &full[s]);
                issued_last = i;
            }
            for (int i = issued_last - kStages + 1; i <= issued_last; ++i) {
                if (i < 0) continue;
                if (!wait_bounded(&full[i % kStages], (i / kStages) & 1, lim, nullptr)) fail();
            }
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS1 = make_idesc_bf16(128, 32, 0, 0);
            const uint32_t idS2 = make_idesc_bf16(64, 16, 1, 0);   // A = W2 as MN-major
            const uint32_t idUpd = make_idesc_bf16(128, 64, 0, 1); // B MN-major (K or E tile)
            const uint32_t idAq = make_idesc_bf16(128, 16, 0, 0);
            const uint32_t idZc = make_idesc_bf16(64, 16, 0, 0);
            const uint32_t w2 = smem_u32(smem + kOffW2), hk = smem_u32(smem + kOffHk), hq = smem_u32(smem + kOffHq);
            const uint32_t et = smem_u32(smem + kOffE), ae = smem_u32(smem + kOffAE), s2 = smem_u32(smem + kOffS2);
            bool ok = true;
            if (p.flags & TTT_FLAG_TEST_STALL) {
                if (!wait_bounded(stall, 0, lim, s_abort)) fail();
                ok = false;
            }
            auto W = [&](uint64_t* b, uint32_t par) {
                if (!wait_bounded(b, par, lim, s_abort)) {
                    fail();
                    ok = false;
                }
                return ok;
            };
            // S5 of batch i2: Z0^T = W2_i2^T Hq_i2^T + (-eta E_i2)^T tril(Hq Hk^T)^T
            auto issue_s5 = [&](int i2) {
                if (!W(hq_rdy, i2 & 1) || !W(aux2, i2 & 1)) return false;
                tc_fence_after();
                const uint32_t w2b = w2 + 32768 * (i2 & 1), hqb = hq + 8192 * (i2 & 1);
                for (int ks = 0; ks < 16; ++ks)
                    umma_bf16(tbase + cZ, make_sdesc(w2b + 2048 * ks, 1024, 1024, kSwizzle128B),
                              make_sdesc(hqb + 2048 * (ks >> 2) + 32 * (ks & 3), 16, 1024, kSwizzle128B), idS2,
                              ks > 0);
                umma_bf16(tbase + cZ, make_sdesc(ae + 2048 * (i2 & 1), 128, 256, kSwizzleNone),
                          make_sdesc(s2, 128, 256, kSwizzleNone), idZc, 1);
                umma_commit(d_z);
                return true;
            };
            for (int i = 0; ok && i < nsteps; ++i) {
                const int s = i % kStages;
                const uint32_t par = (i / kStages) & 1, ip = i & 1;
                const uint32_t st = smem_u32(smem + kOffStages + s * kStageBytes);
                // S1
                if (!W(&full[s], par) || !W(aw1_rdy, ip)) break;
                tc_fence_after();
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_ts(tbase + cA + 32 * tt, tbase + cAW1 + 32 * tt + 8 * ks,
                                make_sdesc(st + kOffK + 32 * ks, 16, 1024, kSwizzle128B), idS1, ks > 0);
                umma_commit(d_a);
                // the previous batch's output path runs while E1 of this batch does
                if (i >= 1 && !issue_s5(i - 1)) break;
                // (S2 and S3 run on the epilogue warps' mma.sync)
                // S4
                if (!W(d1_rdy, ip) || !W(&aux1[s], par)) break;
                tc_fence_after();
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    umma_ts(tbase + cW1 + 64 * tt, tbase + cAD1 + 8 * tt,
                            make_sdesc(st + kOffK, 1024, 1024, kSwizzle128B), idUpd, 1);
                    umma_ts(tbase + cA + 32 * tt + 16, tbase + cAD1 + 8 * tt,
                            make_sdesc(st + kOffS1, 128, 256, kSwizzleNone), idAq, 1);
                    umma_ts(tbase + cW2 + 64 * tt, tbase + cAHk + 8 * tt, make_sdesc(et, 1024, 1024, kSwizzle128B),
                            idUpd, 1);
                }
                umma_commit(d_u);
                umma_commit(&empty[s]);
            }
            if (ok && nsteps >= 1) issue_s5(nsteps - 1);
            umma_commit(drain);
            if (!wait_bounded(drain, 0, lim, nullptr)) fail();
        }
    } else if (warp == 6 || warp == 7) {
        // ------------------------------------------------------------ helpers
        const int hw = warp - 6;
        for (int i = 0; i < nsteps; ++i) {
            const int s = i % kStages;
            uint8_t* st = smem + kOffStages + s * kStageBytes;
            if (hw == 0) {
                // tril(Q K^T) of this batch (both n-tiles)
                if (!wait_bounded(&full[s], (i / kStages) & 1, lim, s_abort)) {
                    if (lane == 0) fail();
                    break;
                }
                // tril(Q K^T + 1): the "+1" carries the bias c1 updated token by token into Aq
                tril_product(smem_u32(st + kOffQ), smem_u32(st + kOffK), 1, 0, lane, st + kOffS1, 1.f);
                tril_product(smem_u32(st + kOffQ), smem_u32(st + kOffK), 1, 1, lane, st + kOffS1, 1.f);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&aux1[s]);
            }
            // tril(Hq Hk^T): n-tile hw
            if (!wait_bounded(hq_rdy, i & 1, lim, s_abort)) {
                if (lane == 0) fail();
                break;
            }
            // tril(Hq Hk^T + 1): the "+1" carries the bias c2 updated token by token
            tril_product(smem_u32(smem + kOffHq + 8192 * (i & 1)), smem_u32(smem + kOffHk + 8192 * (i & 1)), 4, hw,
                         lane, smem + kOffS2, 1.f);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(aux2);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Warps 0-3 and 8-11.  Warp w reads TMEM lane quadrant qd = w & 3 (hidden
        // rows h = 32 qd + lane of each 128-row tile) and takes the tokens of its
        // half hf = w >> 3 (8 hf .. 8 hf + 7) in every elementwise stage, and
        // the m16 x n8 tile (features 16 qd .., tokens of its half) in the
        // d-sized stages.
        const int qd = warp & 3, hf = warp >> 3;
        const int hr[2] = {32 * qd + lane, 128 + 32 * qd + lane};   // hidden rows of this thread
        const bool jl = lane < 16;                                  // M = 64 stages: feature row of this lane
        const int j = 16 * qd + (lane & 15);
        const int pu = p.per_seq ? unit : unit % p.H;
        const uint32_t tl = tbase + ((uint32_t)(32 * qd) << 16);
        uint8_t* w2s = smem + kOffW2;
        uint8_t* hks = smem + kOffHk;
        uint8_t* hqs = smem + kOffHq;
        uint8_t* es = smem + kOffE;
        uint8_t* aes = smem + kOffAE;
        float2* xch = reinterpret_cast<float2*>(smem + kOffXch);   // partial sums of the two token halves
        const int r = lane >> 2, c = lane & 3;   // accumulator layout: rows 16 qd + r (+8), tokens 8 hf + 2c (+1)
        // hidden rows in the accumulator layout: 128 tt + 32 qd + 16 m + r + 8 hh
        auto hrow = [&](int tt, int m, int hh) { return 128 * tt + 32 * qd + 16 * m + r + 8 * hh; };
        float c1[2][2][2], c2f[2] = {0.f, 0.f};  // c1 of rows hrow(tt, m, hh); c2 of rows 16 qd + r + 8 hh
        // LN: gamma, beta of rows 16 qd + r + 8 hh (accumulator layout) and of feature j (output
        // layout); the Q values of the finished mini-batch's output tokens 8 hf .. + 7 at feature j
        float lg[2] = {0.f, 0.f}, lb[2] = {0.f, 0.f}, lgz = 0.f, lbz = 0.f;
        uint32_t qz[4] = {0u, 0u, 0u, 0u};
        if (LN) {
            const int hd = unit % p.H;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                lg[hh] = p.gamma[(size_t)hd * kD + 16 * qd + r + 8 * hh];
                lb[hh] = p.beta[(size_t)hd * kD + 16 * qd + r + 8 * hh];
            }
            lgz = p.gamma[(size_t)hd * kD + j];
            lbz = p.beta[(size_t)hd * kD + j];
        }
        // bf16 [t][h] tile (four 128B-swizzled sub-tiles of 64 hidden rows) from the accumulator
        // layout: x[tt][m][hh] = pair of tokens (2c, 2c+1) of row hrow(tt, m, hh)
        auto stsm_rows = [&](uint32_t base, const uint32_t (&x)[2][2][2]) {
            const int t = 8 * hf + (lane & 7), mi = lane >> 3;
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                // matrix mi = 2 m + hh: hidden rows 128 tt + 32 qd + 16 m + 8 hh .. + 7
                const int h0 = 128 * tt + 32 * qd + 8 * mi;
                const uint32_t addr = base + 2048 * (h0 >> 6) + t * 128 + ((((h0 & 63) >> 3) ^ (t & 7)) << 4);
                stsm_x4_tr(addr, x[tt][0][0], x[tt][0][1], x[tt][1][0], x[tt][1][1]);
            }
        };
        // initial state: this warp writes columns 32 hf .. 32 hf + 31 of W1^T and W2
        {
            const float* W1u = p.W1 + (size_t)pu * kD * kM;
            const float* W2u = p.W2 + (size_t)pu * kM * kD;
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int h = hr[tt];
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        c1[tt][m][hh] = p.c1 ? p.c1[(size_t)pu * kM + hrow(tt, m, hh)] : 0.f;
                uint32_t w[32], pk[16];
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(W1u[(size_t)(32 * hf + i) * kM + h]);
                tmem_st_32x32b_x32(tl + cW1 + 64 * tt + 32 * hf, w);
#pragma unroll
                for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(__uint_as_float(w[2 * k]), __uint_as_float(w[2 * k + 1]));
                tmem_st_32x32b_x16(tl + cAW1 + 32 * tt + 16 * hf, pk);
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(W2u[(size_t)h * kD + 32 * hf + i]);
                tmem_st_32x32b_x32(tl + cW2 + 64 * tt + 32 * hf, w);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(w[8 * k + 0]), __uint_as_float(w[8 * k + 1]));
                    v.y = pack_bf16x2(__uint_as_float(w[8 * k + 2]), __uint_as_float(w[8 * k + 3]));
                    v.z = pack_bf16x2(__uint_as_float(w[8 * k + 4]), __uint_as_float(w[8 * k + 5]));
                    v.w = pack_bf16x2(__uint_as_float(w[8 * k + 6]), __uint_as_float(w[8 * k + 7]));
                    const int ch = 4 * hf + k;
                    *reinterpret_cast<uint4*>(w2s + (h >> 3) * 1024 + (h & 7) * 128 + ((ch ^ (h & 7)) << 4)) = v;
                }
            }
            if (p.c2) {
                c2f[0] = p.c2[(size_t)pu * kD + 16 * qd + r];
                c2f[1] = p.c2[(size_t)pu * kD + 16 * qd + r + 8];
            }
        }
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(aw1_rdy);
            mbar_arrive(w2_rdy);
        }
        bool dead = false;
        auto WT = [&](uint64_t* b, uint32_t par) {
            if (!dead && !wait_bounded(b, par, lim, s_abort)) {
                dead = true;
                fail();
            }
        };
        __nv_bfloat16* Zu = p.Z + (size_t)unit * p.T * kD + j;
        // bf16 W2 (state after batch i's update) -> buffer buf: this warp's 32 columns of row h
        auto refresh_w2 = [&](int buf) {
            uint8_t* dst = w2s + 32768 * buf;
            uint32_t w2r[2][32];   // both tiles' loads in flight before one wait
            tmem_ld_32x32b_x32(tl + cW2 + 32 * hf, w2r[0]);
            tmem_ld_32x32b_x32(tl + cW2 + 64 + 32 * hf, w2r[1]);
            tmem_wait_ld();
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int h = hr[tt];
                const uint32_t* w = w2r[tt];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(w[8 * k + 0]), __uint_as_float(w[8 * k + 1]));
                    v.y = pack_bf16x2(__uint_as_float(w[8 * k + 2]), __uint_as_float(w[8 * k + 3]));
                    v.z = pack_bf16x2(__uint_as_float(w[8 * k + 4]), __uint_as_float(w[8 * k + 5]));
                    v.w = pack_bf16x2(__uint_as_float(w[8 * k + 6]), __uint_as_float(w[8 * k + 7]));
                    const int ch = 4 * hf + k;
                    *reinterpret_cast<uint4*>(dst + (h >> 3) * 1024 + (h & 7) * 128 + ((ch ^ (h & 7)) << 4)) = v;
                }
            }
        };
        int nx = 0;   // exchanges of partial sums so far (two alternating buffers)
        // the other token half's partial sums of this warp's rows: a[k] += other's
        auto exchange2 = [&](float* a, int n) {
            float2* buf = xch + (nx & 1) * 1024;
            ++nx;
            for (int k = 0; k < n; k += 2) buf[(hf * 4 + qd) * 128 + (k >> 1) * 32 + lane] = make_float2(a[k], a[k + 1]);
            named_bar_sync(2, 256);
            for (int k = 0; k < n; k += 2) {
                const float2 o = buf[((1 - hf) * 4 + qd) * 128 + (k >> 1) * 32 + lane];
                a[k] += o.x;
                a[k + 1] += o.y;
            }
        };
        // LN: per-token sums over the 64 features (the four quadrant warps of this token half);
        // same buffers and barrier as exchange2, so every epilogue warp calls it at the same points.
        // Accumulator layout: v[tok][q] for the thread's tokens 2c, 2c+1 and two quantities.
        auto ln_sum_acc = [&](float (&v)[2][2]) {
#pragma unroll
            for (int o = 4; o < 32; o <<= 1)
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int b = 0; b < 2; ++b) v[a][b] += __shfl_xor_sync(0xffffffffu, v[a][b], o);
            float* buf = reinterpret_cast<float*>(xch + (nx & 1) * 1024);
            ++nx;
            if (lane < 4)
                *reinterpret_cast<float4*>(buf + ((hf * 4 + qd) * 4 + c) * 4) = make_float4(v[0][0], v[0][1], v[1][0], v[1][1]);
            named_bar_sync(2, 256);
            float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {
                const float4 x = *reinterpret_cast<const float4*>(buf + ((hf * 4 + w4) * 4 + c) * 4);
                t4.x += x.x; t4.y += x.y; t4.z += x.z; t4.w += x.w;
            }
            v[0][0] = t4.x; v[0][1] = t4.y; v[1][0] = t4.z; v[1][1] = t4.w;
        };
        // output layout (lane = feature j for lane < 16, tokens 8 hf + t): v[t][q], 16 values
        auto ln_sum_out = [&](float (&v)[8][2]) {
#pragma unroll
            for (int o = 1; o < 16; o <<= 1)
#pragma unroll
                for (int t = 0; t < 8; ++t)
#pragma unroll
                    for (int b = 0; b < 2; ++b) v[t][b] += __shfl_xor_sync(0xffffffffu, v[t][b], o);
            float* buf = reinterpret_cast<float*>(xch + (nx & 1) * 1024);
            ++nx;
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    *reinterpret_cast<float2*>(buf + (hf * 4 + qd) * 16 + 2 * t) = make_float2(v[t][0], v[t][1]);
            }
            named_bar_sync(2, 256);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                float a = 0.f, b = 0.f;
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4) {
                    const float2 x = *reinterpret_cast<const float2*>(buf + (hf * 4 + w4) * 16 + 2 * t);
                    a += x.x;
                    b += x.y;
                }
                v[t][0] = a;
                v[t][1] = b;
            }
        };
        float zc2 = 0.f;   // c2 of feature j before the batch's update (the Z bias; the updates
                           // within the batch are the "+1" of tril(Hq Hk^T + 1) in S5)
        // E5 of batch i2: Z = Z0 + c2 -> global, this warp's 8 tokens
        auto finish_z = [&](int i2, float zc) {
            WT(d_z, i2 & 1);
            tc_fence_after();
            uint32_t rz[8];
            tmem_ld_32x32b_x8(tl + cZ + 8 * hf, rz);
            tmem_wait_ld();
            float zv[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) zv[t] = __uint_as_float(rz[t]) + zc;
            if (LN) {
                // Z = Q + gamma LN(pre) + beta over the 64 features of each token
                float sm2[8][2];
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    sm2[t][0] = jl ? zv[t] : 0.f;
                    sm2[t][1] = jl ? zv[t] * zv[t] : 0.f;
                }
                ln_sum_out(sm2);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const float mu = sm2[t][0] * (1.f / kD);
                    const float rs = rsqrtf(fmaxf(sm2[t][1] * (1.f / kD) - mu * mu, 0.f) + p.eps);
                    const float q = (t & 1) ? bf16_hi(qz[t >> 1]) : bf16_lo(qz[t >> 1]);
                    zv[t] = q + lgz * (zv[t] - mu) * rs + lbz;
                }
            }
            if (jl && !dead) {
#pragma unroll
                for (int t = 0; t < 8; ++t) Zu[(size_t)(i2 * kTok + 8 * hf + t) * kD] = __float2bfloat16_rn(zv[t]);
            }
        };
        for (int i = 0; i < nsteps; ++i) {
            const int s = i % kStages;
            const uint32_t par = (i / kStages) & 1, ip = i & 1;
            const uint8_t* st = smem + kOffStages + s * kStageBytes;
            WT(&full[s], par);
            float et2[2];   // eta of tokens 8 hf + 2c, 8 hf + 2c + 1 (the accumulator columns)
            if (p.eta) {
                const float2 e0v = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(st + kOffEta) +
                                                                    8 * hf + 2 * c);
                et2[0] = e0v.x;
                et2[1] = e0v.y;
            } else {
                et2[0] = et2[1] = p.eta_const;
            }
            // E1: A -> Hk, GELU'(A), accumulator layout (m16 tiles (tt, m) of this quadrant,
            // the 8 tokens of this half)
            WT(d_a, ip);
            tc_fence_after();
            float gp[2][2][4];
            {
                uint32_t ra[2][2][4];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int m = 0; m < 2; ++m)
                        tmem_ld_16x256b_x1(tbase + ((uint32_t)(32 * qd + 16 * m) << 16) + cA + 32 * tt + 8 * hf, ra[tt][m]);
                tmem_wait_ld();
                uint32_t hkp[2][2][2];   // [tt][m][hh]: bf16 pairs of tokens (2c, 2c+1)
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        float hk[4], ah[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float a = __uint_as_float(ra[tt][m][e]) + c1[tt][m][e >> 1];
                            gelu_and_grad_fast(a, hk[e], gp[tt][m][e]);
                            ah[e] = -et2[e & 1] * hk[e];
                        }
                        hkp[tt][m][0] = pack_bf16x2(hk[0], hk[1]);
                        hkp[tt][m][1] = pack_bf16x2(hk[2], hk[3]);
                        tmem_st_16x128b_x1(tbase + ((uint32_t)(32 * qd + 16 * m) << 16) + cAHk + 8 * tt + 4 * hf,
                                           pack_bf16x2(ah[0], ah[1]), pack_bf16x2(ah[2], ah[3]));
                    }
                // Hk [t][h] in shared memory: matrices (tokens of this half, 8 hidden rows)
                stsm_rows(smem_u32(hks + 8192 * ip), hkp);
            }
            // S2 on the epilogue warps (mma.sync): E0^T = W2^T Hk^T over the 256 hidden
            // rows; this warp: features 16 qd .. 16 qd + 15, tokens of its half.  Every
            // warp's Hk must be in shared memory first.
            named_bar_sync(1, 256);
            float e0[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const int mi = lane >> 3;
                const uint32_t w2b = smem_u32(w2s + 32768 * ip), hkb = smem_u32(hks + 8192 * ip);
                const int arow = 8 * (mi >> 1) + (lane & 7);   // h within the k-step
                const int ach = 2 * qd + (mi & 1);             // 16-byte chunk of j
                const int brow = 8 * hf + (lane & 7);          // token t (lanes 0-15 give the addresses)
                // four independent accumulators (k-steps mod 4) keep the mma.sync chains short
                float acc[4][4] = {};
#pragma unroll
                for (int ks = 0; ks < 16; ++ks) {
                    uint32_t a[4], b[2];
                    const int h = 16 * ks + arow;
                    ldsm_x4_tr(w2b + (h >> 3) * 1024 + (h & 7) * 128 + ((ach ^ (h & 7)) << 4), a);
                    const int bch = 2 * (ks & 3) + ((lane >> 3) & 1);   // 16-byte chunk of h in its sub-tile
                    ldsm_x2(hkb + 2048 * (ks >> 2) + brow * 128 + ((bch ^ (brow & 7)) << 4), b);
                    mma_16816(acc[ks & 3], a, b[0], b[1]);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) e0[e] = (acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e]);
            }
            // E2: E = E0 + c2 - V -> E tile [t][j], (-eta E)^T [j][t]; c2 update
            {
                const int t8 = 8 * hf + (lane & 7);
                const uint32_t vt = smem_u32(st + kOffV);
                uint32_t v[2];
                ldsm_x2_tr(vt + t8 * 128 + (((2 * qd + ((lane >> 3) & 1)) ^ (t8 & 7)) << 4), v);
                const float etc[2] = {et2[0], et2[1]};
                float ev[4], ae[4];
                if (!LN) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) ev[e] = e0[e] + c2f[e >> 1] - frag_at(v, 0, e);
                } else {
                    // y = E0 + c2; f = k + gamma LN(y) + beta; ev becomes the LN+residual backward
                    uint32_t kv[2];
                    ldsm_x2_tr(smem_u32(st + kOffK) + t8 * 128 + (((2 * qd + ((lane >> 3) & 1)) ^ (t8 & 7)) << 4), kv);
                    float y[4], s1[2][2];
#pragma unroll
                    for (int e = 0; e < 4; ++e) y[e] = e0[e] + c2f[e >> 1];
#pragma unroll
                    for (int tk = 0; tk < 2; ++tk) {
                        s1[tk][0] = y[tk] + y[tk + 2];
                        s1[tk][1] = y[tk] * y[tk] + y[tk + 2] * y[tk + 2];
                    }
                    ln_sum_acc(s1);
                    float mu[2], rs[2], xh[4], g[4], s2[2][2];
#pragma unroll
                    for (int tk = 0; tk < 2; ++tk) {
                        mu[tk] = s1[tk][0] * (1.f / kD);
                        rs[tk] = rsqrtf(fmaxf(s1[tk][1] * (1.f / kD) - mu[tk] * mu[tk], 0.f) + p.eps);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tk = e & 1, hh = e >> 1;
                        xh[e] = (y[e] - mu[tk]) * rs[tk];
                        g[e] = lg[hh] * (frag_at(kv, 0, e) + lg[hh] * xh[e] + lb[hh] - frag_at(v, 0, e));
                    }
#pragma unroll
                    for (int tk = 0; tk < 2; ++tk) {
                        s2[tk][0] = g[tk] + g[tk + 2];
                        s2[tk][1] = g[tk] * xh[tk] + g[tk + 2] * xh[tk + 2];
                    }
                    ln_sum_acc(s2);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tk = e & 1;
                        ev[e] = rs[tk] * (g[e] - s2[tk][0] * (1.f / kD) - xh[e] * s2[tk][1] * (1.f / kD));
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) ae[e] = -etc[e & 1] * ev[e];
                stsm_x2_tr(smem_u32(es) + t8 * 128 + (((2 * qd + ((lane >> 3) & 1)) ^ (t8 & 7)) << 4),
                           pack_bf16x2(ev[0], ev[1]), pack_bf16x2(ev[2], ev[3]));
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    *reinterpret_cast<uint32_t*>(aes + 2048 * ip + nosw_off(16 * qd + r + 8 * hh, 8 * hf + 2 * c)) =
                        pack_bf16x2(ae[2 * hh], ae[2 * hh + 1]);
                // Z bias of this batch for finish_z's thread layout (feature 16 qd + (lane & 15))
                const int l15 = lane & 15;
                const float x0 = __shfl_sync(0xffffffffu, c2f[0], (l15 & 7) * 4);
                const float x1 = __shfl_sync(0xffffffffu, c2f[1], (l15 & 7) * 4);
                const float zc_now = l15 < 8 ? x0 : x1;
                // c2 += sum over the batch's 16 tokens of -eta e (this half, then the other's)
                float cs[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    cs[hh] = ae[2 * hh] + ae[2 * hh + 1];
                    cs[hh] += __shfl_xor_sync(0xffffffffu, cs[hh], 1);
                    cs[hh] += __shfl_xor_sync(0xffffffffu, cs[hh], 2);
                }
                exchange2(cs, 2);
                c2f[0] += cs[0];
                c2f[1] += cs[1];
                // the previous batch's outputs go out first (its bias is zc2), then keep this one's
                if (i >= 1) finish_z(i - 1, zc2);
                zc2 = zc_now;
                if (LN) {
                    // Q of this mini-batch at feature j, tokens 8 hf .. + 7 (for its output LN)
#pragma unroll
                    for (int t = 0; t < 8; t += 2) {
                        const float q0 = ld_bf16(st + kOffQ, sw128_off(8 * hf + t, j));
                        const float q1 = ld_bf16(st + kOffQ, sw128_off(8 * hf + t + 1, j));
                        qz[t >> 1] = pack_bf16x2(q0, q1);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // S3 on the epilogue warps (mma.sync): G^T = W2 E^T (K = 64) for this warp's four
            // m16 tiles of hidden rows and the tokens of its half; every warp's E first
            named_bar_sync(1, 256);
            float g[2][2][4] = {};
            {
                const int mi = lane >> 3;
                const uint32_t w2b = smem_u32(w2s + 32768 * ip), eb = smem_u32(es);
                const int t8 = 8 * hf + (lane & 7);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    uint32_t b[2];
                    ldsm_x2(eb + t8 * 128 + (((2 * ks + ((lane >> 3) & 1)) ^ (t8 & 7)) << 4), b);
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            uint32_t a[4];
                            const int h = 128 * tt + 32 * qd + 16 * m + (lane & 7) + 8 * (mi & 1);
                            const int jch = 2 * ks + (mi >> 1);
                            ldsm_x4(w2b + (h >> 3) * 1024 + (h & 7) * 128 + ((jch ^ (h & 7)) << 4), a);
                            mma_16816(g[tt][m], a, b[0], b[1]);
                        }
                }
            }
            // E3: D1 = G * GELU'(A) -> (-eta D1)^T; c1 update
            float c1_old[2][2][2];
            {
                float csum[8];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        float ad[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) ad[e] = -et2[e & 1] * g[tt][m][e] * gp[tt][m][e];
                        tmem_st_16x128b_x1(tbase + ((uint32_t)(32 * qd + 16 * m) << 16) + cAD1 + 8 * tt + 4 * hf,
                                           pack_bf16x2(ad[0], ad[1]), pack_bf16x2(ad[2], ad[3]));
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float cs = ad[2 * hh] + ad[2 * hh + 1];
                            cs += __shfl_xor_sync(0xffffffffu, cs, 1);
                            cs += __shfl_xor_sync(0xffffffffu, cs, 2);
                            csum[4 * tt + 2 * m + hh] = cs;
                        }
                    }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(d1_rdy);
                exchange2(csum, 8);
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            c1_old[tt][m][hh] = c1[tt][m][hh];
                            c1[tt][m][hh] += csum[4 * tt + 2 * m + hh];
                        }
            }
            // E4: bf16 W1^T for the next S1 first, then Hq = GELU(Aq + c1) -> Hq^T
            // (Aq carries the batch's bias updates through tril(Q K^T + 1)), then bf16 W2
            WT(d_u, ip);
            tc_fence_after();
            uint32_t rq[2][2][4];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                for (int m = 0; m < 2; ++m)
                    tmem_ld_16x256b_x1(tbase + ((uint32_t)(32 * qd + 16 * m) << 16) + cA + 32 * tt + 16 + 8 * hf, rq[tt][m]);
            {
                // both tiles' loads in flight before one wait
                uint32_t w[2][32];
                tmem_ld_32x32b_x32(tl + cW1 + 32 * hf, w[0]);
                tmem_ld_32x32b_x32(tl + cW1 + 64 + 32 * hf, w[1]);
                tmem_wait_ld();
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        pk[k] = pack_bf16x2(__uint_as_float(w[tt][2 * k]), __uint_as_float(w[tt][2 * k + 1]));
                    tmem_st_32x32b_x16(tl + cAW1 + 32 * tt + 16 * hf, pk);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(aw1_rdy);
            {
                uint32_t hqp[2][2][2];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        float hq[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            hq[e] = gelu_fast(__uint_as_float(rq[tt][m][e]) + c1_old[tt][m][e >> 1]);
                        hqp[tt][m][0] = pack_bf16x2(hq[0], hq[1]);
                        hqp[tt][m][1] = pack_bf16x2(hq[2], hq[3]);
                    }
                stsm_rows(smem_u32(hqs + 8192 * ip), hqp);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(hq_rdy);
            refresh_w2((i + 1) & 1);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(w2_rdy);
        }
        if (nsteps >= 1) finish_z(nsteps - 1, zc2);
        // final state (after the last S4; W1^T / W2 accumulators in TMEM): this warp's columns
        if (!dead) {
            float* W1o = p.W1_out + (size_t)unit * kD * kM;
            float* W2o = p.W2_out + (size_t)unit * kM * kD;
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int h = hr[tt];
                uint32_t w[32];
                tmem_ld_32x32b_x32(tl + cW1 + 64 * tt + 32 * hf, w);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) W1o[(size_t)(32 * hf + k) * kM + h] = __uint_as_float(w[k]);
                tmem_ld_32x32b_x32(tl + cW2 + 64 * tt + 32 * hf, w);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) W2o[(size_t)h * kD + 32 * hf + k] = __uint_as_float(w[k]);
            }
            if (p.c1_out && hf == 0 && c == 0) {
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) p.c1_out[(size_t)unit * kM + hrow(tt, m, hh)] = c1[tt][m][hh];
            }
            if (p.c2_out && c == 0 && hf == 0) {
                p.c2_out[(size_t)unit * kD + 16 * qd + r] = c2f[0];
                p.c2_out[(size_t)unit * kD + 16 * qd + r + 8] = c2f[1];
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

}  // namespace mtc
}  // namespace ttt
