// Fused prologue of the TTT layer: the three views of every token (paper
// digest "论文速览 | TTT", section 3.3, multi-view reconstruction) and the
// per-token learning-rate gate (section 4.6), from the layer input
// x [B*T, Dm] (bf16):
//     Q/K/V(token, h, j) = sum_k theta_{q/k/v}[h d + j, k] x(token, k)
//     eta(token, h)      = eta_base * sigmoid(sum_k theta_lr[h, k] x(token, k))
// as one dense contraction on the 5th-generation tensor cores (bf16
// operands, fp32 accumulation in tensor memory).
//
// Tiles: 128 tokens x up to 256 view columns (the gate tile: 128 tokens x H
// rounded up to 16), accumulated over the model width in 64-element
// (128-byte) chunks.  Persistent CTAs, one per SM, walk the tiles with the
// column-tile index fastest, so the CTAs that run together read the same x
// rows through L2 and the theta matrices stay L2-resident.
//
// Roles (192 threads):
//   warp 0     TMA producer: the x chunk (128 x 64) and the theta chunk
//              (up to 256 x 64), 128-byte swizzled, into a 4-stage ring.
//   warp 1     TMEM owner; one lane issues tcgen05.mma (M = 128, N <= 256,
//              K = 16) into one of two 256-column fp32 accumulators, so the
//              epilogue of a tile overlaps the main loop of the next.
//   warps 2-5  epilogue, TMEM lane quadrant warp % 4, one token per thread:
//              a view tile is rounded once to bf16 and written straight into
//              the [B, H, T, d] layout (16 features = 32 contiguous bytes per
//              store); the gate tile is finished in fp32.
// Every wait is bounded; an expired wait sets the status word and a shared
// abort flag, and each role drains what it has in flight before TMEM is
// released.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace ttt {
namespace pro {

constexpr int kBM = 128;   // tokens per tile (TMEM lanes)
constexpr int kBN = 256;   // view columns per tile (accumulator columns)
constexpr int kBK = 64;    // model-width chunk: one 128-byte swizzle row of bf16
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBN * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kOffBar = kStages * kStageBytes;
// full[S], empty[S], acc_full[2], acc_empty[2], drain, stall
constexpr int kNumBars = 2 * kStages + 6;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16;
constexpr uint32_t kTmemCols = 2 * kBN;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kABytes % 1024 == 0 && kStageBytes % 1024 == 0, "swizzled tiles must stay 1024-byte aligned");

struct PrologueParams {
    int rows;          // B * T tokens
    int T, H, d, Hd;   // Hd = H * d columns per view
    int nk;            // model-width chunks: ceil(Dm / 64)
    int nvt;           // column tiles per view: ceil(Hd / 256)
    int ntn;           // column tiles per token tile: 3 nvt, plus 1 with the gate
    long long tiles;   // ceil(rows / 128) * ntn
    int brows;         // rows of a view tile's theta box: min(256, Hd)
    int ng;            // columns of the gate tile: H rounded up to 16
    __nv_bfloat16* Q;
    __nv_bfloat16* K;
    __nv_bfloat16* V;
    float* eta;
    float eta_base;
    int* status;
    unsigned long long wait_ns;
    unsigned flags;
};

// The tile plan of one call (host side): everything in PrologueParams but the pointers.
inline void prologue_plan(PrologueParams& p, long long rows, int T, int H, int d, int Dm, bool gate) {
    const int Hd = H * d;
    p.rows = (int)rows;
    p.T = T;
    p.H = H;
    p.d = d;
    p.Hd = Hd;
    p.nk = (Dm + kBK - 1) / kBK;
    p.nvt = (Hd + kBN - 1) / kBN;
    p.ntn = 3 * p.nvt + (gate ? 1 : 0);
    p.tiles = ((rows + kBM - 1) / kBM) * p.ntn;
    p.brows = Hd < kBN ? Hd : kBN;
    p.ng = (H + 15) / 16 * 16;
}

struct Tile {
    int m0;     // first token
    int view;   // 0, 1, 2: Q, K, V; 3: the gate
    int c0;     // first column within the view
    int n;      // columns (MMA N): a multiple of 16, at most 256
};

__device__ __forceinline__ Tile decode_tile(const PrologueParams& p, long long tile) {
    Tile t;
    const long long mb = tile / p.ntn;
    const int nt = (int)(tile - mb * p.ntn);
    t.m0 = (int)(mb * kBM);
    if (nt < 3 * p.nvt) {
        t.view = nt / p.nvt;
        t.c0 = (nt - t.view * p.nvt) * kBN;
        t.n = min(kBN, p.Hd - t.c0);
    } else {
        t.view = 3;
        t.c0 = 0;
        t.n = p.ng;
    }
    return t;
}

// 16 accumulator columns (fp32 bits) -> 16 bf16 -> two 16-byte stores
__device__ __forceinline__ void store16_bf16(__nv_bfloat16* dst, const uint32_t* v) {
    uint4 w0, w1;
    w0.x = pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1]));
    w0.y = pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3]));
    w0.z = pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5]));
    w0.w = pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7]));
    w1.x = pack_bf16x2(__uint_as_float(v[8]), __uint_as_float(v[9]));
    w1.y = pack_bf16x2(__uint_as_float(v[10]), __uint_as_float(v[11]));
    w1.z = pack_bf16x2(__uint_as_float(v[12]), __uint_as_float(v[13]));
    w1.w = pack_bf16x2(__uint_as_float(v[14]), __uint_as_float(v[15]));
    uint4* d = reinterpret_cast<uint4*>(dst);
    d[0] = w0;
    d[1] = w1;
}

__global__ void __launch_bounds__(kThreads, 1)
    prologue_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmTq,
                    const __grid_constant__ CUtensorMap tmTk, const __grid_constant__ CUtensorMap tmTv,
                    const __grid_constant__ CUtensorMap tmTl, PrologueParams p) {
    // the dynamic buffer starts at the CTA's shared window (1024-aligned)
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicOr(p.status, kStatusBadSmem);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;                   // [kStages] TMA landed
    uint64_t* empty = bars + kStages;        // [kStages] stage consumed by the MMAs
    uint64_t* acc_full = bars + 2 * kStages; // [2] accumulator complete
    uint64_t* acc_empty = acc_full + 2;      // [2] accumulator read out: 4 epilogue warps
    uint64_t* drain = acc_empty + 2;         // final MMA drain
    uint64_t* stall = drain + 1;             // never arrived on (test hook)
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t lim = p.wait_ns;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(drain, 1);
        mbar_init(stall, 1);
        *s_abort = 0;
        fence_mbar_init();
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
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmTq);
            prefetch_tmap(&tmTk);
            prefetch_tmap(&tmTv);
            prefetch_tmap(&tmTl);
            long long it = 0, issued = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x) {
                const Tile tl = decode_tile(p, tile);
                const CUtensorMap* mb = tl.view == 0 ? &tmTq : tl.view == 1 ? &tmTk : tl.view == 2 ? &tmTv : &tmTl;
                const uint32_t bbytes = (uint32_t)(tl.view == 3 ? p.ng : p.brows) * (kBK * 2);
                for (int kc = 0; kc < p.nk; ++kc, ++it) {
                    const int s = (int)(it % kStages);
                    if (it >= kStages &&
                        !wait_bounded(&empty[s], (uint32_t)((it / kStages) - 1) & 1u, lim, s_abort)) {
                        fail();
                        ok = false;
                        break;
                    }
                    if (*s_abort) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * kStageBytes;
                    mbar_arrive_expect_tx(&full[s], kABytes + bbytes);
                    tma_load_2d(st, &tmX, kc * kBK, tl.m0, &full[s]);
                    tma_load_2d(st + kABytes, mb, kc * kBK, tl.c0, &full[s]);
                    issued = it + 1;
                }
            }
            // every issued load must land before the CTA exits (a TMA load
            // always completes, so these waits ignore the abort flag); the
            // last kStages chunks are the latest phase of their barriers
            for (long long g = issued - kStages; g < issued; ++g) {
                if (g < 0) continue;
                if (!wait_bounded(&full[g % kStages], (uint32_t)(g / kStages) & 1u, lim, nullptr)) fail();
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
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
            long long it = 0;
            int ai = 0;
            for (long long tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x, ++ai) {
                const Tile tl = decode_tile(p, tile);
                const int a = ai & 1;
                // the epilogue has read out the previous tile on this accumulator
                if (ai >= 2 && !W(&acc_empty[a], (uint32_t)((ai >> 1) - 1) & 1u)) break;
                tc_fence_after();
                const uint32_t dt = tbase + (uint32_t)(a * kBN);
                const uint32_t idesc = make_idesc_bf16(kBM, tl.n, 0, 0);
                for (int kc = 0; kc < p.nk; ++kc, ++it) {
                    const int s = (int)(it % kStages);
                    if (!W(&full[s], (uint32_t)(it / kStages) & 1u)) break;
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * kStageBytes), sb = sa + kABytes;
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ++ks)
                        umma_bf16(dt, make_sdesc(sa + 32 * ks, 16, 1024, kSwizzle128B),
                                  make_sdesc(sb + 32 * ks, 16, 1024, kSwizzle128B), idesc, (kc | ks) != 0);
                    umma_commit(&empty[s]);   // the stage is free once these MMAs complete
                }
                if (!ok) break;
                umma_commit(&acc_full[a]);
            }
            // drain every MMA issued so far before TMEM is released
            umma_commit(drain);
            if (!wait_bounded(drain, 0, lim, nullptr)) fail();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;   // TMEM lanes 32 q .. 32 q + 31
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int ai = 0;
        for (long long tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++ai) {
            const Tile tl = decode_tile(p, tile);
            const int a = ai & 1;
            // the warp leaves together: a lane that saw the wait expire takes the others with it, so the
            // warp-wide tcgen05.ld below never runs with part of the warp
            const bool got = wait_bounded(&acc_full[a], (uint32_t)(ai >> 1) & 1u, lim, s_abort);
            if (__any_sync(0xffffffffu, !got)) {
                if (lane == 0) fail();
                break;
            }
            tc_fence_after();
            const int r = tl.m0 + 32 * q + lane;
            const bool valid = r < p.rows;
            const int n = valid ? r / p.T : 0;
            const int t = valid ? r - n * p.T : 0;
            const uint32_t taddr = tbase + lane_base + (uint32_t)(a * kBN);
            if (tl.view < 3) {
                __nv_bfloat16* out = tl.view == 0 ? p.Q : tl.view == 1 ? p.K : p.V;
                // (n, h, t, j) of column c = c0 + cc: h = c / d, j = c % d; 16 | d, so a
                // 16-column group stays inside one head
                auto dst = [&](int cc) {
                    const int c = tl.c0 + cc;
                    const int h = c / p.d, j = c - h * p.d;
                    return out + (((size_t)n * p.H + h) * p.T + t) * p.d + j;
                };
                for (int cc = 0; cc < tl.n; cc += 32) {
                    uint32_t v[32];
                    if (tl.n - cc >= 32) {
                        tmem_ld_32x32b_x32(taddr + cc, v);
                        tmem_wait_ld();
                        if (valid) {
                            store16_bf16(dst(cc), v);
                            store16_bf16(dst(cc + 16), v + 16);
                        }
                    } else {
                        tmem_ld_32x32b_x16(taddr + cc, v);
                        tmem_wait_ld();
                        if (valid) store16_bf16(dst(cc), v);
                    }
                }
            } else {
                for (int cc = 0; cc < tl.n; cc += 16) {
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(taddr + cc, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int h = cc + i;
                        if (valid && h < p.H)
                            p.eta[((size_t)n * p.H + h) * p.T + t] =
                                p.eta_base / (1.f + expf(-__uint_as_float(v[i])));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

}  // namespace pro
}  // namespace ttt
