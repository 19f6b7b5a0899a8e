// Host emulation of the sm_100a asynchronous operations used by the tensor-core
// kernels (tc_emu_lfr.h adds the rest of what the TTT-Linear kernel uses), on
// top of emu_core.h: TEST INFRASTRUCTURE, never part of the library.
//
// Semantics (from the PTX ISA's descriptions):
//   mbarrier: an expected arrival count and a transaction count per phase; the
//     phase completes when both reach zero, then the next phase starts with the
//     initial arrival count.  try_wait.parity(P) succeeds once the phase with
//     parity P has completed, i.e. when the current phase's parity differs from P.
//   cp.async.bulk.tensor (2-D tile, 128-byte swizzle): the box is copied to
//     shared memory with the 16-byte chunk c of row r stored at chunk c ^ (r % 8);
//     elements outside the tensor are zero; the whole box's bytes count toward
//     the mbarrier's transaction count.
//   tcgen05.mma kind::f16 (bf16 x bf16 -> f32), K = 16, operands in shared
//     memory (K-major or MN-major with the 128-byte swizzle, K-major without
//     swizzle: the addressing is given at operand_elem below) or A in tensor
//     memory.  D (M x N) is at TMEM lanes 0 .. M-1, columns col .. col + N - 1.
//   tcgen05.ld .32x32b.xN: lane t of the warp reads TMEM lane (base + t),
//     columns col .. col + N - 1; a warp may access the 32 lanes of its
//     quadrant (warp % 4) only.
//   tcgen05.commit: arrives once on the mbarrier when the MMAs issued before it
//     have completed.
// Asynchronous operations complete when they are issued (one of the schedules
// the hardware may produce, which a correct kernel must handle), or, in the
// deferred mode (emu::deferred), later, on an engine thread (see Engine).
#pragma once
#include <atomic>
#include <chrono>
#include <condition_variable>
#include <cuda.h>
#include <deque>
#include <functional>
#include <map>
#include <vector>
#include <mutex>
#include <thread>

#include "emu_core.h"

namespace emu {
struct Bar {
    int count = 0, pending = 0;
    long long tx = 0;
    unsigned phase = 0;
};
inline std::mutex bar_mu;
inline std::map<const void*, Bar> bars;
inline uint32_t tmem[128][512];
inline std::atomic<int> errors{0};   // emulated-hardware rule violations (quadrant, layout)

// what the harness puts in a CUtensorMap
struct FakeMap {
    const void* base;
    unsigned long long cols, rows, pitch;   // elements, elements, bytes
    unsigned box_cols, box_rows, elem;      // elements, elements, bytes per element
    int swizzle128;
};
static_assert(sizeof(FakeMap) <= sizeof(CUtensorMap), "tensor map space");
inline void make_map(CUtensorMap* m, const void* base, unsigned long long cols, unsigned long long rows,
                     unsigned long long pitch, unsigned box_cols, unsigned box_rows, unsigned elem) {
    std::memset(m, 0, sizeof(*m));
    FakeMap f{base, cols, rows, pitch, box_cols, box_rows, elem, 1};
    std::memcpy(m, &f, sizeof(f));
}

inline void complete_if_done(Bar& b) {
    if (b.pending == 0 && b.tx == 0) {
        ++b.phase;
        b.pending = b.count;
    }
}
inline void bar_arrive(const void* bar, long long tx_add) {
    std::lock_guard<std::mutex> lk(bar_mu);
    Bar& b = bars[bar];
    b.tx += tx_add;
    --b.pending;
    complete_if_done(b);
}
inline void bar_complete_tx(const void* bar, long long bytes) {
    std::lock_guard<std::mutex> lk(bar_mu);
    Bar& b = bars[bar];
    b.tx -= bytes;
    complete_if_done(b);
}
inline uint32_t tmem_lane(uint32_t a) { return a >> 16; }
inline uint32_t tmem_col(uint32_t a) { return a & 0xFFFFu; }

// Deferred completion (off by default): TMA and bulk loads, MMAs and commits
// go to two FIFOs that one engine thread works through, each job after a
// pause: loads first (they may overtake MMAs: the copy engine and the tensor
// core are separate units), MMAs and commits in issue order, as tcgen05
// guarantees for one issuing thread, so a commit arrives once the MMAs before
// it have run.  A kernel that touches a buffer before the wait that orders
// it, or reuses one too early, then sees stale or overwritten data.
// pending_stores counts each thread's TMA stores not yet done.
struct Engine {
    std::mutex mu;
    std::condition_variable cv;
    std::deque<std::function<void()>> q[2];   // 0: loads, 1: MMAs and commits
    std::thread th;
    bool started = false, quit = false;
    std::atomic<long> inflight{0};
    void run() {
        for (;;) {
            std::function<void()> job;
            {
                std::unique_lock<std::mutex> lk(mu);
                cv.wait(lk, [&] { return !q[0].empty() || !q[1].empty() || quit; });
                if (q[0].empty() && q[1].empty()) return;
                auto& src = q[0].empty() ? q[1] : q[0];
                job = std::move(src.front());
                src.pop_front();
            }
            std::this_thread::sleep_for(std::chrono::microseconds(30));
            job();
            --inflight;
        }
    }
    void push(std::function<void()> job, int kind) {
        std::lock_guard<std::mutex> lk(mu);
        if (!started) {
            quit = false;
            th = std::thread([this] { run(); });
            started = true;
        }
        ++inflight;
        q[kind].push_back(std::move(job));
        cv.notify_one();
    }
    // wait for the queues to empty, then end the engine thread (a harness call's last step, so that no
    // thread waits on the condition variable when the library is unloaded)
    void finish() {
        while (inflight.load() != 0) std::this_thread::yield();
        {
            std::lock_guard<std::mutex> lk(mu);
            if (!started) return;
            quit = true;
        }
        cv.notify_all();
        th.join();
        started = false;
    }
};
inline Engine engine;
inline std::atomic<bool> deferred{false};
inline std::atomic<int> pending_stores[kMaxThreads];
// In the deferred mode a TMA store is held until its thread waits for it
// (cp.async.bulk.wait_group), the latest point at which it may read shared
// memory; a store never waited for is done when the run ends, after later
// CTAs have reused the shared memory.
inline std::vector<std::function<void()>> held_stores[kMaxThreads];
inline void flush_stores(int tid) {
    for (auto& job : held_stores[tid]) job();
    held_stores[tid].clear();
}
// Deferred tensor-memory loads and stores: a tcgen05.ld reads tensor memory
// at issue, but its registers hold NaN until the thread's tcgen05.wait::ld; a
// tcgen05.st reaches tensor memory at the thread's tcgen05.wait::st (a store
// never waited for is lost).
struct TmemLd {
    uint32_t* dst;
    std::vector<uint32_t> vals;
};
struct TmemSt {
    uint32_t lane, col, val;
};
inline thread_local std::vector<TmemLd> pend_ld;
inline thread_local std::vector<TmemSt> pend_st;
inline void deliver(uint32_t* r, const uint32_t* vals, int n) {
    if (deferred.load()) {
        pend_ld.push_back({r, std::vector<uint32_t>(vals, vals + n)});
        for (int i = 0; i < n; ++i) r[i] = 0x7FC00000u;
    } else {
        for (int i = 0; i < n; ++i) r[i] = vals[i];
    }
}
inline void tmem_put(uint32_t lane, uint32_t col, uint32_t val) {
    if (deferred.load())
        pend_st.push_back({lane & 127, col & 511, val});
    else
        tmem[lane & 127][col & 511] = val;
}
enum { kLoad = 0, kMma = 1 };
inline void async_do(std::function<void()> job, int kind) {
    if (deferred.load())
        engine.push(std::move(job), kind);
    else
        job();
}
}  // namespace emu

#undef __grid_constant__
#define __grid_constant__
inline float __uint_as_float(uint32_t v) {
    float f;
    std::memcpy(&f, &v, 4);
    return f;
}
inline int atomicOr(int* p, int v) { return __atomic_fetch_or(p, v, __ATOMIC_SEQ_CST); }
inline void __syncwarp(unsigned = 0xffffffffu) { emu::warp_sync(); }

namespace ttt {
inline void mbar_init(uint64_t* bar, uint32_t count) {
    std::lock_guard<std::mutex> lk(emu::bar_mu);
    emu::Bar& b = emu::bars[bar];
    b.count = b.pending = (int)count;
    b.tx = 0;
    b.phase = 0;
}
inline void fence_mbar_init() {}
inline void mbar_arrive(uint64_t* bar) { emu::bar_arrive(bar, 0); }
inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) { emu::bar_arrive(bar, bytes); }
inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    std::lock_guard<std::mutex> lk(emu::bar_mu);
    return (emu::bars[bar].phase & 1u) != (parity & 1u);
}
inline uint64_t globaltimer_ns() {
    return (uint64_t)std::chrono::duration_cast<std::chrono::nanoseconds>(
               std::chrono::steady_clock::now().time_since_epoch())
        .count();
}
inline bool wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns, volatile int* abort) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort && *abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) return false;
        emu::spin_yield();
    }
}
inline void fence_proxy_async_smem() {}
inline void prefetch_tmap(const CUtensorMap*) {}
// 2-D tiled load, 128-byte swizzle, out-of-range elements zero
inline void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    emu::FakeMap f;
    std::memcpy(&f, map, sizeof(f));
    uint8_t* d = static_cast<uint8_t*>(dst);
    const unsigned rowb = f.box_cols * f.elem;
    if (((uintptr_t)(d - emu::shared_base)) % 1024 != 0 || rowb != 128 || (x * f.elem) % 16 != 0) ++emu::errors;
    emu::async_do([=] {
        for (unsigned r = 0; r < f.box_rows; ++r)
            for (unsigned cb = 0; cb < rowb; ++cb) {
                const long long gx = (long long)x + cb / f.elem, gy = (long long)y + r;
                uint8_t v = 0;
                if (gx >= 0 && gy >= 0 && (unsigned long long)gx < f.cols && (unsigned long long)gy < f.rows)
                    v = static_cast<const uint8_t*>(f.base)[gy * f.pitch + gx * f.elem + cb % f.elem];
                const unsigned chunk = (cb >> 4) ^ (r & 7);
                d[r * 128 + chunk * 16 + (cb & 15)] = v;
            }
        emu::bar_complete_tx(bar, (long long)rowb * f.box_rows);
    }, emu::kLoad);
}
inline void tmem_alloc(uint32_t* dst, uint32_t) { *dst = 0; }
inline void tmem_relinquish() {}
inline void tmem_dealloc(uint32_t, uint32_t) {}
inline void tc_fence_before() {}
inline void tc_fence_after() {}
inline void tmem_wait_ld() {
    for (auto& l : emu::pend_ld) std::memcpy(l.dst, l.vals.data(), l.vals.size() * 4);
    emu::pend_ld.clear();
}
inline void tmem_wait_st() {
    for (auto& t : emu::pend_st) emu::tmem[t.lane][t.col] = t.val;
    emu::pend_st.clear();
}
template <int N>
inline void tmem_ld_32x32b(uint32_t taddr, uint32_t* r) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const uint32_t l0 = emu::tmem_lane(taddr), c0 = emu::tmem_col(taddr);
    if (l0 / 32 != (uint32_t)(w % 4) || l0 % 32 != 0 || c0 + N > 512) ++emu::errors;
    uint32_t vals[N];
    for (int i = 0; i < N; ++i) vals[i] = emu::tmem[(l0 + lane) & 127][(c0 + i) & 511];
    emu::deliver(r, vals, N);
    emu::warp_sync();
}
inline void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* r) { tmem_ld_32x32b<16>(taddr, r); }
inline void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t* r) { tmem_ld_32x32b<32>(taddr, r); }

// The descriptors are the library's own encoding (make_sdesc, make_idesc_bf16 in ptx.cuh): start address,
// leading (LBO) and stride (SBO) byte offsets, and the layout code (2: 128-byte swizzle, 0: none).
// Element (mn, k) of a bf16 operand, mn the M or N index:
//   K-major, 128-byte swizzle:  start + (mn / 8) SBO + (mn % 8) 128 + 2 k, address bits 4-6 ^= bits 7-9
//   MN-major, 128-byte swizzle: start + (k / 8) SBO + (mn / 64) LBO + (k % 8) 128 + 2 (mn % 64), same XOR
//   K-major, no swizzle (8 x 16-byte core matrices): start + (mn / 8) SBO + (k / 8) LBO + (mn % 8) 16 + 2 (k % 8)
inline float operand_elem(uint64_t desc, bool mn_major, int mn, int k) {
    const uint32_t start = (uint32_t)(desc & 0x3FFFu) << 4;
    const uint32_t lbo = (uint32_t)((desc >> 16) & 0x3FFFu) << 4;
    const uint32_t sbo = (uint32_t)((desc >> 32) & 0x3FFFu) << 4;
    const uint32_t layout = (uint32_t)(desc >> 61);
    uint32_t phys = 0;
    if (layout == 2u) {
        const uint32_t lin = mn_major ? start + (k / 8) * sbo + (mn / 64) * lbo + (k % 8) * 128 + 2 * (mn % 64)
                                      : start + (mn / 8) * sbo + (mn % 8) * 128 + 2 * k;
        phys = lin ^ (((lin >> 7) & 7u) << 4);
    } else if (layout == 0u && !mn_major) {
        phys = start + (mn / 8) * sbo + (k / 8) * lbo + (mn % 8) * 16 + 2 * (k % 8);
    } else {
        ++emu::errors;
    }
    const uint16_t h = emu::ld16(phys);
    uint32_t b = (uint32_t)h << 16;
    float f;
    std::memcpy(&f, &b, 4);
    return f;
}
// D (M x N, fp32) (+)= A B^T over K = 16; a(row, k) and b(col, k) give the operands.  M = 128: row i of D
// at TMEM lane (lane + i); M = 64: rows 16 q .. 16 q + 15 at lanes 32 q + (lane + 0 .. 15) of quadrant q
template <typename FA, typename FB>
inline void umma_apply(uint32_t d_tmem, uint32_t idesc, uint32_t accumulate, FA a, FB b) {
    const int M = (int)((idesc >> 24) & 0x1Fu) << 4, N = (int)((idesc >> 17) & 0x3Fu) << 3;
    if (M == 128 ? (N % 16 != 0 || N < 16 || N > 256) : M == 64 ? (N % 8 != 0 || N < 8 || N > 256) : true)
        ++emu::errors;
    if (M == 64 && emu::tmem_lane(d_tmem) % 32 + 16 > 32) ++emu::errors;
    const uint32_t l0 = emu::tmem_lane(d_tmem), c0 = emu::tmem_col(d_tmem);
    float av[128][16];
    for (int row = 0; row < M; ++row)
        for (int k = 0; k < 16; ++k) av[row][k] = a(row, k);
    for (int col = 0; col < N; ++col) {
        float bv[16];
        for (int k = 0; k < 16; ++k) bv[k] = b(col, k);
        for (int row = 0; row < M; ++row) {
            float acc = 0.f;
            for (int k = 0; k < 16; ++k) acc += av[row][k] * bv[k];
            const uint32_t dl = M == 64 ? l0 + 32 * (row / 16) + row % 16 : l0 + row;
            uint32_t& cell = emu::tmem[dl & 127][(c0 + col) & 511];
            float prev;
            std::memcpy(&prev, &cell, 4);
            const float v = (accumulate ? prev : 0.f) + acc;
            std::memcpy(&cell, &v, 4);
        }
    }
}
inline void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    emu::async_do([=] {
        const bool a_mn = (idesc >> 15) & 1u, b_mn = (idesc >> 16) & 1u;
        umma_apply(
            d_tmem, idesc, accumulate, [&](int row, int k) { return operand_elem(adesc, a_mn, row, k); },
            [&](int col, int k) { return operand_elem(bdesc, b_mn, col, k); });
    }, emu::kMma);
}
// A in tensor memory: element (row, k) at lane (lane + row), column (col + k / 2), the low half for even k
inline float tmem_bf16(uint32_t a_tmem, int row, int k) {
    const uint32_t v = emu::tmem[(emu::tmem_lane(a_tmem) + row) & 127][(emu::tmem_col(a_tmem) + k / 2) & 511];
    return (k & 1) ? emu::bf16_hi(v) : emu::bf16_lo(v);
}
inline void umma_commit(uint64_t* bar) {
    emu::async_do([=] { emu::bar_arrive(bar, 0); }, emu::kMma);
}
}  // namespace ttt
