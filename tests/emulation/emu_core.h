// Host emulation of the CUDA execution model for the CPU tests: TEST
// INFRASTRUCTURE, never part of the library (which has no CPU path).
//
// One CTA at a time.  Each CUDA thread of the CTA is a std::thread running
// the kernel function; __syncthreads is a barrier over the CTA (EBar: all
// threads concurrent, or one at a time under the serial scheduler); a
// warp-collective operation (shuffle, ldmatrix, mma) has every lane write its
// operands to the warp's exchange area, waits on the warp's barrier, computes
// its own result from all lanes' operands, and waits again before the area is
// reused.  Shared memory is one static buffer per kernel family; its
// shared-window addresses are byte offsets from that buffer.
//
// The warp-collective semantics follow the PTX ISA's documented layouts:
//   ldmatrix .m8n8.x4 .b16: lanes 8i .. 8i+7 give the row addresses of matrix
//     i; lane L receives in register i the elements (L/4, 2(L%4)) and
//     (L/4, 2(L%4)+1) of matrix i; with .trans, the elements (2(L%4), L/4) and
//     (2(L%4)+1, L/4).  The first element is the low half.
//   mma .m16n8k16 .row.col, bf16 -> f32, with g = L/4, c = L%4:
//     A (16 x 16): a0 = A[g][2c..2c+1], a1 = A[g+8][2c..], a2 = A[g][2c+8..],
//                  a3 = A[g+8][2c+8..]
//     B (16 x 8):  b0 = B[2c..2c+1][g], b1 = B[2c+8..2c+9][g]
//     C, D (16 x 8, f32): d0 = D[g][2c], d1 = D[g][2c+1], d2 = D[g+8][2c],
//                  d3 = D[g+8][2c+1]
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <atomic>
#include <barrier>
#include <cmath>
#include <condition_variable>
#include <mutex>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace emu {
constexpr int kMaxThreads = 1024;
inline thread_local uint3 tid3, bid3;
inline uint3 grid3;

// Serial mode (off by default; 1: lowest thread first, 2: highest first).
// One thread of the CTA runs at a time and hands the CPU on only where it
// blocks (a barrier not yet complete, a warp collective) or spins (a wait on
// an mbarrier or a store).  At a block the next thread is the ready one of
// lowest (1) or highest (2) index, so the first warp runs as far as it can,
// to its next block-wide barrier, before the others move; a spinning thread
// hands on round-robin and runs again only when no thread that is not
// spinning is ready.  A read of data another thread writes without a
// barrier between them, or a write into data others still read, then shows
// as wrong data in one of the two orders.
inline std::atomic<int> serial{0};
struct Sched {
    std::mutex m;
    std::condition_variable cv[kMaxThreads];   // one per thread: a hand-off wakes only the new owner
    int n = 0, owner = -1;
    bool ready[kMaxThreads];
    bool spinning[kMaxThreads];   // last handed on from a spin-wait: runs only when no other thread is ready
    bool stuck = false;   // every live thread blocked on a barrier: the kernel would hang
};
inline Sched sched;
// the next ready thread after `from`, round-robin (itself last), or -1 (lock held)
inline int sched_next_rr(int from) {
    const int n = sched.n;
    for (int i = 1; i <= n; ++i) {
        const int t = (from + i) % n;
        if (sched.ready[t]) return t;
    }
    return -1;
}
// the ready thread of lowest (1) or highest (2) index that is not spinning, else the next spinner
// round-robin, or -1 (lock held)
inline int sched_next(int from) {
    const int n = sched.n;
    for (int i = 0; i < n; ++i) {
        const int t = serial.load() == 1 ? i : n - 1 - i;
        if (sched.ready[t] && !sched.spinning[t]) return t;
    }
    return sched_next_rr(from);
}
// hand the CPU on (lock held) and wait until it comes back
inline void sched_wake() {
    if (sched.stuck)
        for (int t = 0; t < sched.n; ++t) sched.cv[t].notify_all();
    else if (sched.owner >= 0)
        sched.cv[sched.owner].notify_all();
}
inline void sched_handoff(std::unique_lock<std::mutex>& lk, int tid, bool rr = false) {
    sched.owner = rr ? sched_next_rr(tid) : sched_next(tid);
    if (sched.owner < 0) sched.stuck = true;
    if (sched.owner != tid) {
        sched_wake();
        sched.cv[tid].wait(lk, [&] { return sched.owner == tid || sched.stuck; });
    }
}
// a spin-wait iteration: stay ready, let the others run first
inline void spin_yield() {
    if (!serial.load()) {
        std::this_thread::yield();
        return;
    }
    const int tid = (int)tid3.x;
    std::unique_lock<std::mutex> lk(sched.m);
    sched.ready[tid] = true;
    sched.spinning[tid] = true;
    sched_handoff(lk, tid, true);
}

// A barrier over `count` threads: std::barrier, or in the serial mode the
// scheduler's own.
struct EBar {
    std::barrier<> b;
    int count, arrived = 0;
    long gen = 0;
    explicit EBar(int c) : b(c), count(c) {}
    void wait() {
        if (!serial.load()) {
            b.arrive_and_wait();
            return;
        }
        const int tid = (int)tid3.x;
        std::unique_lock<std::mutex> lk(sched.m);
        sched.spinning[tid] = false;
        if (++arrived == count) {
            arrived = 0;
            ++gen;
            for (int t = 0; t < sched.n; ++t)
                if (waiting_on[t] == this) {
                    waiting_on[t] = nullptr;
                    sched.ready[t] = true;
                }
            sched.ready[tid] = true;   // the last arriver waits its turn like the others
            sched_handoff(lk, tid);
            return;
        }
        waiting_on[tid] = this;
        sched.ready[tid] = false;
        sched_handoff(lk, tid);
    }
    static inline EBar* waiting_on[kMaxThreads];
};
inline EBar* block_bar = nullptr;
inline EBar* warp_bar[kMaxThreads / 32];
inline const uint8_t* shared_base = nullptr;
struct WarpXch {
    float f[32];
    uint32_t u[32][4];
    uint32_t v[32][2];
    float c[32][4];
};
inline WarpXch xch[kMaxThreads / 32];
inline std::atomic<int> sched_errors{0};   // serial runs that found every thread blocked

inline void warp_sync() { warp_bar[tid3.x >> 5]->wait(); }

// Shared-memory guard: with run_grid_bounded, the buffer beyond the launch's
// dynamic size is filled with a pattern before each CTA and checked after
// it; a changed byte counts as an overrun (on the GPU, an access outside the
// CTA's allocation).
inline std::atomic<int> smem_overruns{0};
inline size_t guard_bytes = 0, guard_cap = 0;
constexpr uint8_t kGuard = 0xA5;

template <typename F>
void run_grid(int blocks, int threads, const void* shared, F f) {
    shared_base = static_cast<const uint8_t*>(shared);
    grid3 = make_uint3(blocks, 1, 1);
    for (int bx = 0; bx < blocks; ++bx) {
        EBar bb(threads);
        for (int w = 0; w < threads / 32; ++w) warp_bar[w] = new EBar(32);
        block_bar = &bb;
        {
            std::lock_guard<std::mutex> lk(sched.m);
            sched.n = threads;
            sched.stuck = false;
            for (int t = 0; t < threads; ++t) {
                sched.ready[t] = true;
                sched.spinning[t] = false;
                EBar::waiting_on[t] = nullptr;
            }
            sched.owner = serial.load() == 2 ? threads - 1 : 0;
        }
        uint8_t* guard = const_cast<uint8_t*>(shared_base) + guard_bytes;
        if (guard_cap > guard_bytes) std::memset(guard, kGuard, guard_cap - guard_bytes);
        std::vector<std::thread> th;
        th.reserve(threads);
        for (int t = 0; t < threads; ++t)
            th.emplace_back([&, t, bx] {
                tid3 = make_uint3(t, 0, 0);
                bid3 = make_uint3(bx, 0, 0);
                if (serial.load()) {
                    std::unique_lock<std::mutex> lk(sched.m);
                    sched.cv[t].wait(lk, [&] { return sched.owner == t || sched.stuck; });
                }
                if (!sched.stuck) f();
                if (serial.load()) {
                    std::unique_lock<std::mutex> lk(sched.m);
                    sched.ready[t] = false;
                    if (sched.owner == t) {
                        sched.owner = sched_next(t);
                        bool live = false;
                        for (int u = 0; u < sched.n; ++u) live = live || EBar::waiting_on[u] != nullptr;
                        if (sched.owner < 0 && live) sched.stuck = true;
                        sched_wake();
                    }
                }
            });
        for (auto& x : th) x.join();
        if (sched.stuck) ++sched_errors;
        for (size_t i = 0; guard_cap > guard_bytes && i < guard_cap - guard_bytes; ++i)
            if (guard[i] != kGuard) {
                ++smem_overruns;
                break;
            }
        for (int w = 0; w < threads / 32; ++w) delete warp_bar[w];
    }
}

// run_grid with the shared-memory guard: `bytes` is the launch's dynamic size, `cap` the buffer's
template <typename F>
void run_grid_bounded(int blocks, int threads, void* shared, size_t bytes, size_t cap, F f) {
    if (bytes > cap) {
        ++smem_overruns;
        return;
    }
    guard_bytes = bytes;
    guard_cap = cap;
    run_grid(blocks, threads, shared, f);
    guard_bytes = guard_cap = 0;
}

inline float bf16_lo(uint32_t v) {
    uint32_t b = v << 16;
    float f;
    std::memcpy(&f, &b, 4);
    return f;
}
inline float bf16_hi(uint32_t v) {
    uint32_t b = v & 0xFFFF0000u;
    float f;
    std::memcpy(&f, &b, 4);
    return f;
}
inline uint16_t ld16(uint32_t saddr) {
    uint16_t h;
    std::memcpy(&h, shared_base + saddr, 2);
    return h;
}
}  // namespace emu

#undef threadIdx
#undef blockIdx
#undef gridDim
#define threadIdx emu::tid3
#define blockIdx emu::bid3
#define gridDim emu::grid3
inline void __syncthreads() { emu::block_bar->wait(); }
inline float __shfl_xor_sync(unsigned, float v, int o) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    emu::xch[w].f[lane] = v;
    emu::warp_sync();
    const float r = emu::xch[w].f[lane ^ o];
    emu::warp_sync();
    return r;
}
inline float __shfl_sync(unsigned, float v, int src) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    emu::xch[w].f[lane] = v;
    emu::warp_sync();
    const float r = emu::xch[w].f[src & 31];
    emu::warp_sync();
    return r;
}
inline int __any_sync(unsigned, int pred) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    emu::xch[w].f[lane] = pred ? 1.f : 0.f;
    emu::warp_sync();
    int any = 0;
    for (int i = 0; i < 32; ++i) any |= emu::xch[w].f[i] != 0.f;
    emu::warp_sync();
    return any;
}
inline float rsqrtf(float x) { return 1.0f / std::sqrt(x); }
inline int min(int a, int b) { return a < b ? a : b; }
inline int max(int a, int b) { return a > b ? a : b; }
inline float __expf(float x) { return std::exp(x); }
inline float __fdividef(float a, float b) { return a / b; }
#define __launch_bounds__(...)
#undef __shared__
#define __shared__
#define TTT_HOST_EMULATION 1

namespace ttt {
inline uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(static_cast<const uint8_t*>(p) - emu::shared_base);
}
namespace mbk {
// ldmatrix .m8n8.x4 (.trans when T)
template <bool T>
inline void ldsm_emu(uint32_t addr, uint32_t* r) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    emu::xch[w].u[lane][0] = addr;
    emu::warp_sync();
    for (int i = 0; i < 4; ++i) {
        uint16_t lo, hi;
        if (!T) {
            const uint32_t row = emu::xch[w].u[8 * i + lane / 4][0];
            lo = emu::ld16(row + 4 * (lane % 4));
            hi = emu::ld16(row + 4 * (lane % 4) + 2);
        } else {
            const uint32_t r0 = emu::xch[w].u[8 * i + 2 * (lane % 4)][0];
            const uint32_t r1 = emu::xch[w].u[8 * i + 2 * (lane % 4) + 1][0];
            lo = emu::ld16(r0 + 2 * (lane / 4));
            hi = emu::ld16(r1 + 2 * (lane / 4));
        }
        r[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    emu::warp_sync();
}
inline void ldsm4(uint32_t addr, uint32_t* r) { ldsm_emu<false>(addr, r); }
inline void ldsm4t(uint32_t addr, uint32_t* r) { ldsm_emu<true>(addr, r); }
// mma.m16n8k16.row.col.f32.bf16.bf16.f32, d += a b
inline void mma(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    auto& x = emu::xch[w];
    for (int i = 0; i < 4; ++i) x.u[lane][i] = a[i];
    x.v[lane][0] = b0;
    x.v[lane][1] = b1;
    emu::warp_sync();
    auto A = [&](int row, int k) {   // element of the 16 x 16 A
        const int g = row & 7, hr = row >> 3, c = (k & 7) >> 1, hk = k >> 3;
        const uint32_t v = x.u[4 * g + c][hr + 2 * hk];
        return (k & 1) ? emu::bf16_hi(v) : emu::bf16_lo(v);
    };
    auto B = [&](int k, int col) {   // element of the 16 x 8 B
        const int c = (k & 7) >> 1, hk = k >> 3;
        const uint32_t v = x.v[4 * col + c][hk];
        return (k & 1) ? emu::bf16_hi(v) : emu::bf16_lo(v);
    };
    const int g = lane / 4, c = lane % 4;
    for (int e = 0; e < 4; ++e) {
        const int row = g + 8 * (e >> 1), col = 2 * c + (e & 1);
        float acc = 0.f;
        for (int k = 0; k < 16; ++k) acc += A(row, k) * B(k, col);
        d[e] += acc;
    }
    emu::warp_sync();
}
}  // namespace mbk
}  // namespace ttt
