// Host emulation of the further sm_100a operations that the TTT-Linear
// tensor-core kernel uses, on top of tc_emu.h: TEST INFRASTRUCTURE, never part
// of the library.
//
// Semantics (from the PTX ISA's descriptions):
//   tcgen05.st .32x32b.xN: lane t of the warp writes TMEM lane (base + t),
//     columns col .. col + N - 1; a warp may access its quadrant only.
//   tcgen05.ld .16x256b.x2: 16 TMEM lanes x 8 columns per repetition, the
//     second repetition 8 columns further on; with g = t / 4, c = t % 4,
//     thread t receives (lane g, column 2c), (g, 2c+1), (g+8, 2c), (g+8, 2c+1)
//     of each repetition: the m16n8 accumulator layout of mma.sync.
//   stmatrix .m8n8.x4.trans .b16: lanes 8i .. 8i+7 give the row addresses of
//     matrix i; register i of lane L holds fragment elements (L/4, 2(L%4)) and
//     (L/4, 2(L%4)+1), which land at (2(L%4), L/4) and (2(L%4)+1, L/4).
//   bar.sync id, n: a barrier over n threads, one per id (emu_core.h's EBar).
//   cp.async.bulk (global -> shared): the bytes count toward the mbarrier.
//   cp.async.bulk.tensor store, 2-D tile with a 32-, 64- or 128-byte swizzle:
//     shared byte lin = r * rowbytes + b of the box is read at
//     lin ^ (((lin >> 7) & mask) << 4) (mask 1, 3, 7); rows outside the tensor
//     are not written.
// As in tc_emu.h, asynchronous operations complete when they are issued, or,
// in the deferred mode, later (on the engine thread, or, for tensor-memory
// loads and stores, at the thread's tcgen05.wait).
#pragma once
#include "tc_emu.h"

namespace emu {
inline std::mutex named_mu;
inline EBar* named[16];
inline int named_count[16];
inline void reset_named() {
    for (int i = 0; i < 16; ++i) {
        delete named[i];
        named[i] = nullptr;
        named_count[i] = 0;
    }
}
// a tensor map with the swizzle span (32, 64 or 128 bytes) in the last field
inline void make_map_swz(CUtensorMap* m, const void* base, unsigned long long cols, unsigned long long rows,
                         unsigned long long pitch, unsigned box_cols, unsigned box_rows, unsigned elem, int span) {
    make_map(m, base, cols, rows, pitch, box_cols, box_rows, elem);
    FakeMap f;
    std::memcpy(&f, m, sizeof(f));
    f.swizzle128 = span;
    std::memcpy(m, &f, sizeof(f));
}
template <int N>
inline void tmem_st_32x32b(uint32_t taddr, const uint32_t* r) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const uint32_t l0 = tmem_lane(taddr), c0 = tmem_col(taddr);
    if (l0 / 32 != (uint32_t)(w % 4) || l0 % 32 != 0 || c0 + N > 512) ++errors;
    for (int i = 0; i < N; ++i) tmem_put(l0 + lane, c0 + i, r[i]);
    warp_sync();
}
}  // namespace emu

inline uint32_t __float_as_uint(float f) {
    uint32_t v;
    std::memcpy(&v, &f, 4);
    return v;
}

namespace ttt {
inline void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t* r) { emu::tmem_st_32x32b<16>(taddr, r); }
inline void named_bar_sync(int id, int nthreads) {
    emu::EBar* b;
    {
        std::lock_guard<std::mutex> lk(emu::named_mu);
        if (id < 0 || id >= 16 || (emu::named[id] && emu::named_count[id] != nthreads)) {
            ++emu::errors;
            return;
        }
        if (!emu::named[id]) {
            emu::named[id] = new emu::EBar(nthreads);
            emu::named_count[id] = nthreads;
        }
        b = emu::named[id];
    }
    b->wait();
}
inline void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    if ((emu::shared_base && ((static_cast<uint8_t*>(dst) - emu::shared_base) % 16)) || bytes % 16 ||
        (reinterpret_cast<uintptr_t>(src) % 16))
        ++emu::errors;
    emu::async_do([=] {
        std::memcpy(dst, src, bytes);
        emu::bar_complete_tx(bar, bytes);
    }, emu::kLoad);
}
inline void bulk_commit() {}
// every store of this thread issued so far (one store per group in these kernels, so N = 0 only)
template <int N>
inline void bulk_wait_read() {
    static_assert(N == 0, "one store per group");
    emu::flush_stores(threadIdx.x);
    while (emu::pending_stores[threadIdx.x].load() != 0) emu::spin_yield();
}
template <int N>
inline void bulk_wait() {
    bulk_wait_read<N>();
}
inline void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
    emu::FakeMap f;
    std::memcpy(&f, map, sizeof(f));
    const int span = f.swizzle128 == 1 ? 128 : f.swizzle128;
    const uint32_t mask = span == 128 ? 7u : span == 64 ? 3u : 1u;
    const unsigned rowb = f.box_cols * f.elem;
    const uint8_t* s = static_cast<const uint8_t*>(src);
    if ((unsigned)span != rowb || ((s - emu::shared_base) % (8 * span)) != 0 || x < 0 || y < 0 ||
        (x * f.elem) % 16 != 0)
        ++emu::errors;
    std::atomic<int>* pend = &emu::pending_stores[threadIdx.x];
    ++*pend;
    auto job = [=] {
        for (unsigned r = 0; r < f.box_rows; ++r)
            for (unsigned b = 0; b < rowb; ++b) {
                const unsigned long long gx = (unsigned long long)x + b / f.elem, gy = (unsigned long long)y + r;
                if (gx >= f.cols || gy >= f.rows) continue;
                const uint32_t lin = r * rowb + b;
                const uint32_t phys = lin ^ (((lin >> 7) & mask) << 4);
                static_cast<uint8_t*>(const_cast<void*>(f.base))[gy * f.pitch + gx * f.elem + b % f.elem] = s[phys];
            }
        --*pend;
    };
    if (emu::deferred.load())
        emu::held_stores[threadIdx.x].push_back(job);
    else
        job();
}

namespace tcc {
inline void ldsm_x4(uint32_t addr, uint32_t* r) { mbk::ldsm4(addr, r); }
inline void mma_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) { mbk::mma(d, a, b0, b1); }
inline void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t* r) { emu::tmem_st_32x32b<8>(taddr, r); }
inline void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t* r) { emu::tmem_st_32x32b<32>(taddr, r); }
inline void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    const bool b_mn = (idesc >> 16) & 1u;
    if ((idesc >> 15) & 1u) ++emu::errors;   // an A in tensor memory is K-major
    emu::async_do([=] {
        umma_apply(
            d_tmem, idesc, accumulate, [&](int row, int k) { return tmem_bf16(a_tmem, row, k); },
            [&](int col, int k) { return operand_elem(bdesc, b_mn, col, k); });
    }, emu::kMma);
}
}  // namespace tcc

namespace lfr {
inline void tmem_ld_16x256b_x2(uint32_t taddr, uint32_t* r) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const uint32_t l0 = emu::tmem_lane(taddr), c0 = emu::tmem_col(taddr);
    if (l0 / 32 != (uint32_t)(w % 4) || l0 % 16 != 0 || c0 + 16 > 512) ++emu::errors;
    const int g = lane / 4, c = lane % 4;
    uint32_t vals[8];
    for (int rep = 0; rep < 2; ++rep)
        for (int e = 0; e < 4; ++e)
            vals[4 * rep + e] = emu::tmem[(l0 + g + 8 * (e >> 1)) & 127][(c0 + 8 * rep + 2 * c + (e & 1)) & 511];
    emu::deliver(r, vals, 8);
    emu::warp_sync();
}
inline void stsm_x4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    emu::xch[w].u[lane][0] = addr;
    emu::warp_sync();
    const uint32_t reg[4] = {r0, r1, r2, r3};
    uint8_t* base = const_cast<uint8_t*>(emu::shared_base);
    for (int i = 0; i < 4; ++i) {
        const uint16_t lo = (uint16_t)(reg[i] & 0xFFFFu), hi = (uint16_t)(reg[i] >> 16);
        const uint32_t a0 = emu::xch[w].u[8 * i + 2 * (lane % 4)][0] + 2 * (lane / 4);
        const uint32_t a1 = emu::xch[w].u[8 * i + 2 * (lane % 4) + 1][0] + 2 * (lane / 4);
        std::memcpy(base + a0, &lo, 2);
        std::memcpy(base + a1, &hi, 2);
    }
    emu::warp_sync();
}
inline void ldsm_x4_t(uint32_t addr, uint32_t* r) { mbk::ldsm4t(addr, r); }
inline void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) { mbk::mma(d, a, b0, b1); }
}  // namespace lfr
}  // namespace ttt
