// Host emulation of the CUDA execution model for the CPU tests: TEST
// INFRASTRUCTURE, never part of the library (which has no CPU path).
//
// One CTA at a time.  Each CUDA thread of the CTA is a std::thread running
// the kernel function; __syncthreads is a std::barrier over the CTA; a
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

#include <barrier>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace emu {
constexpr int kMaxThreads = 1024;
inline thread_local uint3 tid3, bid3;
inline uint3 grid3;
inline std::barrier<>* block_bar = nullptr;
inline std::barrier<>* warp_bar[kMaxThreads / 32];
inline const uint8_t* shared_base = nullptr;
struct WarpXch {
    float f[32];
    uint32_t u[32][4];
    uint32_t v[32][2];
    float c[32][4];
};
inline WarpXch xch[kMaxThreads / 32];

inline void warp_sync() { warp_bar[tid3.x >> 5]->arrive_and_wait(); }

template <typename F>
void run_grid(int blocks, int threads, const void* shared, F f) {
    shared_base = static_cast<const uint8_t*>(shared);
    grid3 = make_uint3(blocks, 1, 1);
    for (int bx = 0; bx < blocks; ++bx) {
        std::barrier<> bb(threads);
        for (int w = 0; w < threads / 32; ++w) warp_bar[w] = new std::barrier<>(32);
        block_bar = &bb;
        std::vector<std::thread> th;
        th.reserve(threads);
        for (int t = 0; t < threads; ++t)
            th.emplace_back([&, t, bx] {
                tid3 = make_uint3(t, 0, 0);
                bid3 = make_uint3(bx, 0, 0);
                f();
            });
        for (auto& x : th) x.join();
        for (int w = 0; w < threads / 32; ++w) delete warp_bar[w];
    }
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
inline void __syncthreads() { emu::block_bar->arrive_and_wait(); }
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
