// Host emulation of the further operations that the TTT-MLP tensor-core kernel
// uses, on top of tc_emu_lfr.h: TEST INFRASTRUCTURE, never part of the library.
//
// Semantics (from the PTX ISA's descriptions):
//   ldmatrix / stmatrix .m8n8.xN .b16 (N = 2 or 4): lanes 8i .. 8i+7 give the
//     row addresses of matrix i; register i of lane L holds the elements
//     (L/4, 2(L%4)) and (L/4, 2(L%4)+1) of matrix i, or with .trans the
//     elements (2(L%4), L/4) and (2(L%4)+1, L/4); the first is the low half.
//   tcgen05.ld .16x256b.x1: as one repetition of the x2 form in tc_emu_lfr.h.
//   tcgen05.st .16x128b.x1: 16 TMEM lanes x 4 columns; thread t writes its
//     first register to (lane t/4, column t%4) and its second to
//     (lane t/4 + 8, column t%4).
//   tcgen05.mma with M = 64: see umma_apply in tc_emu.h.
#pragma once
#include "tc_emu_lfr.h"

namespace emu {
template <bool T, int NM>
inline void ldsm_n(uint32_t addr, uint32_t* r) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    xch[w].u[lane][0] = addr;
    warp_sync();
    for (int i = 0; i < NM; ++i) {
        uint16_t lo, hi;
        if (!T) {
            const uint32_t row = xch[w].u[8 * i + lane / 4][0];
            lo = ld16(row + 4 * (lane % 4));
            hi = ld16(row + 4 * (lane % 4) + 2);
        } else {
            lo = ld16(xch[w].u[8 * i + 2 * (lane % 4)][0] + 2 * (lane / 4));
            hi = ld16(xch[w].u[8 * i + 2 * (lane % 4) + 1][0] + 2 * (lane / 4));
        }
        r[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    warp_sync();
}
template <int NM>
inline void stsm_n_trans(uint32_t addr, const uint32_t* reg) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    xch[w].u[lane][0] = addr;
    warp_sync();
    uint8_t* base = const_cast<uint8_t*>(shared_base);
    for (int i = 0; i < NM; ++i) {
        const uint16_t lo = (uint16_t)(reg[i] & 0xFFFFu), hi = (uint16_t)(reg[i] >> 16);
        std::memcpy(base + xch[w].u[8 * i + 2 * (lane % 4)][0] + 2 * (lane / 4), &lo, 2);
        std::memcpy(base + xch[w].u[8 * i + 2 * (lane % 4) + 1][0] + 2 * (lane / 4), &hi, 2);
    }
    warp_sync();
}
}  // namespace emu

namespace ttt {
namespace mtc {
inline void ldsm_x4_tr(uint32_t addr, uint32_t* r) { emu::ldsm_n<true, 4>(addr, r); }
inline void stsm_x4_tr(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    const uint32_t r[4] = {r0, r1, r2, r3};
    emu::stsm_n_trans<4>(addr, r);
}
inline void ldsm_x2(uint32_t addr, uint32_t* r) { emu::ldsm_n<false, 2>(addr, r); }
inline void ldsm_x2_tr(uint32_t addr, uint32_t* r) { emu::ldsm_n<true, 2>(addr, r); }
inline void stsm_x2_tr(uint32_t addr, uint32_t r0, uint32_t r1) {
    const uint32_t r[2] = {r0, r1};
    emu::stsm_n_trans<2>(addr, r);
}
inline void tmem_st_32x32b_x4(uint32_t taddr, const uint32_t* r) { emu::tmem_st_32x32b<4>(taddr, r); }
inline void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t* r) { tmem_ld_32x32b<8>(taddr, r); }
inline void tmem_ld_16x256b_x1(uint32_t taddr, uint32_t* r) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const uint32_t l0 = emu::tmem_lane(taddr), c0 = emu::tmem_col(taddr);
    if (l0 / 32 != (uint32_t)(w % 4) || l0 % 16 != 0 || c0 + 8 > 512) ++emu::errors;
    const int g = lane / 4, c = lane % 4;
    uint32_t vals[4];
    for (int e = 0; e < 4; ++e) vals[e] = emu::tmem[(l0 + g + 8 * (e >> 1)) & 127][(c0 + 2 * c + (e & 1)) & 511];
    emu::deliver(r, vals, 4);
    emu::warp_sync();
}
inline void tmem_st_16x128b_x1(uint32_t taddr, uint32_t r0, uint32_t r1) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const uint32_t l0 = emu::tmem_lane(taddr), c0 = emu::tmem_col(taddr);
    if (l0 / 32 != (uint32_t)(w % 4) || l0 % 16 != 0 || c0 + 4 > 512) ++emu::errors;
    const int g = lane / 4, c = lane % 4;
    emu::tmem_put(l0 + g, c0 + c, r0);
    emu::tmem_put(l0 + g + 8, c0 + c, r1);
    emu::warp_sync();
}
}  // namespace mtc
}  // namespace ttt
