// Building blocks shared by the tensor-core kernels: the parameter block of
// the TTT-Linear kernels, shared-memory layout helpers, mma.sync fragment
// loaders, tcgen05.st wrappers and tcgen05.mma with A in tensor memory.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace ttt {
namespace tcc {

// Arguments of the TTT-Linear tensor-core kernel (one launch: U = B * H
// units of T tokens, nsteps = T / 16 mini-batches).
struct LinearParams {
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

#ifndef TTT_HOST_EMULATION   // the host emulation supplies these two
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

#endif
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
#ifndef TTT_HOST_EMULATION   // the host emulation supplies these
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
#endif

}  // namespace tcc
}  // namespace ttt
