// libttt: C ABI of the TTT inner-loop forward on B200 (sm_100a).
//
// Host side: argument validation (synchronous, before any launch), kernel
// selection, TMA descriptor creation and launch.  The declarations and the
// contract of every entry point are in include/ttt.h.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/ttt.h"
#include "common.cuh"
#include "decode.cuh"
#include "linear_frag.cuh"
#include "mlp_decode.cuh"
#include "mlp_tc.cuh"
#include "simt.cuh"
#include "simt_backward.cuh"
#include "simt_backward_ln.cuh"
#include "simt_mlp_backward.cuh"
#include "mma_backward.cuh"
#include "mma_forward.cuh"
#include "mma_ln.cuh"
#include "mma_mlp_backward.cuh"
#include "prologue.cuh"
#include "simt_prologue.cuh"
#include "tmap.h"

namespace ttt {

// Per-device status word (bit kStatusTimeout: a bounded wait expired).
__device__ int g_status_word;

namespace {

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
std::mutex g_mu;

// Device address of the status word on the current device (looked up once
// per device with that device current).
int* status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

ttt_status launch_status() {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        fprintf(stderr, "libttt: launch failed: %s\n", cudaGetErrorString(e));
        return TTT_ERR_CUDA;
    }
    return TTT_OK;
}

// Raise the dynamic shared memory limit of a kernel once per device.
template <typename K>
bool set_smem(K kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return true;
    if (bytes > 227 * 1024) return false;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess;
}

unsigned long long wait_ns(unsigned ms) { return 1000000ull * (ms ? ms : kDefaultWaitMs); }

// ---------------------------------------------------------------------------
// TTT-Linear
// ---------------------------------------------------------------------------
template <int D, bool LN, typename IO>
ttt_status launch_simt_linear(const ttt_linear_args* a, cudaStream_t st) {
    SimtLinearParams p;
    p.H = a->H;
    p.T = a->T;
    p.b = a->b;
    p.Q = a->Q;
    p.K = a->K;
    p.V = a->V;
    p.eta = a->eta;
    p.eta_const = a->eta_const;
    p.W0 = a->W0;
    p.W0_bstride = a->W0_bstride;
    p.c0 = a->c0;
    p.c0_bstride = a->c0_bstride;
    p.gamma = a->ln_gamma;
    p.beta = a->ln_beta;
    p.eps = a->ln_eps;
    p.Z = a->Z;
    p.W_out = a->W_out;
    p.c_out = a->c_out;
    p.W_states = a->W_states;
    p.c_states = a->c_states;
    const size_t smem = simt_linear_smem(D, a->b);
    auto k = simt_linear_kernel<D, LN, IO>;
    if (!set_smem(k, smem)) return TTT_ERR_UNSUPPORTED;
    k<<<a->B * a->H, kSimtThreads, smem, st>>>(p);
    return launch_status();
}

template <int D, bool LN>
ttt_status simt_linear_dtype(const ttt_linear_args* a, cudaStream_t st) {
    return a->io_dtype == TTT_F32 ? launch_simt_linear<D, LN, float>(a, st)
                                  : launch_simt_linear<D, LN, __nv_bfloat16>(a, st);
}

template <bool LN>
ttt_status simt_linear(const ttt_linear_args* a, cudaStream_t st) {
    switch (a->d) {
        case 16: return simt_linear_dtype<16, LN>(a, st);
        case 32: return simt_linear_dtype<32, LN>(a, st);
        case 64: return simt_linear_dtype<64, LN>(a, st);
        default: return TTT_ERR_UNSUPPORTED;
    }
}

template <bool LN>
ttt_status tc_linear(const ttt_linear_args* a, cudaStream_t st) {
    using namespace lfr;
    const long long U = (long long)a->B * a->H;
    const long long rows = U * a->T;
    CUtensorMap mQ, mK, mV;
    const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!encode_2d(&mQ, a->Q, bf, kD, rows, kD * 2, kD, kTok, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&mK, a->K, bf, kD, rows, kD * 2, kD, kTok, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&mV, a->V, bf, kD, rows, kD * 2, kD, kTok, CU_TENSOR_MAP_SWIZZLE_128B))
        return TTT_ERR_CUDA;
    tcc::LinearParams p;
    p.U = (int)U;
    p.H = a->H;
    p.T = a->T;
    p.nsteps = a->T / kTok;
    p.eta = a->eta;
    p.eta_const = a->eta_const;
    p.W0 = a->W0;
    p.W0_bstride = a->W0_bstride;
    p.c0 = a->c0;
    p.c0_bstride = a->c0_bstride;
    p.gamma = a->ln_gamma;
    p.beta = a->ln_beta;
    p.eps = a->ln_eps;
    p.Z = static_cast<__nv_bfloat16*>(a->Z);
    p.W_out = a->W_out;
    p.c_out = a->c_out;
    p.status = status_ptr();
    p.wait_ns = wait_ns(a->wait_timeout_ms);
    p.flags = a->flags;
    if (!p.status) return TTT_ERR_CUDA;
    const int grid = (int)((U + 1) / 2);
    // pairs of mini-batches per tensor-core round trip; Z is written by TMA
    // stores of 32-token (and, for an odd last mini-batch, 16-token) boxes of
    // the 32 (two units per CTA) or 16 (one unit per CTA) features of a warp
    const bool one = (a->flags & TTT_FLAG_ONE_UNIT_PER_CTA) ||
                     (!(a->flags & TTT_FLAG_TWO_UNITS_PER_CTA) && U <= kOneUnitMaxUnits);
    const uint32_t zcols = one ? 16 : 32;
    const auto zswz = one ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap mZ, mZ1;
    if (!encode_2d(&mZ, a->Z, bf, kD, rows, kD * 2, zcols, 2 * kTok, zswz) ||
        !encode_2d(&mZ1, a->Z, bf, kD, rows, kD * 2, zcols, kTok, zswz))
        return TTT_ERR_CUDA;
    auto k = one ? lfr::linear_frag_kernel<LN, 1> : lfr::linear_frag_kernel<LN, 2>;
    if (!set_smem(k, lfr::kSmemBytes)) return TTT_ERR_CUDA;
    k<<<one ? (int)U : grid, lfr::kThreads, lfr::kSmemBytes, st>>>(mQ, mK, mV, mZ, mZ1, p);
    return launch_status();
}

ttt_status validate_common(int B, int H, int T, int d, int b, ttt_dtype io) {
    if (B < 0 || H < 0 || T < 0 || b < 1) return TTT_ERR_INVALID_ARG;
    if (io != TTT_F32 && io != TTT_BF16) return TTT_ERR_INVALID_ARG;
    if (d <= 0) return TTT_ERR_INVALID_ARG;
    if (T % b != 0) return TTT_ERR_INVALID_ARG;
    if (d != 16 && d != 32 && d != 64) return TTT_ERR_UNSUPPORTED;
    if (b > 64) return TTT_ERR_UNSUPPORTED;
    const long long rows = (long long)B * H * T;
    if ((long long)B * H > (1ll << 30) || rows >= (1ll << 31)) return TTT_ERR_UNSUPPORTED;
    return TTT_OK;
}

}  // namespace
}  // namespace ttt

using namespace ttt;

extern "C" ttt_status ttt_linear_forward(const ttt_linear_args* a, cudaStream_t stream) {
    if (!a) return TTT_ERR_INVALID_ARG;
    ttt_status v = validate_common(a->B, a->H, a->T, a->d, a->b, a->io_dtype);
    if (v != TTT_OK) return v;
    const long long units = (long long)a->B * a->H;
    if (units == 0) return TTT_OK;
    if (a->T > 0 && (!ok_ptr(a->Q) || !ok_ptr(a->K) || !ok_ptr(a->V) || !ok_opt(a->Z)))
        return TTT_ERR_INVALID_ARG;
    if (!ok_ptr(a->W0) || !ok_ptr(a->W_out) || !ok_opt(a->eta)) return TTT_ERR_INVALID_ARG;
    if (a->W0_bstride < 0 || a->c0_bstride < 0) return TTT_ERR_INVALID_ARG;
    if (a->use_ln != 0 && a->use_ln != 1) return TTT_ERR_INVALID_ARG;
    if (a->use_ln) {
        if (!ok_ptr(a->ln_gamma) || !ok_ptr(a->ln_beta) || !ok_opt(a->c0) || !ok_opt(a->c_out))
            return TTT_ERR_INVALID_ARG;
        if (!(a->ln_eps > 0.f)) return TTT_ERR_INVALID_ARG;
    }
    if (a->flags & ~(TTT_FLAG_FORCE_SIMT | TTT_FLAG_TEST_STALL | TTT_FLAG_ONE_UNIT_PER_CTA |
                     TTT_FLAG_TWO_UNITS_PER_CTA | TTT_FLAG_LN_MMA_TRAINING))
        return TTT_ERR_INVALID_ARG;
    if ((a->flags & TTT_FLAG_ONE_UNIT_PER_CTA) && (a->flags & TTT_FLAG_TWO_UNITS_PER_CTA))
        return TTT_ERR_INVALID_ARG;
    if (a->W_states) {
        if (!aligned16(a->W_states)) return TTT_ERR_INVALID_ARG;
        if (a->use_ln && !ok_ptr(a->c_states)) return TTT_ERR_INVALID_ARG;
    }
    if (a->W_states && a->use_ln && (a->flags & TTT_FLAG_LN_MMA_TRAINING) && a->io_dtype == TTT_BF16 &&
        a->d == 64 && a->b == 16 && a->T > 0 && !(a->flags & TTT_FLAG_FORCE_SIMT)) {
        // LN+residual training on mma.sync: the forward that writes (W, c) at every mini-batch start
        if (a->flags & TTT_FLAG_TEST_STALL) return TTT_ERR_UNSUPPORTED;
        mbk::FwdLnStatesParams p{a->H,      a->T,          a->Q,    a->K,          a->V,        a->eta,
                                 a->eta_const, a->W0,      a->W0_bstride, a->c0,   a->c0_bstride, a->ln_gamma,
                                 a->ln_beta, a->ln_eps,    a->Z,    a->W_out,      a->c_out,    a->W_states,
                                 a->c_states};
        mbk::mma_ln_forward_states_kernel<<<(unsigned)units, mbk::kThreads, mbk::kLFSmemBytes, stream>>>(p);
        return launch_status();
    }
    const bool states_on_simt = a->W_states && a->use_ln;   // the LN states come from the fp32 kernel
    const bool tc = a->io_dtype == TTT_BF16 && a->d == 64 && a->b == 16 && a->T > 0 && a->Z &&
                    !(a->flags & TTT_FLAG_FORCE_SIMT) && !states_on_simt;
    if (tc && a->W_states) {
        // training: the mma.sync forward that also writes the batch-start states
        if (a->flags & TTT_FLAG_TEST_STALL) return TTT_ERR_UNSUPPORTED;
        mbk::FwdStatesParams p{a->H, a->T, a->Q, a->K, a->V, a->eta, a->eta_const, a->W0, a->W0_bstride,
                               a->Z, a->W_out, a->W_states};
        mbk::mma_linear_forward_states_kernel<<<(unsigned)units, mbk::kThreads, mbk::kFSmemBytes, stream>>>(p);
        return launch_status();
    }
    if (tc) return a->use_ln ? tc_linear<true>(a, stream) : tc_linear<false>(a, stream);
    if (a->flags & TTT_FLAG_TEST_STALL) return TTT_ERR_UNSUPPORTED;
    return a->use_ln ? simt_linear<true>(a, stream) : simt_linear<false>(a, stream);
}

// ---------------------------------------------------------------------------
// TTT-MLP
// ---------------------------------------------------------------------------
namespace ttt {
namespace {

template <int D, typename IO>
ttt_status launch_simt_mlp(const ttt_mlp_args* a, cudaStream_t st) {
    SimtMlpParams p;
    p.H = a->H;
    p.T = a->T;
    p.b = a->b;
    p.Q = a->Q;
    p.K = a->K;
    p.V = a->V;
    p.eta = a->eta;
    p.eta_const = a->eta_const;
    p.W1 = a->W1;
    p.c1 = a->c1;
    p.W2 = a->W2;
    p.c2 = a->c2;
    p.per_seq = a->params_per_sequence;
    p.Z = a->Z;
    p.W1_out = a->W1_out;
    p.c1_out = a->c1_out;
    p.W2_out = a->W2_out;
    p.c2_out = a->c2_out;
    p.gamma = a->ln_gamma;
    p.beta = a->ln_beta;
    p.eps = a->ln_eps;
    p.W_states = a->W_states;
    const size_t smem = simt_mlp_smem(D, a->b, a->use_ln != 0);
    auto k = a->use_ln ? simt_mlp_kernel<D, IO, true> : simt_mlp_kernel<D, IO, false>;
    if (!set_smem(k, smem)) return TTT_ERR_UNSUPPORTED;
    k<<<a->B * a->H, kSimtThreads, smem, st>>>(p);
    return launch_status();
}

template <int D>
ttt_status simt_mlp_dtype(const ttt_mlp_args* a, cudaStream_t st) {
    return a->io_dtype == TTT_F32 ? launch_simt_mlp<D, float>(a, st) : launch_simt_mlp<D, __nv_bfloat16>(a, st);
}

}  // namespace
}  // namespace ttt

namespace ttt {
namespace {
ttt_status tc_mlp(const ttt_mlp_args* a, cudaStream_t st) {
    using namespace mtc;
    const long long U = (long long)a->B * a->H;
    const long long rows = U * a->T;
    CUtensorMap mQ, mK, mV;
    const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!encode_2d(&mQ, a->Q, bf, kD, rows, kD * 2, kD, kTok, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&mK, a->K, bf, kD, rows, kD * 2, kD, kTok, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&mV, a->V, bf, kD, rows, kD * 2, kD, kTok, CU_TENSOR_MAP_SWIZZLE_128B))
        return TTT_ERR_CUDA;
    Params p;
    p.H = a->H;
    p.T = a->T;
    p.nsteps = a->T / kTok;
    p.per_seq = a->params_per_sequence;
    p.eta = a->eta;
    p.eta_const = a->eta_const;
    p.W1 = a->W1;
    p.c1 = a->c1;
    p.W2 = a->W2;
    p.c2 = a->c2;
    p.Z = static_cast<__nv_bfloat16*>(a->Z);
    p.W1_out = a->W1_out;
    p.c1_out = a->c1_out;
    p.W2_out = a->W2_out;
    p.c2_out = a->c2_out;
    p.status = status_ptr();
    p.wait_ns = wait_ns(a->wait_timeout_ms);
    p.flags = a->flags;
    p.gamma = a->ln_gamma;
    p.beta = a->ln_beta;
    p.eps = a->ln_eps;
    if (!p.status) return TTT_ERR_CUDA;
    auto k = a->use_ln ? mlp_tc_kernel<true> : mlp_tc_kernel<false>;
    if (!set_smem(k, kSmemBytes)) return TTT_ERR_CUDA;
    k<<<(int)U, kThreads, kSmemBytes, st>>>(mQ, mK, mV, p);
    return launch_status();
}
}  // namespace
}  // namespace ttt

extern "C" ttt_status ttt_mlp_forward(const ttt_mlp_args* a, cudaStream_t stream) {
    if (!a) return TTT_ERR_INVALID_ARG;
    ttt_status v = validate_common(a->B, a->H, a->T, a->d, a->b, a->io_dtype);
    if (v != TTT_OK) return v;
    const long long units = (long long)a->B * a->H;
    if (units == 0) return TTT_OK;
    if (a->T > 0 && (!ok_ptr(a->Q) || !ok_ptr(a->K) || !ok_ptr(a->V) || !ok_ptr(a->Z)))
        return TTT_ERR_INVALID_ARG;
    if (!ok_ptr(a->W1) || !ok_ptr(a->W2) || !ok_opt(a->c1) || !ok_opt(a->c2) || !ok_opt(a->eta))
        return TTT_ERR_INVALID_ARG;
    if (!ok_ptr(a->W1_out) || !ok_ptr(a->W2_out) || !ok_opt(a->c1_out) || !ok_opt(a->c2_out))
        return TTT_ERR_INVALID_ARG;
    if (a->params_per_sequence != 0 && a->params_per_sequence != 1) return TTT_ERR_INVALID_ARG;
    if (a->flags & ~(TTT_FLAG_FORCE_SIMT | TTT_FLAG_TEST_STALL)) return TTT_ERR_INVALID_ARG;
    if (a->use_ln != 0 && a->use_ln != 1) return TTT_ERR_INVALID_ARG;
    if (a->use_ln && (!ok_ptr(a->ln_gamma) || !ok_ptr(a->ln_beta) || !(a->ln_eps > 0.f))) return TTT_ERR_INVALID_ARG;
    if (!ok_opt(a->W_states)) return TTT_ERR_INVALID_ARG;
    if (a->W_states && a->io_dtype == TTT_BF16 && a->d == 64 && a->b == 16 && a->T > 0 &&
        !(a->flags & TTT_FLAG_FORCE_SIMT)) {
        // training: the mma.sync forward that writes the batch-start states
        if (a->flags & TTT_FLAG_TEST_STALL) return TTT_ERR_UNSUPPORTED;
        mmb::MlpFwdStatesParams p{a->H,      a->T,     a->Q,     a->K,      a->V,     a->eta,
                                  a->eta_const, a->W1, a->c1,    a->W2,     a->c2,    a->params_per_sequence,
                                  a->Z,      a->W1_out, a->c1_out, a->W2_out, a->c2_out, a->W_states,
                                  a->ln_gamma, a->ln_beta, a->ln_eps};
        auto k = a->use_ln ? mmb::mma_mlp_forward_states_kernel<true> : mmb::mma_mlp_forward_states_kernel<false>;
        if (!set_smem(k, mmb::kSmemBytes)) return TTT_ERR_CUDA;
        k<<<(unsigned)units, mmb::kThreads, mmb::kSmemBytes, stream>>>(p);
        return launch_status();
    }
    const bool tc = a->io_dtype == TTT_BF16 && a->d == 64 && a->b == 16 && a->T > 0 &&
                    !(a->flags & TTT_FLAG_FORCE_SIMT) && !a->W_states;
    if (tc) return tc_mlp(a, stream);
    if (a->flags & TTT_FLAG_TEST_STALL) return TTT_ERR_UNSUPPORTED;
    switch (a->d) {
        case 16: return simt_mlp_dtype<16>(a, stream);
        case 32: return simt_mlp_dtype<32>(a, stream);
        case 64: return simt_mlp_dtype<64>(a, stream);
        default: return TTT_ERR_UNSUPPORTED;
    }
}

// ---------------------------------------------------------------------------
// Decode
// ---------------------------------------------------------------------------
namespace ttt {
namespace {
template <int D, typename IO>
ttt_status launch_decode_t(const ttt_decode_args* a, cudaStream_t st) {
    DecodeParams p{a->W, a->q, a->k, a->v, a->eta, a->eta_const, a->z,
                   a->c, a->ln_gamma, a->ln_beta, a->ln_eps, a->H};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a->B * a->H));
    cfg.blockDim = dim3(D * 4);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    const cudaError_t e = a->use_ln ? cudaLaunchKernelEx(&cfg, decode_kernel<D, IO, true>, p)
                                    : cudaLaunchKernelEx(&cfg, decode_kernel<D, IO, false>, p);
    if (e != cudaSuccess) return launch_status();
    return launch_status();
}
template <int D>
ttt_status launch_decode(const ttt_decode_args* a, cudaStream_t st) {
    return a->io_dtype == TTT_F32 ? launch_decode_t<D, float>(a, st) : launch_decode_t<D, __nv_bfloat16>(a, st);
}
}  // namespace
}  // namespace ttt

extern "C" ttt_status ttt_linear_decode_step(const ttt_decode_args* a, cudaStream_t stream) {
    if (!a) return TTT_ERR_INVALID_ARG;
    if (a->B < 0 || a->H < 0 || a->d <= 0) return TTT_ERR_INVALID_ARG;
    if (a->io_dtype != TTT_F32 && a->io_dtype != TTT_BF16) return TTT_ERR_INVALID_ARG;
    if (a->d != 16 && a->d != 32 && a->d != 64) return TTT_ERR_UNSUPPORTED;
    if ((long long)a->B * a->H > (1ll << 30)) return TTT_ERR_UNSUPPORTED;
    if ((long long)a->B * a->H == 0) return TTT_OK;
    if (!ok_ptr(a->W) || !ok_ptr(a->q) || !ok_ptr(a->k) || !ok_ptr(a->v) || !ok_ptr(a->z) || !ok_opt(a->eta))
        return TTT_ERR_INVALID_ARG;
    if (a->use_ln != 0 && a->use_ln != 1) return TTT_ERR_INVALID_ARG;
    if (a->use_ln && (!ok_ptr(a->c) || !ok_ptr(a->ln_gamma) || !ok_ptr(a->ln_beta) || !(a->ln_eps > 0.f)))
        return TTT_ERR_INVALID_ARG;
    switch (a->d) {
        case 16: return launch_decode<16>(a, stream);
        case 32: return launch_decode<32>(a, stream);
        default: return launch_decode<64>(a, stream);
    }
}

namespace ttt {
namespace {
template <int D, typename IO>
ttt_status launch_mlp_decode_t(const ttt_mlp_decode_args* a, cudaStream_t st) {
    MlpDecodeParams p{a->W1, a->c1, a->W2, a->c2, a->q, a->k, a->v, a->eta, a->eta_const, a->z};
    mlp_decode_kernel<D, IO><<<(unsigned)(a->B * a->H), 4 * D, 0, st>>>(p);
    return launch_status();
}
template <int D>
ttt_status launch_mlp_decode(const ttt_mlp_decode_args* a, cudaStream_t st) {
    return a->io_dtype == TTT_F32 ? launch_mlp_decode_t<D, float>(a, st)
                                  : launch_mlp_decode_t<D, __nv_bfloat16>(a, st);
}
}  // namespace
}  // namespace ttt

extern "C" ttt_status ttt_mlp_decode_step(const ttt_mlp_decode_args* a, cudaStream_t stream) {
    if (!a) return TTT_ERR_INVALID_ARG;
    if (a->B < 0 || a->H < 0 || a->d <= 0) return TTT_ERR_INVALID_ARG;
    if (a->io_dtype != TTT_F32 && a->io_dtype != TTT_BF16) return TTT_ERR_INVALID_ARG;
    if (a->d != 16 && a->d != 32 && a->d != 64) return TTT_ERR_UNSUPPORTED;
    if ((long long)a->B * a->H > (1ll << 30)) return TTT_ERR_UNSUPPORTED;
    if ((long long)a->B * a->H == 0) return TTT_OK;
    if (!ok_ptr(a->W1) || !ok_ptr(a->c1) || !ok_ptr(a->W2) || !ok_ptr(a->c2) || !ok_ptr(a->q) || !ok_ptr(a->k) ||
        !ok_ptr(a->v) || !ok_ptr(a->z) || !ok_opt(a->eta))
        return TTT_ERR_INVALID_ARG;
    switch (a->d) {
        case 16: return launch_mlp_decode<16>(a, stream);
        case 32: return launch_mlp_decode<32>(a, stream);
        default: return launch_mlp_decode<64>(a, stream);
    }
}

namespace ttt {
namespace {
template <int D, typename IO>
ttt_status launch_ln_backward_t(const ttt_linear_backward_args* a, cudaStream_t st) {
    SimtLnBackwardParams p{a->H, a->T, a->b, a->Q, a->K, a->V, a->eta, a->eta_const, a->W_states, a->c_states,
                           a->ln_gamma, a->ln_beta, a->ln_eps, a->dZ, a->dW_out, a->dc_out, a->dQ, a->dK, a->dV,
                           a->deta, a->dW0, a->dc0, a->dgamma, a->dbeta};
    const size_t smem = simt_ln_backward_smem(D, a->b);
    auto k = simt_ln_backward_kernel<D, IO>;
    if (!set_smem(k, smem)) return TTT_ERR_UNSUPPORTED;
    k<<<a->B * a->H, kSimtThreads, smem, st>>>(p);
    return launch_status();
}
template <int D>
ttt_status launch_ln_backward(const ttt_linear_backward_args* a, cudaStream_t st) {
    return a->io_dtype == TTT_F32 ? launch_ln_backward_t<D, float>(a, st)
                                  : launch_ln_backward_t<D, __nv_bfloat16>(a, st);
}
template <int D, typename IO>
ttt_status launch_linear_backward_t(const ttt_linear_backward_args* a, cudaStream_t st) {
    SimtBackwardParams p{a->H, a->T, a->b, a->Q, a->K, a->V, a->eta, a->eta_const, a->W_states,
                         a->dZ, a->dW_out, a->dQ, a->dK, a->dV, a->deta, a->dW0};
    const size_t smem = simt_backward_smem(D, a->b);
    auto k = simt_linear_backward_kernel<D, IO>;
    if (!set_smem(k, smem)) return TTT_ERR_UNSUPPORTED;
    k<<<a->B * a->H, kSimtThreads, smem, st>>>(p);
    return launch_status();
}
template <int D>
ttt_status launch_linear_backward(const ttt_linear_backward_args* a, cudaStream_t st) {
    return a->io_dtype == TTT_F32 ? launch_linear_backward_t<D, float>(a, st)
                                  : launch_linear_backward_t<D, __nv_bfloat16>(a, st);
}
}  // namespace
}  // namespace ttt

extern "C" ttt_status ttt_linear_backward(const ttt_linear_backward_args* a, cudaStream_t stream) {
    if (!a) return TTT_ERR_INVALID_ARG;
    ttt_status v = validate_common(a->B, a->H, a->T, a->d, a->b, a->io_dtype);
    if (v != TTT_OK) return v;
    const long long units = (long long)a->B * a->H;
    if (units == 0) return TTT_OK;
    if (a->T > 0 && (!ok_ptr(a->Q) || !ok_ptr(a->K) || !ok_ptr(a->V) || !ok_ptr(a->W_states) ||
                     !ok_ptr(a->dQ) || !ok_ptr(a->dK) || !ok_ptr(a->dV)))
        return TTT_ERR_INVALID_ARG;
    if (!ok_ptr(a->dW0) || !ok_opt(a->eta) || !ok_opt(a->dZ) || !ok_opt(a->dW_out) || !ok_opt(a->deta))
        return TTT_ERR_INVALID_ARG;
    if (a->flags & ~(TTT_FLAG_FORCE_SIMT | TTT_FLAG_LN_MMA_TRAINING)) return TTT_ERR_INVALID_ARG;
    if (a->use_ln != 0 && a->use_ln != 1) return TTT_ERR_INVALID_ARG;
    if (a->use_ln) {
        if ((a->T > 0 && !ok_ptr(a->c_states)) || !ok_ptr(a->ln_gamma) || !ok_ptr(a->ln_beta) ||
            !(a->ln_eps > 0.f) || !ok_opt(a->dc_out) || !ok_ptr(a->dc0) || !ok_ptr(a->dgamma) || !ok_ptr(a->dbeta))
            return TTT_ERR_INVALID_ARG;
        if ((a->flags & TTT_FLAG_LN_MMA_TRAINING) && !(a->flags & TTT_FLAG_FORCE_SIMT) && a->io_dtype == TTT_BF16 &&
            a->d == 64 && a->b == 16) {
            SimtLnBackwardParams p{a->H,      a->T,      a->b,     a->Q,      a->K,      a->V,
                                   a->eta,    a->eta_const, a->W_states, a->c_states, a->ln_gamma, a->ln_beta,
                                   a->ln_eps, a->dZ,     a->dW_out, a->dc_out, a->dQ,     a->dK,
                                   a->dV,     a->deta,   a->dW0,   a->dc0,    a->dgamma, a->dbeta};
            mbk::mma_ln_backward_kernel<<<(unsigned)units, mbk::kThreads, mbk::kLBSmemBytes, stream>>>(p);
            return launch_status();
        }
        switch (a->d) {
            case 16: return launch_ln_backward<16>(a, stream);
            case 32: return launch_ln_backward<32>(a, stream);
            default: return launch_ln_backward<64>(a, stream);
        }
    }
    if (a->io_dtype == TTT_BF16 && a->d == 64 && a->b == 16 && !(a->flags & TTT_FLAG_FORCE_SIMT)) {
        SimtBackwardParams p{a->H, a->T, a->b, a->Q, a->K, a->V, a->eta, a->eta_const, a->W_states,
                             a->dZ, a->dW_out, a->dQ, a->dK, a->dV, a->deta, a->dW0};
        mbk::mma_linear_backward_kernel<<<(unsigned)units, mbk::kThreads, mbk::kSmemBytes, stream>>>(p);
        return launch_status();
    }
    switch (a->d) {
        case 16: return launch_linear_backward<16>(a, stream);
        case 32: return launch_linear_backward<32>(a, stream);
        default: return launch_linear_backward<64>(a, stream);
    }
}

namespace ttt {
namespace {
template <int D, typename IO>
ttt_status launch_mlp_backward_t(const ttt_mlp_backward_args* a, cudaStream_t st) {
    SimtMlpBackwardParams p{a->H,       a->T,       a->b,       a->Q,       a->K,       a->V,
                            a->eta,     a->eta_const, a->W_states, a->dZ,   a->dW1_out, a->dc1_out,
                            a->dW2_out, a->dc2_out, a->dQ,      a->dK,      a->dV,      a->deta,
                            a->dW1,     a->dc1,     a->dW2,     a->dc2,     a->ln_gamma, a->ln_beta,
                            a->ln_eps,  a->dgamma,  a->dbeta};
    const size_t smem = simt_mlp_backward_smem(D, a->b, a->use_ln != 0);
    auto k = a->use_ln ? simt_mlp_backward_kernel<D, IO, true> : simt_mlp_backward_kernel<D, IO, false>;
    if (!set_smem(k, smem)) return TTT_ERR_UNSUPPORTED;
    k<<<(unsigned)(a->B * a->H), kSimtThreads, smem, st>>>(p);
    return launch_status();
}
template <int D>
ttt_status launch_mlp_backward(const ttt_mlp_backward_args* a, cudaStream_t st) {
    return a->io_dtype == TTT_F32 ? launch_mlp_backward_t<D, float>(a, st)
                                  : launch_mlp_backward_t<D, __nv_bfloat16>(a, st);
}
}  // namespace
}  // namespace ttt

extern "C" ttt_status ttt_mlp_backward(const ttt_mlp_backward_args* a, cudaStream_t stream) {
    if (!a) return TTT_ERR_INVALID_ARG;
    ttt_status v = validate_common(a->B, a->H, a->T, a->d, a->b, a->io_dtype);
    if (v != TTT_OK) return v;
    const long long units = (long long)a->B * a->H;
    if (units == 0) return TTT_OK;
    if (a->T > 0 && (!ok_ptr(a->Q) || !ok_ptr(a->K) || !ok_ptr(a->V) || !ok_ptr(a->W_states) ||
                     !ok_ptr(a->dQ) || !ok_ptr(a->dK) || !ok_ptr(a->dV)))
        return TTT_ERR_INVALID_ARG;
    if (!ok_ptr(a->dW1) || !ok_ptr(a->dc1) || !ok_ptr(a->dW2) || !ok_ptr(a->dc2)) return TTT_ERR_INVALID_ARG;
    if (!ok_opt(a->eta) || !ok_opt(a->dZ) || !ok_opt(a->deta) || !ok_opt(a->dW1_out) || !ok_opt(a->dc1_out) ||
        !ok_opt(a->dW2_out) || !ok_opt(a->dc2_out))
        return TTT_ERR_INVALID_ARG;
    if (a->flags & ~TTT_FLAG_FORCE_SIMT) return TTT_ERR_INVALID_ARG;
    if (a->use_ln != 0 && a->use_ln != 1) return TTT_ERR_INVALID_ARG;
    if (a->use_ln && (!ok_ptr(a->ln_gamma) || !ok_ptr(a->ln_beta) || !(a->ln_eps > 0.f) || !ok_ptr(a->dgamma) ||
                      !ok_ptr(a->dbeta)))
        return TTT_ERR_INVALID_ARG;
    if (a->io_dtype == TTT_BF16 && a->d == 64 && a->b == 16 && a->T > 0 && !(a->flags & TTT_FLAG_FORCE_SIMT)) {
        SimtMlpBackwardParams p{a->H,       a->T,       a->b,       a->Q,       a->K,       a->V,
                                a->eta,     a->eta_const, a->W_states, a->dZ,   a->dW1_out, a->dc1_out,
                                a->dW2_out, a->dc2_out, a->dQ,      a->dK,      a->dV,      a->deta,
                                a->dW1,     a->dc1,     a->dW2,     a->dc2,     a->ln_gamma, a->ln_beta,
                                a->ln_eps,  a->dgamma,  a->dbeta};
        auto k = a->use_ln ? mmb::mma_mlp_backward_kernel<true> : mmb::mma_mlp_backward_kernel<false>;
        if (!set_smem(k, mmb::kSmemBytes)) return TTT_ERR_CUDA;
        k<<<(unsigned)units, mmb::kThreads, mmb::kSmemBytes, stream>>>(p);
        return launch_status();
    }
    if (simt_mlp_backward_smem(a->d, a->b, a->use_ln != 0) > 227 * 1024) return TTT_ERR_UNSUPPORTED;
    switch (a->d) {
        case 16: return launch_mlp_backward<16>(a, stream);
        case 32: return launch_mlp_backward<32>(a, stream);
        default: return launch_mlp_backward<64>(a, stream);
    }
}

// ---------------------------------------------------------------------------
// Prologue: views and learning-rate gate from the layer input
// ---------------------------------------------------------------------------
extern "C" ttt_status ttt_qkv_prologue(const ttt_qkv_prologue_args* a, cudaStream_t stream) {
    if (!a) return TTT_ERR_INVALID_ARG;
    if (a->B < 0 || a->T < 0 || a->Dm <= 0 || a->H <= 0 || a->d <= 0) return TTT_ERR_INVALID_ARG;
    if (a->io_dtype != TTT_F32 && a->io_dtype != TTT_BF16) return TTT_ERR_INVALID_ARG;
    if ((a->theta_lr == nullptr) != (a->eta == nullptr)) return TTT_ERR_INVALID_ARG;
    if (a->flags & ~(TTT_FLAG_TEST_STALL | TTT_FLAG_FORCE_SIMT)) return TTT_ERR_INVALID_ARG;
    if (a->d != 16 && a->d != 32 && a->d != 64) return TTT_ERR_UNSUPPORTED;
    if (a->H > 256 || a->Dm % 8 != 0) return TTT_ERR_UNSUPPORTED;
    const long long rows = (long long)a->B * a->T;
    if (rows >= (1ll << 31)) return TTT_ERR_UNSUPPORTED;
    if (rows == 0) return TTT_OK;
    if (!ok_ptr(a->x) || !ok_ptr(a->theta_q) || !ok_ptr(a->theta_k) || !ok_ptr(a->theta_v) || !ok_ptr(a->Q) ||
        !ok_ptr(a->K) || !ok_ptr(a->V) || !ok_opt(a->theta_lr) || !ok_opt(a->eta))
        return TTT_ERR_INVALID_ARG;

    if (a->io_dtype == TTT_F32 || (a->flags & TTT_FLAG_FORCE_SIMT)) {
        // fp32 CUDA cores (every dtype); no device-side waits, so no stall hook
        if (a->flags & TTT_FLAG_TEST_STALL) return TTT_ERR_UNSUPPORTED;
        SimtPrologueParams q{(int)rows, a->T,       a->Dm, a->H, a->d, a->x, a->theta_q, a->theta_k,
                             a->theta_v, a->theta_lr, a->eta_base, a->Q, a->K, a->V, a->eta};
        const long long ncol = 3LL * a->H * a->d + (a->theta_lr ? a->H : 0);
        const dim3 grid((unsigned)((rows + kProTok - 1) / kProTok), (unsigned)((ncol + kProCols - 1) / kProCols));
        if (a->io_dtype == TTT_F32)
            simt_prologue_kernel<float><<<grid, kSimtThreads, kProSmemBytes, stream>>>(q);
        else
            simt_prologue_kernel<__nv_bfloat16><<<grid, kSimtThreads, kProSmemBytes, stream>>>(q);
        return launch_status();
    }
    using namespace pro;
    const int Hd = a->H * a->d;
    PrologueParams p;
    prologue_plan(p, rows, a->T, a->H, a->d, a->Dm, a->theta_lr != nullptr);
    p.Q = static_cast<__nv_bfloat16*>(a->Q);
    p.K = static_cast<__nv_bfloat16*>(a->K);
    p.V = static_cast<__nv_bfloat16*>(a->V);
    p.eta = a->eta;
    p.eta_base = a->eta_base;
    p.status = status_ptr();
    p.wait_ns = wait_ns(a->wait_timeout_ms);
    p.flags = a->flags;
    if (!p.status) return TTT_ERR_CUDA;

    // x [rows, Dm] and theta [Hd or H, Dm], K-major tiles of 64 model-width
    // elements (128 bytes, 128-byte swizzle); without the gate its map is a
    // copy of x's and is never read
    const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const uint64_t pitch = (uint64_t)a->Dm * 2;
    CUtensorMap mX, mTq, mTk, mTv, mTl;
    if (!encode_2d(&mX, a->x, bf, a->Dm, rows, pitch, kBK, kBM, sw) ||
        !encode_2d(&mTq, a->theta_q, bf, a->Dm, Hd, pitch, kBK, p.brows, sw) ||
        !encode_2d(&mTk, a->theta_k, bf, a->Dm, Hd, pitch, kBK, p.brows, sw) ||
        !encode_2d(&mTv, a->theta_v, bf, a->Dm, Hd, pitch, kBK, p.brows, sw))
        return TTT_ERR_CUDA;
    if (a->theta_lr) {
        if (!encode_2d(&mTl, a->theta_lr, bf, a->Dm, a->H, pitch, kBK, p.ng, sw)) return TTT_ERR_CUDA;
    } else {
        mTl = mX;
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return TTT_ERR_CUDA;
    const int grid = (int)(p.tiles < sms ? p.tiles : sms);
    if (!set_smem(prologue_kernel, kSmemBytes)) return TTT_ERR_CUDA;
    prologue_kernel<<<grid, kThreads, kSmemBytes, stream>>>(mX, mTq, mTk, mTv, mTl, p);
    return launch_status();
}

extern "C" const char* ttt_status_string(ttt_status s) {
    switch (s) {
        case TTT_OK: return "TTT_OK";
        case TTT_ERR_INVALID_ARG: return "TTT_ERR_INVALID_ARG";
        case TTT_ERR_UNSUPPORTED: return "TTT_ERR_UNSUPPORTED";
        case TTT_ERR_CUDA: return "TTT_ERR_CUDA";
        case TTT_ERR_TIMEOUT: return "TTT_ERR_TIMEOUT";
    }
    return "TTT_ERR_UNKNOWN";
}

extern "C" ttt_status ttt_last_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return TTT_ERR_CUDA;
    int* p = status_ptr();
    if (!p) return TTT_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TTT_ERR_CUDA;
    if (h != 0) {
        const int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return TTT_ERR_CUDA;
    }
    if (h & kStatusBadSmem) return TTT_ERR_CUDA;
    return (h & kStatusTimeout) ? TTT_ERR_TIMEOUT : TTT_OK;
}

extern "C" const char* ttt_version(void) { return "ttt-b200 0.1.0 (sm_100a)"; }
