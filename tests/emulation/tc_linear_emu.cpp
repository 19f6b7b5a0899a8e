// Entry point of the CPU tests' host emulation of the TTT-Linear tensor-core
// kernel (tcgen05 with TMEM-resident state, TMA loads and stores, mma.sync
// epilogue): TEST INFRASTRUCTURE; the library has no CPU path.  The kernel is
// the one already verified on the B200, so this run pins the emulated tcgen05
// semantics (operand descriptors, TMEM loads and stores, the accumulator
// layout of the 16x256b load, the swizzled TMA store) to hardware behaviour.
#include "tc_emu_lfr.h"

namespace ttt {
namespace lfr {
alignas(1024) uint8_t smem[128 * 1024];
}
}  // namespace ttt

#include "../../test_sequence_layers_head_b200/csrc/linear_frag.cuh"

// test knobs: launch flags and the wait limit of the next run (the stall hook
// TTT_FLAG_TEST_STALL makes the MMA issuer wait on a barrier nothing arrives on)
static unsigned g_flags = 0;
static unsigned long long g_wait_ns = 120ull * 1000000000ull;   // generous: the emulated threads share few host cores
extern "C" void emu_linear_tc_knobs(unsigned flags, unsigned long long wait_ns) {
    g_flags = flags;
    g_wait_ns = wait_ns;
}
// deferred completion of the asynchronous operations (tc_emu.h, Engine) for the next runs
extern "C" void emu_deferred(int on) { emu::deferred = on != 0; }

// The TTT-Linear prefill (plain or LN+residual) with the library's tensor maps,
// parameters and grid; upc = units per CTA (1 or 2).  Returns the number of
// emulated-hardware rule violations (0 when none), or -1 for a bad request.
extern "C" int emu_linear_tc(int ln, int upc, int B, int H, int T, const void* Q, const void* K, const void* V,
                             const float* eta, float eta_const, const float* W0, long long W0_bstride,
                             const float* c0, long long c0_bstride, const float* gamma, const float* beta, float eps,
                             void* Z, float* W_out, float* c_out, int* status) {
    using namespace ttt::lfr;
    if (T < kTok || T % kTok || (upc != 1 && upc != 2) || static_cast<int>(sizeof(smem)) < kSmemBytes) return -1;
    const long long U = (long long)B * H, rows = U * T;
    CUtensorMap mQ, mK, mV, mZ, mZ1;
    emu::make_map(&mQ, Q, kD, rows, kD * 2, kD, kTok, 2);
    emu::make_map(&mK, K, kD, rows, kD * 2, kD, kTok, 2);
    emu::make_map(&mV, V, kD, rows, kD * 2, kD, kTok, 2);
    const unsigned zcols = upc == 1 ? 16 : 32;
    emu::make_map_swz(&mZ, Z, kD, rows, kD * 2, zcols, 2 * kTok, 2, 2 * zcols);
    emu::make_map_swz(&mZ1, Z, kD, rows, kD * 2, zcols, kTok, 2, 2 * zcols);
    Params p{};
    p.U = (int)U;
    p.H = H;
    p.T = T;
    p.nsteps = T / kTok;
    p.eta = eta;
    p.eta_const = eta_const;
    p.W0 = W0;
    p.W0_bstride = W0_bstride;
    p.c0 = c0;
    p.c0_bstride = c0_bstride;
    p.gamma = gamma;
    p.beta = beta;
    p.eps = eps;
    p.Z = static_cast<__nv_bfloat16*>(Z);
    p.W_out = W_out;
    p.c_out = c_out;
    p.status = status;
    p.wait_ns = g_wait_ns;
    p.flags = g_flags;
    emu::errors = 0;
    emu::reset_named();
    const int grid = upc == 1 ? (int)U : (int)((U + 1) / 2);
    if (ln) {
        if (upc == 1)
            emu::run_grid_bounded(grid, kThreads, smem, kSmemBytes, sizeof(smem), [&] { linear_frag_kernel<true, 1>(mQ, mK, mV, mZ, mZ1, p); });
        else
            emu::run_grid_bounded(grid, kThreads, smem, kSmemBytes, sizeof(smem), [&] { linear_frag_kernel<true, 2>(mQ, mK, mV, mZ, mZ1, p); });
    } else {
        if (upc == 1)
            emu::run_grid_bounded(grid, kThreads, smem, kSmemBytes, sizeof(smem), [&] { linear_frag_kernel<false, 1>(mQ, mK, mV, mZ, mZ1, p); });
        else
            emu::run_grid_bounded(grid, kThreads, smem, kSmemBytes, sizeof(smem), [&] { linear_frag_kernel<false, 2>(mQ, mK, mV, mZ, mZ1, p); });
    }
    emu::reset_named();
    emu::engine.finish();
    for (int t = 0; t < emu::kMaxThreads; ++t) emu::flush_stores(t);
    return emu::errors.load();
}

// serial scheduling of the next runs (emu_core.h: 0 off, 1 ascending, 2 descending thread order), and the
// number of runs since the last call in which every live thread was blocked (a hang on the GPU)
extern "C" void emu_serial(int mode) { emu::serial = mode; }
extern "C" int emu_sched_errors() { return emu::sched_errors.exchange(0); }

// shared-memory overruns (accesses beyond the launch's dynamic size) since the last call
extern "C" int emu_smem_overruns() { return emu::smem_overruns.exchange(0); }
