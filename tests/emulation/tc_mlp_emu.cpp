// Entry point of the CPU tests' host emulation of the TTT-MLP tensor-core
// kernel (tcgen05, M = 128 and M = 64 accumulators, TMEM-resident state):
// TEST INFRASTRUCTURE; the library has no CPU path.  The kernel is the one
// already verified on the B200, so this run pins the emulated M = 64
// accumulator layout, MN-major A operands, the 16x128b TMEM store and the
// x2 ldmatrix / stmatrix forms to hardware behaviour.
#include "tc_emu_mtc.h"

namespace ttt {
namespace mtc {
alignas(1024) uint8_t smem[160 * 1024];
}
}  // namespace ttt

#include "../../test_sequence_layers_head_b200/csrc/mlp_tc.cuh"

// test knobs: launch flags and the wait limit of the next run (the stall hook
// TTT_FLAG_TEST_STALL makes the MMA issuer wait on a barrier nothing arrives on)
static unsigned g_flags = 0;
static unsigned long long g_wait_ns = 120ull * 1000000000ull;   // generous: the emulated threads share few host cores
extern "C" void emu_mlp_tc_knobs(unsigned flags, unsigned long long wait_ns) {
    g_flags = flags;
    g_wait_ns = wait_ns;
}
// deferred completion of the asynchronous operations (tc_emu.h, Engine) for the next runs
extern "C" void emu_deferred(int on) { emu::deferred = on != 0; }

// The TTT-MLP prefill (plain or LN+residual on the output layer) with the
// library's tensor maps, parameters and grid (one unit per CTA).  Returns the
// number of emulated-hardware rule violations (0 when none), or -1 for a bad
// request.
extern "C" int emu_mlp_tc(int ln, int B, int H, int T, int per_seq, const void* Q, const void* K, const void* V,
                          const float* eta, float eta_const, const float* W1, const float* c1, const float* W2,
                          const float* c2, const float* gamma, const float* beta, float eps, void* Z, float* W1_out,
                          float* c1_out, float* W2_out, float* c2_out, int* status) {
    using namespace ttt::mtc;
    if (T < kTok || T % kTok || static_cast<int>(sizeof(smem)) < kSmemBytes) return -1;
    const long long U = (long long)B * H, rows = U * T;
    CUtensorMap mQ, mK, mV;
    emu::make_map(&mQ, Q, kD, rows, kD * 2, kD, kTok, 2);
    emu::make_map(&mK, K, kD, rows, kD * 2, kD, kTok, 2);
    emu::make_map(&mV, V, kD, rows, kD * 2, kD, kTok, 2);
    Params p{};
    p.H = H;
    p.T = T;
    p.nsteps = T / kTok;
    p.per_seq = per_seq;
    p.eta = eta;
    p.eta_const = eta_const;
    p.W1 = W1;
    p.c1 = c1;
    p.W2 = W2;
    p.c2 = c2;
    p.Z = static_cast<__nv_bfloat16*>(Z);
    p.W1_out = W1_out;
    p.c1_out = c1_out;
    p.W2_out = W2_out;
    p.c2_out = c2_out;
    p.status = status;
    p.wait_ns = g_wait_ns;
    p.flags = g_flags;
    p.gamma = gamma;
    p.beta = beta;
    p.eps = eps;
    emu::errors = 0;
    emu::reset_named();
    if (ln)
        emu::run_grid_bounded((int)U, kThreads, smem, kSmemBytes, sizeof(smem), [&] { mlp_tc_kernel<true>(mQ, mK, mV, p); });
    else
        emu::run_grid_bounded((int)U, kThreads, smem, kSmemBytes, sizeof(smem), [&] { mlp_tc_kernel<false>(mQ, mK, mV, p); });
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
