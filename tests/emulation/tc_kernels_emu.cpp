// Entry points of the CPU tests' host emulation of the tensor-core (tcgen05)
// kernels (tc_emu.h and emu_core.h have the execution model): TEST
// INFRASTRUCTURE; the library has no CPU path.
#include "tc_emu.h"

namespace ttt {
namespace pro {
alignas(1024) uint8_t smem[4 * 65536];
}
}  // namespace ttt

#include "../../test_sequence_layers_head_b200/csrc/prologue.cuh"

// test knobs: launch flags and the wait limit of the next run (the stall hook
// TTT_FLAG_TEST_STALL makes the MMA issuer wait on a barrier nothing arrives on)
static unsigned g_flags = 0;
static unsigned long long g_wait_ns = 120ull * 1000000000ull;   // generous: the emulated threads share few host cores
extern "C" void emu_prologue_tc_knobs(unsigned flags, unsigned long long wait_ns) {
    g_flags = flags;
    g_wait_ns = wait_ns;
}
// deferred completion of the asynchronous operations (tc_emu.h, Engine) for the next runs
extern "C" void emu_deferred(int on) { emu::deferred = on != 0; }

// the fused prologue on tcgen05 with the library's tile plan and tensor maps, on `grid` persistent CTAs;
// returns the number of emulated-hardware rule violations (0 when none), or -1 for a bad request
extern "C" int emu_prologue_tc(int B, int T, int Dm, int H, int d, const void* x, const void* tq, const void* tk,
                               const void* tv, const void* tl, float eta_base, void* Q, void* K, void* V,
                               float* eta, int grid, int* status) {
    using namespace ttt::pro;
    const long long rows = (long long)B * T;
    if (rows == 0 || Dm % 8 || H > 256) return -1;
    PrologueParams p{};
    prologue_plan(p, rows, T, H, d, Dm, tl != nullptr);
    p.Q = static_cast<__nv_bfloat16*>(Q);
    p.K = static_cast<__nv_bfloat16*>(K);
    p.V = static_cast<__nv_bfloat16*>(V);
    p.eta = eta;
    p.eta_base = eta_base;
    p.status = status;
    p.wait_ns = g_wait_ns;
    p.flags = g_flags;
    const unsigned long long pitch = (unsigned long long)Dm * 2;
    CUtensorMap mX, mTq, mTk, mTv, mTl;
    emu::make_map(&mX, x, Dm, rows, pitch, kBK, kBM, 2);
    emu::make_map(&mTq, tq, Dm, p.Hd, pitch, kBK, p.brows, 2);
    emu::make_map(&mTk, tk, Dm, p.Hd, pitch, kBK, p.brows, 2);
    emu::make_map(&mTv, tv, Dm, p.Hd, pitch, kBK, p.brows, 2);
    if (tl)
        emu::make_map(&mTl, tl, Dm, H, pitch, kBK, p.ng, 2);
    else
        mTl = mX;
    const int g = (int)(p.tiles < grid ? p.tiles : grid);
    emu::errors = 0;
    // a persistent CTA walks tiles blockIdx.x, blockIdx.x + gridDim.x, ...: gridDim must be the grid
    emu::run_grid_bounded(g, kThreads, smem, kSmemBytes, sizeof(smem), [&] { prologue_kernel(mX, mTq, mTk, mTv, mTl, p); });
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
