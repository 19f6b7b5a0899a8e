// Entry points of the CPU tests' host emulation of the library's kernels
// (emu_core.h has the execution model): TEST INFRASTRUCTURE; the library has
// no CPU path.  Each entry point runs a kernel pair on host arrays exactly as
// the library launches it on a GPU (one CTA per unit).
#include "emu_core.h"

// the kernels' dynamic shared arrays
namespace ttt {
alignas(1024) float sm[65536];
namespace mbk {
alignas(1024) uint8_t smem[65536];
}
namespace mmb {
alignas(1024) uint8_t smem[4 * 65536];
}
}  // namespace ttt

#include "../../test_sequence_layers_head_b200/csrc/simt.cuh"
#include "../../test_sequence_layers_head_b200/csrc/simt_mlp_backward.cuh"
#include "../../test_sequence_layers_head_b200/csrc/mma_forward.cuh"
#include "../../test_sequence_layers_head_b200/csrc/mma_ln.cuh"
#include "../../test_sequence_layers_head_b200/csrc/simt_prologue.cuh"
#include "../../test_sequence_layers_head_b200/csrc/mma_mlp_backward.cuh"

namespace {

// TTT-MLP forward writing the batch-start states, then the backward from them
template <int D, typename IO>
int train(int B, int H, int T, int b, const IO* Q, const IO* K, const IO* V, const float* eta, float eta_const,
          const float* W1, const float* c1, const float* W2, const float* c2, const IO* dZ, const float* dW1o,
          const float* dc1o, const float* dW2o, const float* dc2o, IO* Z, float* W1_out, float* c1_out, float* W2_out,
          float* c2_out, float* W_states, IO* dQ, IO* dK, IO* dV, float* deta, float* dW1, float* dc1, float* dW2,
          float* dc2) {
    if (ttt::simt_mlp_smem(D, b, false) > sizeof(ttt::sm) || ttt::simt_mlp_backward_smem(D, b) > sizeof(ttt::sm))
        return 2;
    ttt::SimtMlpParams p{};
    p.H = H;
    p.T = T;
    p.b = b;
    p.Q = Q;
    p.K = K;
    p.V = V;
    p.eta = eta;
    p.eta_const = eta_const;
    p.W1 = W1;
    p.c1 = c1;
    p.W2 = W2;
    p.c2 = c2;
    p.per_seq = 0;
    p.Z = Z;
    p.W1_out = W1_out;
    p.c1_out = c1_out;
    p.W2_out = W2_out;
    p.c2_out = c2_out;
    p.W_states = W_states;
    emu::run_grid_bounded(B * H, ttt::kSimtThreads, ttt::sm, ttt::simt_mlp_smem(D, b, false), sizeof(ttt::sm),
                          [&] { ttt::simt_mlp_kernel<D, IO, false>(p); });
    ttt::SimtMlpBackwardParams q{H,  T,  b,  Q,     K,     V,     eta,  eta_const, W_states, dZ,  dW1o,
                                 dc1o, dW2o, dc2o, dQ, dK, dV, deta, dW1, dc1, dW2, dc2};
    emu::run_grid_bounded(B * H, ttt::kSimtThreads, ttt::sm, ttt::simt_mlp_backward_smem(D, b), sizeof(ttt::sm),
                          [&] { ttt::simt_mlp_backward_kernel<D, IO>(q); });
    return 0;
}

}  // namespace

#define TRAIN_ARGS                                                                                                \
    B, H, T, b, static_cast<const IO*>(Q), static_cast<const IO*>(K), static_cast<const IO*>(V), eta, eta_const, \
        W1, c1, W2, c2, static_cast<const IO*>(dZ), dW1o, dc1o, dW2o, dc2o, static_cast<IO*>(Z), W1_out, c1_out,  \
        W2_out, c2_out, W_states, static_cast<IO*>(dQ), static_cast<IO*>(dK), static_cast<IO*>(dV), deta, dW1,   \
        dc1, dW2, dc2

// io: 0 = fp32, 1 = bf16 (Q, K, V, dZ, Z, dQ, dK, dV)
extern "C" int emu_mlp_train(int io, int B, int H, int T, int d, int b, const void* Q, const void* K, const void* V,
                             const float* eta, float eta_const, const float* W1, const float* c1, const float* W2,
                             const float* c2, const void* dZ, const float* dW1o, const float* dc1o, const float* dW2o,
                             const float* dc2o, void* Z, float* W1_out, float* c1_out, float* W2_out, float* c2_out,
                             float* W_states, void* dQ, void* dK, void* dV, float* deta, float* dW1, float* dc1,
                             float* dW2, float* dc2) {
    if (io == 0) {
        using IO = float;
        switch (d) {
            case 16: return train<16, IO>(TRAIN_ARGS);
            case 32: return train<32, IO>(TRAIN_ARGS);
            case 64: return train<64, IO>(TRAIN_ARGS);
        }
    } else {
        using IO = __nv_bfloat16;
        switch (d) {
            case 16: return train<16, IO>(TRAIN_ARGS);
            case 32: return train<32, IO>(TRAIN_ARGS);
            case 64: return train<64, IO>(TRAIN_ARGS);
        }
    }
    return 1;
}

// TTT-Linear training on the tensor-core (mma.sync) kernels, bf16, d = 64, b = 16:
// the forward writing the batch-start states, then the backward
extern "C" int emu_linear_train_mma(int B, int H, int T, const void* Q, const void* K, const void* V,
                                    const float* eta, float eta_const, const float* W0, long long W0_bstride,
                                    void* Z, float* W_out, float* W_states, const void* dZ, const float* dW_out,
                                    void* dQ, void* dK, void* dV, float* deta, float* dW0) {
    using namespace ttt::mbk;
    if (kFSmemBytes > (int)sizeof(smem) || kSmemBytes > (int)sizeof(smem)) return 2;
    FwdStatesParams f{H, T, Q, K, V, eta, eta_const, W0, W0_bstride, Z, W_out, W_states};
    emu::run_grid_bounded(B * H, kThreads, smem, kFSmemBytes, sizeof(smem), [&] { mma_linear_forward_states_kernel(f); });
    ttt::SimtBackwardParams p{H, T, 16, Q, K, V, eta, eta_const, W_states, dZ, dW_out, dQ, dK, dV, deta, dW0};
    emu::run_grid_bounded(B * H, kThreads, smem, kSmemBytes, sizeof(smem), [&] { mma_linear_backward_kernel(p); });
    return 0;
}

// TTT-Linear with LN+residual on the tensor-core (mma.sync) kernels, bf16, d = 64, b = 16: the forward
// writing the batch-start states (W, c)
extern "C" int emu_ln_forward_mma(int B, int H, int T, const void* Q, const void* K, const void* V, const float* eta,
                                  float eta_const, const float* W0, const float* c0, const float* gamma,
                                  const float* beta, float eps, void* Z, float* W_out, float* c_out, float* W_states,
                                  float* c_states) {
    using namespace ttt::mbk;
    if (kLFSmemBytes > (int)sizeof(smem)) return 2;
    FwdLnStatesParams f{H, T, Q, K, V, eta, eta_const, W0, 0, c0, 0, gamma, beta, eps, Z, W_out, c_out,
                        W_states, c_states};
    emu::run_grid_bounded(B * H, kThreads, smem, kLFSmemBytes, sizeof(smem), [&] { mma_ln_forward_states_kernel(f); });
    return 0;
}

// TTT-Linear with LN+residual on the tensor-core (mma.sync) kernels: the forward writing the batch-start
// states, then the backward from them
extern "C" int emu_ln_train_mma(int B, int H, int T, const void* Q, const void* K, const void* V, const float* eta,
                                float eta_const, const float* W0, const float* c0, const float* gamma,
                                const float* beta, float eps, float* W_out, float* c_out, float* W_states,
                                float* c_states, const void* dZ, const float* dW_out, const float* dc_out, void* dQ,
                                void* dK, void* dV, float* deta, float* dW0, float* dc0, float* dgamma,
                                float* dbeta) {
    using namespace ttt::mbk;
    if (kLFSmemBytes > (int)sizeof(smem) || kLBSmemBytes > (int)sizeof(smem)) return 2;
    FwdLnStatesParams f{H, T, Q, K, V, eta, eta_const, W0, 0, c0, 0, gamma, beta, eps, nullptr, W_out, c_out,
                        W_states, c_states};
    emu::run_grid_bounded(B * H, kThreads, smem, kLFSmemBytes, sizeof(smem), [&] { mma_ln_forward_states_kernel(f); });
    ttt::SimtLnBackwardParams q{H,  T,  16, Q,  K,      V,      eta,    eta_const, W_states, c_states, gamma, beta,
                                eps, dZ, dW_out, dc_out, dQ, dK, dV, deta, dW0, dc0, dgamma, dbeta};
    emu::run_grid_bounded(B * H, kThreads, smem, kLBSmemBytes, sizeof(smem), [&] { mma_ln_backward_kernel(q); });
    return 0;
}

// The same kernels one launch at a time (the tests' dry runs call them as the library would)
extern "C" int emu_mlp_forward(int io, int B, int H, int T, int d, int b, const void* Q, const void* K, const void* V,
                               const float* eta, float eta_const, const float* W1, const float* c1, const float* W2,
                               const float* c2, void* Z, float* W1_out, float* c1_out, float* W2_out, float* c2_out,
                               float* W_states) {
    ttt::SimtMlpParams p{};
    p.H = H;
    p.T = T;
    p.b = b;
    p.Q = Q;
    p.K = K;
    p.V = V;
    p.eta = eta;
    p.eta_const = eta_const;
    p.W1 = W1;
    p.c1 = c1;
    p.W2 = W2;
    p.c2 = c2;
    p.Z = Z;
    p.W1_out = W1_out;
    p.c1_out = c1_out;
    p.W2_out = W2_out;
    p.c2_out = c2_out;
    p.W_states = W_states;
    if (ttt::simt_mlp_smem(d, b, false) > sizeof(ttt::sm)) return 2;
    auto run = [&](auto kernel) {
        emu::run_grid_bounded(B * H, ttt::kSimtThreads, ttt::sm, ttt::simt_mlp_smem(d, b, false), sizeof(ttt::sm),
                              [&] { kernel(p); });
    };
    if (io == 0) {
        if (d == 16) run(ttt::simt_mlp_kernel<16, float, false>);
        else if (d == 32) run(ttt::simt_mlp_kernel<32, float, false>);
        else run(ttt::simt_mlp_kernel<64, float, false>);
    } else {
        if (d == 16) run(ttt::simt_mlp_kernel<16, __nv_bfloat16, false>);
        else if (d == 32) run(ttt::simt_mlp_kernel<32, __nv_bfloat16, false>);
        else run(ttt::simt_mlp_kernel<64, __nv_bfloat16, false>);
    }
    return 0;
}
extern "C" int emu_mlp_backward(int io, int B, int H, int T, int d, int b, const void* Q, const void* K,
                                const void* V, const float* eta, float eta_const, const float* W_states,
                                const void* dZ, const float* dW1o, const float* dc1o, const float* dW2o,
                                const float* dc2o, void* dQ, void* dK, void* dV, float* deta, float* dW1, float* dc1,
                                float* dW2, float* dc2) {
    ttt::SimtMlpBackwardParams q{H,    T,    b,  Q,  K,  V,    eta, eta_const, W_states, dZ,  dW1o,
                                 dc1o, dW2o, dc2o, dQ, dK, dV, deta, dW1,      dc1,      dW2, dc2};
    if (ttt::simt_mlp_backward_smem(d, b) > sizeof(ttt::sm)) return 2;
    auto run = [&](auto kernel) {
        emu::run_grid_bounded(B * H, ttt::kSimtThreads, ttt::sm, ttt::simt_mlp_backward_smem(d, b), sizeof(ttt::sm),
                              [&] { kernel(q); });
    };
    if (io == 0) {
        if (d == 16) run(ttt::simt_mlp_backward_kernel<16, float>);
        else if (d == 32) run(ttt::simt_mlp_backward_kernel<32, float>);
        else run(ttt::simt_mlp_backward_kernel<64, float>);
    } else {
        if (d == 16) run(ttt::simt_mlp_backward_kernel<16, __nv_bfloat16>);
        else if (d == 32) run(ttt::simt_mlp_backward_kernel<32, __nv_bfloat16>);
        else run(ttt::simt_mlp_backward_kernel<64, __nv_bfloat16>);
    }
    return 0;
}
extern "C" int emu_ln_backward_mma(int B, int H, int T, const void* Q, const void* K, const void* V, const float* eta,
                                   float eta_const, const float* W_states, const float* c_states, const float* gamma,
                                   const float* beta, float eps, const void* dZ, const float* dW_out,
                                   const float* dc_out, void* dQ, void* dK, void* dV, float* deta, float* dW0,
                                   float* dc0, float* dgamma, float* dbeta) {
    using namespace ttt::mbk;
    ttt::SimtLnBackwardParams q{H,  T,  16, Q,  K,      V,      eta,    eta_const, W_states, c_states, gamma, beta,
                                eps, dZ, dW_out, dc_out, dQ, dK, dV, deta, dW0, dc0, dgamma, dbeta};
    emu::run_grid_bounded(B * H, kThreads, smem, kLBSmemBytes, sizeof(smem), [&] { mma_ln_backward_kernel(q); });
    return 0;
}

// the fused prologue on fp32 CUDA cores (grid: token blocks x column blocks, run as one flat loop of CTAs)
extern "C" int emu_prologue_simt(int io, int B, int T, int Dm, int H, int d, const void* x, const void* tq,
                                 const void* tk, const void* tv, const void* tl, float eta_base, void* Q, void* K,
                                 void* V, float* eta) {
    const int rows = B * T;
    if (rows == 0) return 0;
    ttt::SimtPrologueParams q{rows, T, Dm, H, d, x, tq, tk, tv, tl, eta_base, Q, K, V, eta};
    const long long ncol = 3LL * H * d + (tl ? H : 0);
    const int gx = (rows + ttt::kProTok - 1) / ttt::kProTok, gy = (int)((ncol + ttt::kProCols - 1) / ttt::kProCols);
    emu::run_grid_bounded(gx * gy, ttt::kSimtThreads, ttt::sm, ttt::kProSmemBytes, sizeof(ttt::sm), [&] {
        const unsigned flat = emu::bid3.x;
        emu::bid3 = make_uint3(flat % gx, flat / gx, 0);
        if (io == 0)
            ttt::simt_prologue_kernel<float>(q);
        else
            ttt::simt_prologue_kernel<__nv_bfloat16>(q);
    });
    return 0;
}

// the TTT-MLP backward on mma.sync (bf16, d = 64, b = 16), from states written by the CUDA-core forward
extern "C" int emu_mlp_backward_mma(int B, int H, int T, const void* Q, const void* K, const void* V,
                                    const float* eta, float eta_const, const float* W_states, const void* dZ,
                                    const float* dW1o, const float* dc1o, const float* dW2o, const float* dc2o,
                                    void* dQ, void* dK, void* dV, float* deta, float* dW1, float* dc1, float* dW2,
                                    float* dc2) {
    static_assert(ttt::mmb::kSmemBytes <= (int)sizeof(ttt::mmb::smem), "emulated shared memory");
    ttt::SimtMlpBackwardParams q{H,    T,    16, Q,  K,  V,    eta, eta_const, W_states, dZ,  dW1o,
                                 dc1o, dW2o, dc2o, dQ, dK, dV, deta, dW1,      dc1,      dW2, dc2};
    emu::run_grid_bounded(B * H, ttt::mmb::kThreads, ttt::mmb::smem, ttt::mmb::kSmemBytes, sizeof(ttt::mmb::smem), [&] { ttt::mmb::mma_mlp_backward_kernel<false>(q); });
    return 0;
}

// the TTT-MLP forward writing the batch-start states on mma.sync (bf16, d = 64, b = 16)
extern "C" int emu_mlp_forward_mma(int B, int H, int T, const void* Q, const void* K, const void* V, const float* eta,
                                   float eta_const, const float* W1, const float* c1, const float* W2,
                                   const float* c2, void* Z, float* W1_out, float* c1_out, float* W2_out,
                                   float* c2_out, float* W_states) {
    ttt::mmb::MlpFwdStatesParams f{H,  T,      Q,      K,      V,      eta,    eta_const, W1,      c1,
                                   W2, c2,     0,      Z,      W1_out, c1_out, W2_out,    c2_out, W_states};
    emu::run_grid_bounded(B * H, ttt::mmb::kThreads, ttt::mmb::smem, ttt::mmb::kSmemBytes, sizeof(ttt::mmb::smem), [&] { ttt::mmb::mma_mlp_forward_states_kernel<false>(f); });
    return 0;
}

// TTT-MLP with LN+residual on fp32 CUDA cores: the forward writing the batch-start states, then the backward
extern "C" int emu_mlp_ln_train(int io, int B, int H, int T, int d, int b, const void* Q, const void* K,
                                const void* V, const float* eta, float eta_const, const float* W1, const float* c1,
                                const float* W2, const float* c2, const float* gamma, const float* beta, float eps,
                                const void* dZ, const float* dW1o, const float* dc1o, const float* dW2o,
                                const float* dc2o, float* W_states, void* dQ, void* dK, void* dV, float* deta,
                                float* dW1, float* dc1, float* dW2, float* dc2, float* dgamma, float* dbeta) {
    std::vector<uint8_t> Z((size_t)B * H * T * d * (io ? 2 : 4) + 16);
    std::vector<float> W1o((size_t)B * H * d * 4 * d), c1o((size_t)B * H * 4 * d), W2o((size_t)B * H * 4 * d * d),
        c2o((size_t)B * H * d);
    ttt::SimtMlpParams f{};
    f.H = H;
    f.T = T;
    f.b = b;
    f.Q = Q;
    f.K = K;
    f.V = V;
    f.eta = eta;
    f.eta_const = eta_const;
    f.W1 = W1;
    f.c1 = c1;
    f.W2 = W2;
    f.c2 = c2;
    f.Z = Z.data();
    f.W1_out = W1o.data();
    f.c1_out = c1o.data();
    f.W2_out = W2o.data();
    f.c2_out = c2o.data();
    f.gamma = gamma;
    f.beta = beta;
    f.eps = eps;
    f.W_states = W_states;
    ttt::SimtMlpBackwardParams q{H,    T,    b,  Q,  K,  V,    eta, eta_const, W_states, dZ,  dW1o,
                                 dc1o, dW2o, dc2o, dQ, dK, dV, deta, dW1,      dc1,      dW2, dc2,
                                 gamma, beta, eps, dgamma, dbeta};
    if (ttt::simt_mlp_smem(d, b, true) > sizeof(ttt::sm) || ttt::simt_mlp_backward_smem(d, b, true) > sizeof(ttt::sm))
        return 2;
    auto go = [&](auto fwd, auto bwd) {
        emu::run_grid_bounded(B * H, ttt::kSimtThreads, ttt::sm, ttt::simt_mlp_smem(d, b, true), sizeof(ttt::sm),
                              [&] { fwd(f); });
        emu::run_grid_bounded(B * H, ttt::kSimtThreads, ttt::sm, ttt::simt_mlp_backward_smem(d, b, true),
                              sizeof(ttt::sm), [&] { bwd(q); });
    };
    if (io == 0) {
        if (d == 16) go(ttt::simt_mlp_kernel<16, float, true>, ttt::simt_mlp_backward_kernel<16, float, true>);
        else if (d == 32) go(ttt::simt_mlp_kernel<32, float, true>, ttt::simt_mlp_backward_kernel<32, float, true>);
        else go(ttt::simt_mlp_kernel<64, float, true>, ttt::simt_mlp_backward_kernel<64, float, true>);
    } else {
        if (d == 16)
            go(ttt::simt_mlp_kernel<16, __nv_bfloat16, true>, ttt::simt_mlp_backward_kernel<16, __nv_bfloat16, true>);
        else
            go(ttt::simt_mlp_kernel<64, __nv_bfloat16, true>, ttt::simt_mlp_backward_kernel<64, __nv_bfloat16, true>);
    }
    return 0;
}

// the two launches of emu_mlp_ln_train one at a time (the tests' dry runs call them as the library would)
extern "C" int emu_mlp_ln_forward(int io, int B, int H, int T, int d, int b, const void* Q, const void* K,
                                  const void* V, const float* eta, float eta_const, const float* W1, const float* c1,
                                  const float* W2, const float* c2, const float* gamma, const float* beta, float eps,
                                  void* Z, float* W1_out, float* c1_out, float* W2_out, float* c2_out,
                                  float* W_states) {
    ttt::SimtMlpParams f{};
    f.H = H;
    f.T = T;
    f.b = b;
    f.Q = Q;
    f.K = K;
    f.V = V;
    f.eta = eta;
    f.eta_const = eta_const;
    f.W1 = W1;
    f.c1 = c1;
    f.W2 = W2;
    f.c2 = c2;
    f.Z = Z;
    f.W1_out = W1_out;
    f.c1_out = c1_out;
    f.W2_out = W2_out;
    f.c2_out = c2_out;
    f.gamma = gamma;
    f.beta = beta;
    f.eps = eps;
    f.W_states = W_states;
    auto run = [&](auto kernel) {
        emu::run_grid_bounded(B * H, ttt::kSimtThreads, ttt::sm, ttt::simt_mlp_smem(d, b, true), sizeof(ttt::sm),
                              [&] { kernel(f); });
    };
    if (io == 0) {
        if (d == 16) run(ttt::simt_mlp_kernel<16, float, true>);
        else if (d == 32) run(ttt::simt_mlp_kernel<32, float, true>);
        else run(ttt::simt_mlp_kernel<64, float, true>);
    } else {
        if (d == 16) run(ttt::simt_mlp_kernel<16, __nv_bfloat16, true>);
        else if (d == 32) run(ttt::simt_mlp_kernel<32, __nv_bfloat16, true>);
        else run(ttt::simt_mlp_kernel<64, __nv_bfloat16, true>);
    }
    return 0;
}
extern "C" int emu_mlp_ln_backward(int io, int B, int H, int T, int d, int b, const void* Q, const void* K,
                                   const void* V, const float* eta, float eta_const, const float* W_states,
                                   const void* dZ, const float* dW1o, const float* dc1o, const float* dW2o,
                                   const float* dc2o, const float* gamma, const float* beta, float eps, void* dQ,
                                   void* dK, void* dV, float* deta, float* dW1, float* dc1, float* dW2, float* dc2,
                                   float* dgamma, float* dbeta) {
    ttt::SimtMlpBackwardParams q{H,    T,    b,  Q,  K,  V,    eta, eta_const, W_states, dZ,  dW1o,
                                 dc1o, dW2o, dc2o, dQ, dK, dV, deta, dW1,      dc1,      dW2, dc2,
                                 gamma, beta, eps, dgamma, dbeta};
    auto run = [&](auto kernel) {
        emu::run_grid_bounded(B * H, ttt::kSimtThreads, ttt::sm, ttt::simt_mlp_backward_smem(d, b, true),
                              sizeof(ttt::sm), [&] { kernel(q); });
    };
    if (io == 0) {
        if (d == 16) run(ttt::simt_mlp_backward_kernel<16, float, true>);
        else if (d == 32) run(ttt::simt_mlp_backward_kernel<32, float, true>);
        else run(ttt::simt_mlp_backward_kernel<64, float, true>);
    } else {
        if (d == 16) run(ttt::simt_mlp_backward_kernel<16, __nv_bfloat16, true>);
        else if (d == 32) run(ttt::simt_mlp_backward_kernel<32, __nv_bfloat16, true>);
        else run(ttt::simt_mlp_backward_kernel<64, __nv_bfloat16, true>);
    }
    return 0;
}

// the TTT-MLP with LN+residual backward on mma.sync (bf16, d = 64, b = 16), from the CUDA-core LN forward's states
extern "C" int emu_mlp_ln_backward_mma(int B, int H, int T, const void* Q, const void* K, const void* V,
                                       const float* eta, float eta_const, const float* W_states, const void* dZ,
                                       const float* dW1o, const float* dc1o, const float* dW2o, const float* dc2o,
                                       const float* gamma, const float* beta, float eps, void* dQ, void* dK,
                                       void* dV, float* deta, float* dW1, float* dc1, float* dW2, float* dc2,
                                       float* dgamma, float* dbeta) {
    ttt::SimtMlpBackwardParams q{H,    T,    16, Q,  K,  V,    eta, eta_const, W_states, dZ,  dW1o,
                                 dc1o, dW2o, dc2o, dQ, dK, dV, deta, dW1,      dc1,      dW2, dc2,
                                 gamma, beta, eps, dgamma, dbeta};
    emu::run_grid_bounded(B * H, ttt::mmb::kThreads, ttt::mmb::smem, ttt::mmb::kSmemBytes, sizeof(ttt::mmb::smem), [&] { ttt::mmb::mma_mlp_backward_kernel<true>(q); });
    return 0;
}

// the TTT-MLP with LN+residual forward writing the batch-start states on mma.sync (bf16, d = 64, b = 16)
extern "C" int emu_mlp_ln_forward_mma(int B, int H, int T, const void* Q, const void* K, const void* V,
                                      const float* eta, float eta_const, const float* W1, const float* c1,
                                      const float* W2, const float* c2, const float* gamma, const float* beta,
                                      float eps, void* Z, float* W1_out, float* c1_out, float* W2_out, float* c2_out,
                                      float* W_states) {
    ttt::mmb::MlpFwdStatesParams f{H,  T,      Q,      K,      V,      eta,    eta_const, W1,      c1,
                                   W2, c2,     0,      Z,      W1_out, c1_out, W2_out,    c2_out, W_states,
                                   gamma, beta, eps};
    emu::run_grid_bounded(B * H, ttt::mmb::kThreads, ttt::mmb::smem, ttt::mmb::kSmemBytes, sizeof(ttt::mmb::smem), [&] { ttt::mmb::mma_mlp_forward_states_kernel<true>(f); });
    return 0;
}

// serial scheduling of the next runs (emu_core.h: 0 off, 1 ascending, 2 descending thread order), and the
// number of runs since the last call in which every live thread was blocked (a hang on the GPU)
extern "C" void emu_serial(int mode) { emu::serial = mode; }
extern "C" int emu_sched_errors() { return emu::sched_errors.exchange(0); }

// shared-memory overruns (accesses beyond the launch's dynamic size) since the last call
extern "C" int emu_smem_overruns() { return emu::smem_overruns.exchange(0); }
