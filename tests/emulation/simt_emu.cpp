// Host emulation of the CUDA execution model for the fp32 CUDA-core (SIMT)
// kernels' source, used by tests/test_simt_emulation.py.  TEST
// INFRASTRUCTURE: the library has no CPU path; this file only lets the CPU
// test suite run the kernels' own source (index arithmetic, phase order,
// barrier placement) against the float64 oracle where no GPU is present.
//
// One CTA at a time: 256 std::threads run the kernel function; __syncthreads
// is a std::barrier over them, a warp shuffle goes through a per-warp
// exchange array between two barriers of that warp, and the kernels'
// dynamic shared array is one static buffer.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <barrier>
#include <cmath>
#include <thread>
#include <vector>

namespace emu {
constexpr int NT = 256;
thread_local uint3 tid3, bid3;
std::barrier<>* block_bar = nullptr;
std::barrier<>* warp_bar[NT / 32];
float xch[NT / 32][32];
}  // namespace emu

#undef threadIdx
#undef blockIdx
#define threadIdx emu::tid3
#define blockIdx emu::bid3
inline void __syncthreads() { emu::block_bar->arrive_and_wait(); }
inline float __shfl_xor_sync(unsigned, float v, int o) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    emu::xch[w][lane] = v;
    emu::warp_bar[w]->arrive_and_wait();
    const float r = emu::xch[w][lane ^ o];
    emu::warp_bar[w]->arrive_and_wait();
    return r;
}
inline float rsqrtf(float x) { return 1.0f / std::sqrt(x); }
inline float __expf(float x) { return std::exp(x); }
inline float __fdividef(float a, float b) { return a / b; }
#define __launch_bounds__(...)
#undef __shared__
#define __shared__

// the kernels declare `extern __shared__ float sm[]` inside namespace ttt
namespace ttt {
alignas(16) float sm[65536];
}

#include "../../test_sequence_layers_head_b200/csrc/simt.cuh"
#include "../../test_sequence_layers_head_b200/csrc/simt_mlp_backward.cuh"

namespace {

template <typename F>
void run_grid(int blocks, F f) {
    for (int bx = 0; bx < blocks; ++bx) {
        std::barrier<> bb(emu::NT);
        for (int w = 0; w < emu::NT / 32; ++w) emu::warp_bar[w] = new std::barrier<>(32);
        emu::block_bar = &bb;
        std::vector<std::thread> th;
        for (int t = 0; t < emu::NT; ++t)
            th.emplace_back([&, t, bx] {
                emu::tid3 = make_uint3(t, 0, 0);
                emu::bid3 = make_uint3(bx, 0, 0);
                f();
            });
        for (auto& x : th) x.join();
        for (int w = 0; w < emu::NT / 32; ++w) delete emu::warp_bar[w];
    }
}

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
    run_grid(B * H, [&] { ttt::simt_mlp_kernel<D, IO, false>(p); });
    ttt::SimtMlpBackwardParams q{H,  T,  b,  Q,     K,     V,     eta,  eta_const, W_states, dZ,  dW1o,
                                 dc1o, dW2o, dc2o, dQ, dK, dV, deta, dW1, dc1, dW2, dc2};
    run_grid(B * H, [&] { ttt::simt_mlp_backward_kernel<D, IO>(q); });
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
