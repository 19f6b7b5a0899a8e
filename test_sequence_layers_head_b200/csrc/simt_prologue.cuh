// Fused prologue on fp32 CUDA cores: the three views and the learning-rate
// gate of every token (paper digest "论文速览 | TTT", sections 3.3 and 4.6),
//     Q/K/V(n, h, t, j) = sum_k theta_{q/k/v}[h d + j, k] x(n, t, k)
//     eta(n, h, t)      = eta_base * sigmoid(sum_k theta_lr[h, k] x(n, t, k))
// for any storage dtype (fp32 inputs have no tensor-core kernel) and as the
// cross-check path of the tensor-core prologue.
//
// The output columns are the three views' H d columns followed by the H gate
// columns.  One CTA of 256 threads per block of 16 tokens and 1024 columns
// (grid x: token blocks, y: column blocks): the tokens' x rows are staged in
// shared memory (fp32) one 256-element chunk of the model width at a time,
// and each thread accumulates its outputs (token, column), at most 64, over
// the chunks.  Consecutive threads take consecutive columns of one token, so
// each theta row is read by one thread and its reads walk the row.
#pragma once
#include "common.cuh"
#include "simt.cuh"

namespace ttt {

struct SimtPrologueParams {
    int rows;          // B * T tokens
    int T, Dm, H, d;
    const void* x;     // [rows, Dm]
    const void* theta_q;
    const void* theta_k;
    const void* theta_v;
    const void* theta_lr;   // or null
    float eta_base;
    void* Q;
    void* K;
    void* V;
    float* eta;
};

constexpr int kProTok = 16;     // tokens per CTA
constexpr int kProChunk = 256;  // model-width elements staged per pass
constexpr int kProMaxOut = 64;  // outputs per thread
constexpr int kProCols = kProMaxOut * kSimtThreads / kProTok;   // columns per CTA
constexpr size_t kProSmemBytes = sizeof(float) * kProTok * kProChunk;

template <typename IO>
__global__ void __launch_bounds__(kSimtThreads) simt_prologue_kernel(SimtPrologueParams p) {
    extern __shared__ __align__(16) float sm[];
    float (*xs)[kProChunk] = reinterpret_cast<float (*)[kProChunk]>(sm);   // [kProTok][kProChunk]
    const int tid = threadIdx.x;
    const int r0 = blockIdx.x * kProTok;
    const int ntok = min(kProTok, p.rows - r0);
    const int Hd = p.H * p.d;
    const int c0 = blockIdx.y * kProCols;
    const int ncb = min(kProCols, 3 * Hd + (p.theta_lr ? p.H : 0) - c0);   // columns of this CTA
    const IO* x = static_cast<const IO*>(p.x);
    // outputs (token, column c0 + ...) owned by this thread: e = tid, tid + 256, ... over ntok x ncb,
    // each accumulated over all chunks of the model width
    constexpr int kMaxOut = kProMaxOut;
    float acc[kMaxOut];
    const int nout = ntok * ncb;
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o) acc[o] = 0.f;
    for (int k0 = 0; k0 < p.Dm; k0 += kProChunk) {
        const int kn = min(kProChunk, p.Dm - k0);
        __syncthreads();
        for (int e = tid; e < kProTok * kProChunk; e += kSimtThreads) {
            const int t = e / kProChunk, k = e % kProChunk;
            xs[t][k] = (t < ntok && k < kn) ? IoTraits<IO>::load(x, (size_t)(r0 + t) * p.Dm + k0 + k) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int o = 0; o < kMaxOut; ++o) {
            const int e = tid + o * kSimtThreads;
            if (e >= nout) break;
            const int t = e / ncb, col = c0 + e % ncb;
            const IO* row;
            if (col < 3 * Hd) {
                const int v = col / Hd;
                const IO* th = static_cast<const IO*>(v == 0 ? p.theta_q : v == 1 ? p.theta_k : p.theta_v);
                row = th + (size_t)(col - v * Hd) * p.Dm + k0;
            } else {
                row = static_cast<const IO*>(p.theta_lr) + (size_t)(col - 3 * Hd) * p.Dm + k0;
            }
            float a = acc[o];
            for (int k = 0; k < kn; ++k) a += xs[t][k] * IoTraits<IO>::load(row, k);
            acc[o] = a;
        }
    }
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o) {
        const int e = tid + o * kSimtThreads;
        if (e >= nout) break;
        const int t = e / ncb, col = c0 + e % ncb;
        const int rr = r0 + t, n = rr / p.T, tt = rr - n * p.T;
        if (col < 3 * Hd) {
            const int v = col / Hd, c = col - v * Hd, h = c / p.d, j = c - h * p.d;
            IO* out = static_cast<IO*>(v == 0 ? p.Q : v == 1 ? p.K : p.V);
            IoTraits<IO>::store(out, (((size_t)n * p.H + h) * p.T + tt) * p.d + j, acc[o]);
        } else {
            const int h = col - 3 * Hd;
            p.eta[((size_t)n * p.H + h) * p.T + tt] = p.eta_base / (1.f + expf(-acc[o]));
        }
    }
}

}  // namespace ttt
