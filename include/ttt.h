/*
 * ttt.h -- C ABI of the TTT layer inner-loop forward on NVIDIA B200 (sm_100a).
 *
 * Paper: "Learning to (Learn at Test Time): RNNs with Expressive Hidden
 * States".  Passages are cited by section of the paper digest "论文速览 | TTT"
 * (equinox-blog).
 *
 * In a TTT layer each (sequence, head) unit carries a hidden state that is
 * the weight set W of a small model f.  Tokens are processed in mini-batches
 * of b tokens; within a mini-batch every token's gradient of the
 * reconstruction loss 1/2 ||f(k_t; W) - v_t||^2 is taken at the mini-batch's
 * starting state W0, the updates W_t = W_{t-1} - eta_t * grad_t accumulate
 * token by token, and the output is z_t = f(q_t; W_t) (section 3.1: update,
 * then output; section 3.3: multi-view loss and output; section 3.5:
 * mini-batch gradient descent).  The GPU computes this in the dual form
 * (sections 3.6-3.7): per mini-batch,
 *     E = K W0 - V,   Z = Q W0 - (tril(Q K^T) * eta_s) E,   W_b = W0 - K^T diag(eta) E
 * for the linear model, with the analogous two-pass form for LN+residual and
 * for the MLP.
 *
 * Conventions shared by every entry point
 *   - Row vectors: f(x) = x W with W stored d_in x d_out, row-major.
 *   - Half-loss gradient: eta multiplies grad of 1/2 ||f - v||^2.  (The
 *     pages' dual form W_b = W0 - 2 eta (W0 X - X) X^T carries the 2 in eta.)
 *   - eta: per-token learning rate (section 4.6), one fp32 value per token,
 *     or a constant when the pointer is NULL.
 *   - All pointers are DEVICE pointers owned by the caller.  The library
 *     allocates nothing per call and keeps no state between calls beyond a
 *     device-side status word per device.
 *   - Calls are asynchronous on `stream`; results are valid after the stream
 *     is synchronised.  Inputs are never modified, except W in decode.
 *   - Errors: invalid arguments are rejected synchronously, before any launch
 *     (TTT_ERR_INVALID_ARG / TTT_ERR_UNSUPPORTED).  A failed launch returns
 *     TTT_ERR_CUDA.  Device-side waits are bounded; an expired wait ends the
 *     kernel early and is reported by ttt_last_device_status().
 *   - Alignment: every pointer must be 16-byte aligned.
 */
#ifndef TTT_H_
#define TTT_H_

#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TTT_OK = 0,
    TTT_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, T % b != 0 */
    TTT_ERR_UNSUPPORTED = 2,  /* valid request with no kernel for it (e.g. d not in {16,32,64}) */
    TTT_ERR_CUDA = 3,         /* launch or runtime error reported by CUDA */
    TTT_ERR_TIMEOUT = 4       /* a bounded device-side wait expired */
} ttt_status;

typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;

/* flags (bit set) */
#define TTT_FLAG_FORCE_SIMT 0x1u   /* use the fp32 CUDA-core kernel even where the tensor-core one applies */
#define TTT_FLAG_ONE_UNIT_PER_CTA 0x2u  /* tensor-core linear kernel: one (sequence, head) unit per CTA */
#define TTT_FLAG_TWO_UNITS_PER_CTA 0x4u /* tensor-core linear kernel: two units per CTA */
#define TTT_FLAG_LN_MMA_TRAINING 0x8u /* LN+residual training (ttt_linear_forward with W_states, ttt_linear_backward)
                                        on the mma.sync tensor-core kernels (BF16, d = 64, b = 16); without it those
                                        calls run on the fp32 CUDA-core kernels */
#define TTT_FLAG_TEST_STALL 0x100u /* test hook: one device wait is made to expire (see ttt_last_device_status) */
/* Without either UNITS_PER_CTA flag the library takes one unit per CTA when
 * B*H <= 148 (the SM count: the work is a serial chain per unit, and one unit
 * per CTA halves the serial work of each warp) and two otherwise.  Both
 * layouts compute the same operations in the same order. */

/*
 * ttt_linear_forward -- prefill of TTT-Linear or TTT-Linear with LN+residual.
 *
 * Inner model (section 4.4):
 *   use_ln == 0:  f(x) = x W
 *   use_ln == 1:  f(x) = x + LN(x W + c), LN over the d features with biased
 *                 variance, eps = ln_eps, per-head gamma/beta fixed during the
 *                 inner loop; the gradient flows through LN into W and c.
 *
 * Arguments
 *   B, H, T, d, b  sequences, heads, tokens, head dim, mini-batch size.
 *                  T % b == 0 is required.  Supported: d in {16, 32, 64},
 *                  1 <= b <= 64.  The tensor-core kernel serves io_dtype BF16,
 *                  d = 64, b = 16; every other valid case runs on the fp32
 *                  CUDA-core kernel.
 *   io_dtype       dtype of Q, K, V and Z (TTT_F32 or TTT_BF16).
 *   Q, K, V        [B, H, T, d] contiguous (views theta_Q x, theta_K x,
 *                  theta_V x of section 3.3; the projections are the caller's).
 *   eta            [B, H, T] fp32, or NULL: every token uses eta_const.
 *   W0             initial state (learnable theta_init, section 4.5), fp32,
 *                  unit (n, h) reads W0 + n * W0_bstride + h * d * d.
 *                  W0_bstride = 0: one [H, d, d] shared by all sequences;
 *                  W0_bstride = H*d*d: [B, H, d, d] (e.g. a resumed state).
 *   c0             LN only: initial bias [H, d] with the same batch-stride
 *                  rule (c0_bstride), or NULL for zeros.
 *   ln_gamma, ln_beta  LN only: [H, d] fp32.
 *   Z              output [B, H, T, d] in io_dtype, or NULL: only the final
 *                  state is computed, on the fp32 CUDA-core kernel (the
 *                  "computing W" part of the mini-batch size study, section
 *                  5.3).
 *   W_out          output final state [B, H, d, d] fp32.
 *   c_out          LN only: final bias [B, H, d] fp32, or NULL.
 *   flags          TTT_FLAG_* bits; 0 for normal use.
 *   wait_timeout_ms  limit of every device-side wait (0: 2000 ms).
 *   W_states       optional output for the backward (gradient checkpointing
 *                  through time, section 6.12): the state at the start of
 *                  every mini-batch, [B, H, T/b, d, d] fp32, T/b states per
 *                  unit.  NULL: not written.  With use_ln == 0, io_dtype
 *                  BF16, d = 64, b = 16 it runs the mma.sync forward (bf16
 *                  operands, fp32 state), otherwise the fp32 CUDA-core kernel.
 *   c_states       with use_ln and W_states: the bias at the start of every
 *                  mini-batch, [B, H, T/b, d] fp32 (required then).
 */
typedef struct {
    int B, H, T, d, b;
    ttt_dtype io_dtype;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W0;
    long long W0_bstride;
    const float* c0;
    long long c0_bstride;
    int use_ln;
    const float* ln_gamma;
    const float* ln_beta;
    float ln_eps;
    void* Z;
    float* W_out;
    float* c_out;
    unsigned flags;
    unsigned wait_timeout_ms;
    float* W_states;
    float* c_states;
} ttt_linear_args;

ttt_status ttt_linear_forward(const ttt_linear_args* args, cudaStream_t stream);

/*
 * ttt_linear_backward -- outer-loop gradients of the TTT-Linear prefill
 * (use_ln == 0): given dZ = dL/dZ and dW_out = dL/dW_out of a scalar loss L,
 * returns dL/dQ, dL/dK, dL/dV, dL/deta and dL/dW0.  The outer loop trains
 * the projections, the initial state and the learning rates through the
 * inner loop's updates (section 3.4).  The mini-batches are visited last to
 * first; each recomputes its residual E = K W - V and the causal products
 * from its batch-start state W (section 6.12: only the kappa = T/b boundary
 * states are kept), which ttt_linear_forward wrote to W_states.
 *
 *   B, H, T, d, b, io_dtype, Q, K, V, eta, eta_const
 *                  the forward's arguments (same rules; T % b == 0,
 *                  d in {16, 32, 64}, 1 <= b <= 64).
 *   W_states       [B, H, T/b, d, d] fp32 from the forward with the same inputs.
 *   dZ             [B, H, T, d] in io_dtype, or NULL for zero.
 *   dW_out         [B, H, d, d] fp32, or NULL for zero.
 *   dQ, dK, dV     outputs [B, H, T, d] in io_dtype.
 *   deta           output [B, H, T] fp32, or NULL when not wanted.
 *   dW0            output [B, H, d, d] fp32, one per sequence (a W0 shared
 *                  over the batch receives the sum over B).
 *   flags          0, or TTT_FLAG_FORCE_SIMT.
 *   use_ln         1: the LN+residual model (ttt_linear_forward's use_ln);
 *                  then also
 *     c_states       [B, H, T/b, d] fp32 from the forward,
 *     ln_gamma, ln_beta, ln_eps   the forward's LN parameters,
 *     dc_out         [B, H, d] fp32 dL/dc_out, or NULL for zero,
 *     dc0, dgamma, dbeta   outputs [B, H, d] fp32: dL/dc0, dL/dgamma and
 *                  dL/dbeta per (sequence, head) unit (sum what is shared).
 * Plain: io_dtype BF16 with d = 64 and b = 16 runs on the tensor cores
 * (mma.sync, bf16 operands, fp32 accumulation; the state gradient is carried
 * in fp32); every other case, TTT_FLAG_FORCE_SIMT, or use_ln, on the fp32
 * CUDA-core kernels (LN: b <= 32 at d = 64).  One CTA per (sequence, head)
 * unit.
 */
typedef struct {
    int B, H, T, d, b;
    ttt_dtype io_dtype;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W_states;
    const void* dZ;
    const float* dW_out;
    void* dQ;
    void* dK;
    void* dV;
    float* deta;
    float* dW0;
    unsigned flags;
    int use_ln;
    const float* c_states;
    const float* ln_gamma;
    const float* ln_beta;
    float ln_eps;
    const float* dc_out;
    float* dc0;
    float* dgamma;
    float* dbeta;
} ttt_linear_backward_args;

ttt_status ttt_linear_backward(const ttt_linear_backward_args* args, cudaStream_t stream);

/*
 * ttt_mlp_forward -- prefill of TTT-MLP, f(x) = GELU(x W1 + c1) W2 + c2 with
 * hidden size m = 4d (section 4.4), exact-erf GELU, dual form of section 3.7.
 *
 *   B, H, T, d, b  as above; supported: io_dtype BF16, d = 64, b = 16
 *                  (tensor-core kernel) or any io_dtype with d in {16, 32}
 *                  and b <= 64 (CUDA-core kernel).  T % b == 0.
 *   Q, K, V, eta, eta_const, Z   as for ttt_linear_forward.
 *   W1 [.., d, m], c1 [.., m], W2 [.., m, d], c2 [.., d]  fp32 initial
 *                  parameters: [H, ...] shared over sequences when
 *                  params_per_sequence == 0, [B, H, ...] when 1.  c1 / c2 may
 *                  be NULL (zeros).
 *   W1_out [B,H,d,m], c1_out [B,H,m], W2_out [B,H,m,d], c2_out [B,H,d]
 *                  final parameters (fp32); c1_out / c2_out may be NULL.
 *   use_ln         1: LN+residual on the output layer (section 4.4: the form
 *                  TTT-MLP takes in practice),
 *                  f(x) = x + ln_gamma * LN(GELU(x W1 + c1) W2 + c2) + ln_beta,
 *                  LN as in ttt_linear_forward (ln_gamma, ln_beta [H, d] fp32,
 *                  ln_eps > 0).  Same kernel choice as the plain model.
 *                  0: plain.
 *   W_states       NULL, or [B, H, T/b, 2dm + m + d] fp32: the state at the
 *                  start of every mini-batch, each one W1 [d][m], c1 [m],
 *                  W2 [m][d], c2 [d] (the checkpoints ttt_mlp_backward reads;
 *                  section 6.12).  BF16 with d = 64, b = 16 runs on an
 *                  mma.sync tensor-core kernel (plain or use_ln), every other
 *                  case (and TTT_FLAG_FORCE_SIMT) on the fp32 CUDA-core kernel.
 */
typedef struct {
    int B, H, T, d, b;
    ttt_dtype io_dtype;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W1;
    const float* c1;
    const float* W2;
    const float* c2;
    int params_per_sequence;
    void* Z;
    float* W1_out;
    float* c1_out;
    float* W2_out;
    float* c2_out;
    unsigned flags;
    unsigned wait_timeout_ms;
    int use_ln;
    const float* ln_gamma;
    const float* ln_beta;
    float ln_eps;
    float* W_states;
} ttt_mlp_args;

ttt_status ttt_mlp_forward(const ttt_mlp_args* args, cudaStream_t stream);

/*
 * ttt_mlp_backward -- outer-loop gradients of the TTT-MLP prefill, plain or
 * with LN+residual on the output layer (use_ln):
 * reverse-mode differentiation of ttt_mlp_forward through the inner loop's
 * updates (section 3.4), one mini-batch at a time in reverse order from the
 * batch-start states ttt_mlp_forward wrote to W_states (section 6.12).
 *
 *   B, H, T, d, b, io_dtype, Q, K, V, eta, eta_const
 *                  exactly as given to the forward that wrote W_states.
 *                  BF16 with d = 64, b = 16 runs on the tensor cores
 *                  (mma.sync); every other case (and TTT_FLAG_FORCE_SIMT) on
 *                  fp32 CUDA cores: d in {16, 32, 64}, b up to the
 *                  shared-memory limit (16 at d = 64).
 *   W_states       [B, H, T/b, 2dm + m + d] fp32, from ttt_mlp_forward.
 *   dZ             [B, H, T, d] io_dtype, or NULL (zero).
 *   dW1_out [B,H,d,m], dc1_out [B,H,m], dW2_out [B,H,m,d], dc2_out [B,H,d]
 *                  gradients with respect to the final state, each or NULL
 *                  (zero).
 * Outputs
 *   dQ, dK, dV     [B, H, T, d] io_dtype.
 *   deta           [B, H, T] fp32, or NULL (not computed).
 *   dW1 [B,H,d,m], dc1 [B,H,m], dW2 [B,H,m,d], dc2 [B,H,d]
 *                  gradients with respect to each unit's initial state (for
 *                  parameters shared over sequences, the caller sums over B).
 *                  They also serve as the kernel's running adjoint, so they
 *                  must not overlap any input.
 *   flags          TTT_FLAG_FORCE_SIMT; any other bit is TTT_ERR_INVALID_ARG.
 *   use_ln         1: the model of ttt_mlp_forward with use_ln (ln_gamma,
 *                  ln_beta [H, d], ln_eps as given to it); the outputs dgamma,
 *                  dbeta [B, H, d] receive the per-unit gradients of gamma and
 *                  beta.  BF16 with d = 64, b = 16 runs on the mma.sync
 *                  kernel as for the plain model; every other case on the
 *                  fp32 CUDA-core kernel (b up to 16 at d = 64 for shared
 *                  memory).  0: plain.
 */
typedef struct {
    int B, H, T, d, b;
    ttt_dtype io_dtype;
    const void* Q;
    const void* K;
    const void* V;
    const float* eta;
    float eta_const;
    const float* W_states;
    const void* dZ;
    const float* dW1_out;
    const float* dc1_out;
    const float* dW2_out;
    const float* dc2_out;
    void* dQ;
    void* dK;
    void* dV;
    float* deta;
    float* dW1;
    float* dc1;
    float* dW2;
    float* dc2;
    unsigned flags;
    int use_ln;
    const float* ln_gamma;
    const float* ln_beta;
    float ln_eps;
    float* dgamma;
    float* dbeta;
} ttt_mlp_backward_args;

ttt_status ttt_mlp_backward(const ttt_mlp_backward_args* args, cudaStream_t stream);

/*
 * ttt_linear_decode_step -- one generated token per unit, TTT-Linear plain or
 * LN+residual, primal form with b = 1 (section 6.11: decode is token by token
 * and uses the primal form; section 3.1: update, then output).
 *   plain:  e = k W - v,   W <- W - eta k^T e,   z = q W   (W after the update),
 *           computed as z = q W_old - eta (q . k) e so W is read and written once.
 *   use_ln: f(x) = x + LN(x W + c) (section 4.4; gamma, beta fixed): the
 *           gradient of 1/2 ||f(k) - v||^2 through LN gives delta (the
 *           gradient at the pre-activation); W <- W - eta k^T delta,
 *           c <- c - eta delta, z = f(q) with the updated W and c.
 *
 *   B, H, d        d in {16, 32, 64}.
 *   io_dtype       dtype of q, k, v and z.
 *   W              [B, H, d, d] fp32, updated in place.
 *   q, k, v        [B, H, d].
 *   eta            [B, H] fp32, or NULL for eta_const.
 *   z              output [B, H, d] in io_dtype.
 *   use_ln         0: plain.  1: LN+residual; then
 *   c              [B, H, d] fp32 bias state, updated in place;
 *   ln_gamma, ln_beta  [H, d] fp32;  ln_eps > 0 (1e-6 in the tests).
 *   With use_ln = 0 the last five fields are ignored.
 */
typedef struct {
    int B, H, d;
    ttt_dtype io_dtype;
    float* W;
    const void* q;
    const void* k;
    const void* v;
    const float* eta;
    float eta_const;
    void* z;
    int use_ln;
    float* c;
    const float* ln_gamma;
    const float* ln_beta;
    float ln_eps;
} ttt_decode_args;

ttt_status ttt_linear_decode_step(const ttt_decode_args* args, cudaStream_t stream);

/*
 * ttt_mlp_decode_step -- one generated token per unit, TTT-MLP
 * f(x) = GELU(x W1 + c1) W2 + c2 with hidden size m = 4 d (section 4.4),
 * primal form with b = 1 (section 6.11; section 3.1: update, then output):
 *     a = k W1 + c1,  h = GELU(a),  e = h W2 + c2 - v,
 *     delta1 = (e W2^T) * GELU'(a),
 *     W1 -= eta k^T delta1,  c1 -= eta delta1,  W2 -= eta h^T e,  c2 -= eta e,
 *     z = f(q) with the updated state.
 * GELU is the exact erf form.
 *
 *   B, H, d        d in {16, 32, 64}; m = 4 d.
 *   io_dtype       dtype of q, k, v and z.
 *   W1 [B,H,d,m], c1 [B,H,m], W2 [B,H,m,d], c2 [B,H,d]
 *                  fp32 state, updated in place.
 *   q, k, v        [B, H, d].
 *   eta            [B, H] fp32, or NULL for eta_const.
 *   z              output [B, H, d] in io_dtype.
 */
typedef struct {
    int B, H, d;
    ttt_dtype io_dtype;
    float* W1;
    float* c1;
    float* W2;
    float* c2;
    const void* q;
    const void* k;
    const void* v;
    const float* eta;
    float eta_const;
    void* z;
} ttt_mlp_decode_args;

ttt_status ttt_mlp_decode_step(const ttt_mlp_decode_args* args, cudaStream_t stream);

/*
 * ttt_qkv_prologue -- the inputs of the inner loop from the layer input: the
 * three views of every token (section 3.3, multi-view reconstruction: the
 * training view theta_K x_t, the label view theta_V x_t and the test view
 * theta_Q x_t) and the learnable per-token learning rate (section 4.6):
 *     Q[n,h,t,j] = sum_k theta_q[h d + j, k] x[n,t,k]      (K, V alike)
 *     eta[n,h,t] = eta_base * sigmoid(sum_k theta_lr[h,k] x[n,t,k])
 * For BF16 input, one dense contraction on the tensor cores (bf16 operands,
 * fp32 accumulation); the epilogue writes each view in the [B, H, T, d]
 * layout that the inner-loop entry points read, rounded once to bf16, and
 * applies the gate in fp32.  F32 input (and BF16 with TTT_FLAG_FORCE_SIMT)
 * runs on fp32 CUDA cores.
 *
 *   B, T           sequences and tokens per sequence (any T >= 0).
 *   Dm             width of the layer input; Dm % 8 == 0 (16-byte rows).
 *   H, d           heads and head dim; d in {16, 32, 64}, 1 <= H <= 256.
 *   io_dtype       BF16 or F32: x, the theta matrices and Q, K, V.
 *   x              [B, T, Dm].
 *   theta_q, theta_k, theta_v
 *                  [H*d, Dm] each, the pages' column form: head h owns rows
 *                  h*d .. h*d+d-1.
 *   theta_lr       [H, Dm], or NULL for no gate (then eta must be NULL too).
 *   eta_base       scale of the gate, in the half-loss convention of the
 *                  inner-loop entry points (twice the pages' value).
 *   Q, K, V        outputs [B, H, T, d] in io_dtype.
 *   eta            output [B, H, T] fp32, or NULL with theta_lr NULL.
 *   flags          TTT_FLAG_FORCE_SIMT, TTT_FLAG_TEST_STALL (tensor-core
 *                  kernel only); any other bit is TTT_ERR_INVALID_ARG.
 *   wait_timeout_ms  limit of one device-side wait (0: 2000 ms).
 * Outputs must not overlap the inputs.
 */
typedef struct {
    int B, T, Dm, H, d;
    ttt_dtype io_dtype;
    const void* x;
    const void* theta_q;
    const void* theta_k;
    const void* theta_v;
    const void* theta_lr;
    float eta_base;
    void* Q;
    void* K;
    void* V;
    float* eta;
    unsigned flags;
    unsigned wait_timeout_ms;
} ttt_qkv_prologue_args;

ttt_status ttt_qkv_prologue(const ttt_qkv_prologue_args* args, cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char* ttt_status_string(ttt_status s);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device.  Returns TTT_ERR_TIMEOUT if any kernel launched since the
 * last call gave up a bounded wait, TTT_ERR_CUDA on a CUDA error, else TTT_OK.
 */
ttt_status ttt_last_device_status(cudaStream_t stream);

/* Library version string. */
const char* ttt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H_ */
