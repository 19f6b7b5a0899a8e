"""Python driver of the float64 CPU oracle (test infrastructure only).

Thin ctypes marshalling around ``oracle/ttt_oracle.c``; every step of the
arithmetic is in that C file.  Inputs are numpy arrays of the exact stored
values (float64); outputs are float64.  Only the tests, the smoke check and
the benchmark's CPU-baseline leg import this module.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        # A test may point this at a deliberately broken build of the same
        # source to check that the pins catch planted mistakes.
        path = os.environ.get("TTT_ORACLE_LIB_OVERRIDE") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER(ctypes.c_double)
        i, ll, dbl = ctypes.c_int, ctypes.c_longlong, ctypes.c_double
        L.ttt_oracle_linear_forward.argtypes = [i, i, i, i, i, P, P, P, P, P, ll, P, ll, i, P, P, dbl,
                                                P, P, P, i]
        L.ttt_oracle_linear_forward.restype = i
        L.ttt_oracle_mlp_forward.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, ll, P, P, P, P, P, i]
        L.ttt_oracle_mlp_forward.restype = i
        L.ttt_oracle_mlp_ln_forward.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, ll, i, P, P, dbl,
                                                P, P, P, P, P, i]
        L.ttt_oracle_mlp_ln_forward.restype = i
        L.ttt_oracle_linear_decode_step.argtypes = [i, i, i, P, P, P, P, P, P]
        L.ttt_oracle_linear_decode_step.restype = i
        L.ttt_oracle_linear_backward.argtypes = [i, i, i, i, i, P, P, P, P, P, ll, P, P, P, P, P, P, P, i]
        L.ttt_oracle_linear_backward.restype = i
        L.ttt_oracle_linear_ln_backward.argtypes = [i, i, i, i, i, P, P, P, P, P, ll, P, ll, P, P, dbl, P, P, P,
                                                    P, P, P, P, P, P, P, P, i]
        L.ttt_oracle_linear_ln_backward.restype = i
        L.ttt_oracle_mlp_backward.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, ll, P, P, P, P, P,
                                              P, P, P, P, P, P, P, P, i]
        L.ttt_oracle_mlp_backward.restype = i
        L.ttt_oracle_mlp_ln_backward.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, ll, P, P, dbl, P, P, P,
                                                 P, P, P, P, P, P, P, P, P, P, P, P, i]
        L.ttt_oracle_mlp_ln_backward.restype = i
        L.ttt_oracle_qkv_prologue.argtypes = [i, i, i, i, i, P, P, P, P, P, dbl, P, P, P, P, i]
        L.ttt_oracle_qkv_prologue.restype = i
        _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def linear_forward(Q, K, V, eta, W0, b, c0=None, gamma=None, beta=None, use_ln=False, eps=1e-6,
                   threads=None):
    """Primal mini-batch TTT-Linear (optionally LN+residual) forward.

    Q, K, V: [B,H,T,d]; eta: [B,H,T]; W0: [H,d,d] (shared) or [B,H,d,d];
    c0, gamma, beta: [H,d] (c0 may also be [B,H,d]).
    Returns (Z [B,H,T,d], W_out [B,H,d,d], c_out [B,H,d]).
    """
    Q, K, V, eta, W0 = map(_f64, (Q, K, V, eta, W0))
    c0, gamma, beta = map(_f64, (c0, gamma, beta))
    B, H, T, d = Q.shape
    W0_bstride = 0 if W0.ndim == 3 else H * d * d
    c0_bstride = 0
    if c0 is not None and c0.ndim == 3:
        c0_bstride = H * d
    if use_ln and c0 is None:
        c0 = np.zeros((H, d))
    Z = np.empty((B, H, T, d))
    W_out = np.empty((B, H, d, d))
    c_out = np.empty((B, H, d))
    rc = lib().ttt_oracle_linear_forward(B, H, T, d, b, _p(Q), _p(K), _p(V), _p(eta), _p(W0), W0_bstride,
                                         _p(c0), c0_bstride, int(bool(use_ln)), _p(gamma), _p(beta), eps,
                                         _p(Z), _p(W_out), _p(c_out), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    return Z, W_out, c_out


def mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b, threads=None, use_ln=False, gamma=None, beta=None, eps=1e-6):
    """Primal mini-batch TTT-MLP forward, f(x) = GELU(x W1 + c1) W2 + c2, or
    with use_ln f(x) = x + gamma LN(GELU(x W1 + c1) W2 + c2) + beta.

    Parameters are [H,...] (shared over the batch) or [B,H,...]; gamma, beta [H,d].
    Returns (Z, W1_out [B,H,d,m], c1_out [B,H,m], W2_out [B,H,m,d], c2_out [B,H,d]).
    """
    Q, K, V, eta, W1, c1, W2, c2 = map(_f64, (Q, K, V, eta, W1, c1, W2, c2))
    gamma, beta = map(_f64, (gamma, beta))
    B, H, T, d = Q.shape
    m = W1.shape[-1]
    per_seq = 1 if W1.ndim == 4 else 0
    Z = np.empty((B, H, T, d))
    W1o, c1o = np.empty((B, H, d, m)), np.empty((B, H, m))
    W2o, c2o = np.empty((B, H, m, d)), np.empty((B, H, d))
    rc = lib().ttt_oracle_mlp_ln_forward(B, H, T, d, m, b, _p(Q), _p(K), _p(V), _p(eta), _p(W1), _p(c1),
                                         _p(W2), _p(c2), per_seq, int(bool(use_ln)), _p(gamma), _p(beta), eps,
                                         _p(Z), _p(W1o), _p(c1o), _p(W2o), _p(c2o), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    return Z, W1o, c1o, W2o, c2o


def linear_decode_step(W, q, k, v, eta):
    """One b=1 decode step for every unit.  W [B,H,d,d] is updated in a copy.

    Returns (W_new, z [B,H,d]).
    """
    W = np.array(W, dtype=np.float64, copy=True, order="C")
    q, k, v, eta = map(_f64, (q, k, v, eta))
    B, H, d = q.shape
    z = np.empty((B, H, d))
    rc = lib().ttt_oracle_linear_decode_step(B, H, d, _p(W), _p(q), _p(k), _p(v), _p(eta), _p(z))
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    return W, z


def linear_backward(Q, K, V, eta, W0, b, dZ=None, dW_out=None, threads=None):
    """Outer-loop gradients of the TTT-Linear forward (no LN), reverse mode
    through the primal loop.  dZ [B,H,T,d] and dW_out [B,H,d,d] are the
    gradients of a scalar loss with respect to the forward's outputs (None:
    zero).  Returns (dQ, dK, dV [B,H,T,d], deta [B,H,T], dW0 [B,H,d,d]),
    dW0 per sequence (sum over B for a shared W0)."""
    Q, K, V, eta, W0, dZ, dW_out = map(_f64, (Q, K, V, eta, W0, dZ, dW_out))
    B, H, T, d = Q.shape
    W0_bstride = 0 if W0.ndim == 3 else H * d * d
    dQ, dK, dV = np.empty((B, H, T, d)), np.empty((B, H, T, d)), np.empty((B, H, T, d))
    deta, dW0 = np.empty((B, H, T)), np.empty((B, H, d, d))
    rc = lib().ttt_oracle_linear_backward(B, H, T, d, b, _p(Q), _p(K), _p(V), _p(eta), _p(W0), W0_bstride,
                                          _p(dZ), _p(dW_out), _p(dQ), _p(dK), _p(dV), _p(deta), _p(dW0),
                                          threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    return dQ, dK, dV, deta, dW0


def linear_ln_backward(Q, K, V, eta, W0, b, c0, gamma, beta, eps=1e-6, dZ=None, dW_out=None, dc_out=None,
                       threads=None):
    """Outer-loop gradients of the LN+residual TTT-Linear forward, reverse mode
    through the primal loop.  Returns (dQ, dK, dV, deta, dW0, dc0, dgamma,
    dbeta); dW0, dc0, dgamma and dbeta are per unit [B,H,...] (sum over what
    is shared)."""
    Q, K, V, eta, W0, c0, gamma, beta = map(_f64, (Q, K, V, eta, W0, c0, gamma, beta))
    dZ, dW_out, dc_out = map(_f64, (dZ, dW_out, dc_out))
    B, H, T, d = Q.shape
    W0_bstride = 0 if W0.ndim == 3 else H * d * d
    c0_bstride = 0 if (c0 is None or c0.ndim == 2) else H * d
    dQ, dK, dV = np.empty((B, H, T, d)), np.empty((B, H, T, d)), np.empty((B, H, T, d))
    deta, dW0, dc0 = np.empty((B, H, T)), np.empty((B, H, d, d)), np.empty((B, H, d))
    dgamma, dbeta = np.empty((B, H, d)), np.empty((B, H, d))
    rc = lib().ttt_oracle_linear_ln_backward(B, H, T, d, b, _p(Q), _p(K), _p(V), _p(eta), _p(W0), W0_bstride,
                                             _p(c0), c0_bstride, _p(gamma), _p(beta), eps, _p(dZ), _p(dW_out),
                                             _p(dc_out), _p(dQ), _p(dK), _p(dV), _p(deta), _p(dW0), _p(dc0),
                                             _p(dgamma), _p(dbeta), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    return dQ, dK, dV, deta, dW0, dc0, dgamma, dbeta


def mlp_backward(Q, K, V, eta, W1, c1, W2, c2, b, dZ=None, dW1_out=None, dc1_out=None, dW2_out=None,
                 dc2_out=None, threads=None):
    """Outer-loop gradients of the TTT-MLP forward (no LN), reverse mode through
    the primal loop.  Parameters [H,...] (shared) or [B,H,...].  Returns
    (dQ, dK, dV, deta, dW1, dc1, dW2, dc2), the parameter gradients per unit
    [B,H,...] (sum over B for shared parameters)."""
    Q, K, V, eta, W1, c1, W2, c2 = map(_f64, (Q, K, V, eta, W1, c1, W2, c2))
    dZ, dW1_out, dc1_out, dW2_out, dc2_out = map(_f64, (dZ, dW1_out, dc1_out, dW2_out, dc2_out))
    B, H, T, d = Q.shape
    m = W1.shape[-1]
    per_seq = 1 if W1.ndim == 4 else 0
    dQ, dK, dV = np.empty((B, H, T, d)), np.empty((B, H, T, d)), np.empty((B, H, T, d))
    deta = np.empty((B, H, T))
    dW1, dc1 = np.empty((B, H, d, m)), np.empty((B, H, m))
    dW2, dc2 = np.empty((B, H, m, d)), np.empty((B, H, d))
    rc = lib().ttt_oracle_mlp_backward(B, H, T, d, m, b, _p(Q), _p(K), _p(V), _p(eta), _p(W1), _p(c1), _p(W2),
                                       _p(c2), per_seq, _p(dZ), _p(dW1_out), _p(dc1_out), _p(dW2_out),
                                       _p(dc2_out), _p(dQ), _p(dK), _p(dV), _p(deta), _p(dW1), _p(dc1), _p(dW2),
                                       _p(dc2), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    return dQ, dK, dV, deta, dW1, dc1, dW2, dc2


def qkv_prologue(x, theta_q, theta_k, theta_v, theta_lr, eta_base, d, threads=None):
    """The views and the learning-rate gate from the layer input x [B, T, Dm]:
    theta_q/k/v [H*d, Dm] (head h owns rows h*d .. h*d+d-1), theta_lr [H, Dm].
    Returns (Q, K, V) [B, H, T, d] and eta [B, H, T]."""
    x, theta_q, theta_k, theta_v, theta_lr = map(_f64, (x, theta_q, theta_k, theta_v, theta_lr))
    B, T, Dm = x.shape
    H = theta_lr.shape[0]
    if theta_q.shape != (H * d, Dm) or theta_k.shape != (H * d, Dm) or theta_v.shape != (H * d, Dm):
        raise ValueError("oracle: view matrices must be [H*d, Dm]")
    if theta_lr.shape != (H, Dm):
        raise ValueError("oracle: theta_lr must be [H, Dm]")
    Q, K, V = np.empty((B, H, T, d)), np.empty((B, H, T, d)), np.empty((B, H, T, d))
    eta = np.empty((B, H, T))
    rc = lib().ttt_oracle_qkv_prologue(B, T, Dm, H, d, _p(x), _p(theta_q), _p(theta_k), _p(theta_v),
                                       _p(theta_lr), float(eta_base), _p(Q), _p(K), _p(V), _p(eta),
                                       threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    return Q, K, V, eta


def mlp_ln_backward(Q, K, V, eta, W1, c1, W2, c2, b, gamma, beta, eps=1e-6, dZ=None, dW1_out=None, dc1_out=None,
                    dW2_out=None, dc2_out=None, threads=None):
    """Outer-loop gradients of TTT-MLP with LN+residual on the output layer,
    reverse mode through the primal loop.  Parameters [H,...] (shared) or
    [B,H,...]; gamma, beta [H,d].  Returns (dQ, dK, dV, deta, dW1, dc1, dW2,
    dc2, dgamma, dbeta), the parameter gradients per unit [B,H,...] (sum over
    what is shared)."""
    Q, K, V, eta, W1, c1, W2, c2, gamma, beta = map(_f64, (Q, K, V, eta, W1, c1, W2, c2, gamma, beta))
    dZ, dW1_out, dc1_out, dW2_out, dc2_out = map(_f64, (dZ, dW1_out, dc1_out, dW2_out, dc2_out))
    B, H, T, d = Q.shape
    m = W1.shape[-1]
    per_seq = 1 if W1.ndim == 4 else 0
    dQ, dK, dV = np.empty((B, H, T, d)), np.empty((B, H, T, d)), np.empty((B, H, T, d))
    deta = np.empty((B, H, T))
    dW1, dc1 = np.empty((B, H, d, m)), np.empty((B, H, m))
    dW2, dc2 = np.empty((B, H, m, d)), np.empty((B, H, d))
    dgamma, dbeta = np.empty((B, H, d)), np.empty((B, H, d))
    rc = lib().ttt_oracle_mlp_ln_backward(B, H, T, d, m, b, _p(Q), _p(K), _p(V), _p(eta), _p(W1), _p(c1), _p(W2),
                                          _p(c2), per_seq, _p(gamma), _p(beta), float(eps), _p(dZ), _p(dW1_out),
                                          _p(dc1_out), _p(dW2_out), _p(dc2_out), _p(dQ), _p(dK), _p(dV), _p(deta),
                                          _p(dW1), _p(dc1), _p(dW2), _p(dc2), _p(dgamma), _p(dbeta),
                                          threads or default_threads())
    if rc != 0:
        raise ValueError("oracle: invalid arguments")
    return dQ, dK, dV, deta, dW1, dc1, dW2, dc2, dgamma, dbeta
