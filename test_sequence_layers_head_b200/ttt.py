"""ctypes binding of libttt (include/ttt.h).

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every step of the computation runs in the library's
CUDA kernels.  Functions take CUDA tensors and return CUDA tensors; outputs
may be passed in (preallocated) or are allocated with torch.

Raises :class:`TTTError` when the library returns a non-OK status and
:class:`RuntimeError` when the library is missing (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libttt.so")

TTT_OK, TTT_ERR_INVALID_ARG, TTT_ERR_UNSUPPORTED, TTT_ERR_CUDA, TTT_ERR_TIMEOUT = range(5)
TTT_F32, TTT_BF16 = 0, 1
FLAG_FORCE_SIMT = 0x1
FLAG_ONE_UNIT_PER_CTA = 0x2
FLAG_TWO_UNITS_PER_CTA = 0x4
FLAG_LN_MMA_TRAINING = 0x8
FLAG_TEST_STALL = 0x100

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_ll = ctypes.c_longlong
_u = ctypes.c_uint


class LinearArgs(ctypes.Structure):
    _fields_ = [("B", _i), ("H", _i), ("T", _i), ("d", _i), ("b", _i), ("io_dtype", _i),
                ("Q", _vp), ("K", _vp), ("V", _vp), ("eta", _vp), ("eta_const", _f),
                ("W0", _vp), ("W0_bstride", _ll), ("c0", _vp), ("c0_bstride", _ll),
                ("use_ln", _i), ("ln_gamma", _vp), ("ln_beta", _vp), ("ln_eps", _f),
                ("Z", _vp), ("W_out", _vp), ("c_out", _vp), ("flags", _u), ("wait_timeout_ms", _u),
                ("W_states", _vp), ("c_states", _vp)]


class MlpArgs(ctypes.Structure):
    _fields_ = [("B", _i), ("H", _i), ("T", _i), ("d", _i), ("b", _i), ("io_dtype", _i),
                ("Q", _vp), ("K", _vp), ("V", _vp), ("eta", _vp), ("eta_const", _f),
                ("W1", _vp), ("c1", _vp), ("W2", _vp), ("c2", _vp), ("params_per_sequence", _i),
                ("Z", _vp), ("W1_out", _vp), ("c1_out", _vp), ("W2_out", _vp), ("c2_out", _vp),
                ("flags", _u), ("wait_timeout_ms", _u), ("use_ln", _i), ("ln_gamma", _vp), ("ln_beta", _vp),
                ("ln_eps", _f), ("W_states", _vp)]


class MlpBackwardArgs(ctypes.Structure):
    _fields_ = [("B", _i), ("H", _i), ("T", _i), ("d", _i), ("b", _i), ("io_dtype", _i), ("Q", _vp), ("K", _vp),
                ("V", _vp), ("eta", _vp), ("eta_const", _f), ("W_states", _vp), ("dZ", _vp), ("dW1_out", _vp),
                ("dc1_out", _vp), ("dW2_out", _vp), ("dc2_out", _vp), ("dQ", _vp), ("dK", _vp), ("dV", _vp),
                ("deta", _vp), ("dW1", _vp), ("dc1", _vp), ("dW2", _vp), ("dc2", _vp), ("flags", _u),
                ("use_ln", _i), ("ln_gamma", _vp), ("ln_beta", _vp), ("ln_eps", _f), ("dgamma", _vp),
                ("dbeta", _vp)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("B", _i), ("H", _i), ("d", _i), ("io_dtype", _i), ("W", _vp), ("q", _vp), ("k", _vp),
                ("v", _vp), ("eta", _vp), ("eta_const", _f), ("z", _vp), ("use_ln", _i), ("c", _vp),
                ("ln_gamma", _vp), ("ln_beta", _vp), ("ln_eps", _f)]


class BackwardArgs(ctypes.Structure):
    _fields_ = [("B", _i), ("H", _i), ("T", _i), ("d", _i), ("b", _i), ("io_dtype", _i), ("Q", _vp), ("K", _vp),
                ("V", _vp), ("eta", _vp), ("eta_const", _f), ("W_states", _vp), ("dZ", _vp), ("dW_out", _vp),
                ("dQ", _vp), ("dK", _vp), ("dV", _vp), ("deta", _vp), ("dW0", _vp), ("flags", _u),
                ("use_ln", _i), ("c_states", _vp), ("ln_gamma", _vp), ("ln_beta", _vp), ("ln_eps", _f),
                ("dc_out", _vp), ("dc0", _vp), ("dgamma", _vp), ("dbeta", _vp)]


class MlpDecodeArgs(ctypes.Structure):
    _fields_ = [("B", _i), ("H", _i), ("d", _i), ("io_dtype", _i), ("W1", _vp), ("c1", _vp), ("W2", _vp),
                ("c2", _vp), ("q", _vp), ("k", _vp), ("v", _vp), ("eta", _vp), ("eta_const", _f), ("z", _vp)]


class QkvPrologueArgs(ctypes.Structure):
    _fields_ = [("B", _i), ("T", _i), ("Dm", _i), ("H", _i), ("d", _i), ("io_dtype", _i), ("x", _vp),
                ("theta_q", _vp), ("theta_k", _vp), ("theta_v", _vp), ("theta_lr", _vp), ("eta_base", _f),
                ("Q", _vp), ("K", _vp), ("V", _vp), ("eta", _vp), ("flags", _u), ("wait_timeout_ms", _u)]


class TTTError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)}")
        self.code = code


_lib = None

# Every symbol include/ttt.h declares.
EXPORTS = ("ttt_linear_forward", "ttt_linear_backward", "ttt_mlp_forward", "ttt_linear_decode_step",
           "ttt_mlp_decode_step", "ttt_mlp_backward", "ttt_qkv_prologue", "ttt_status_string",
           "ttt_last_device_status", "ttt_version")


def library() -> ctypes.CDLL:
    """Load libttt.so (built in-tree by ``build.py``); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libttt.so not found at {LIB_PATH}; build it with "
                               "`python -m test_sequence_layers_head_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        L.ttt_linear_forward.argtypes = [ctypes.POINTER(LinearArgs), _vp]
        L.ttt_linear_forward.restype = _i
        L.ttt_linear_backward.argtypes = [ctypes.POINTER(BackwardArgs), _vp]
        L.ttt_linear_backward.restype = _i
        L.ttt_mlp_forward.argtypes = [ctypes.POINTER(MlpArgs), _vp]
        L.ttt_mlp_forward.restype = _i
        L.ttt_linear_decode_step.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
        L.ttt_linear_decode_step.restype = _i
        L.ttt_mlp_decode_step.argtypes = [ctypes.POINTER(MlpDecodeArgs), _vp]
        L.ttt_mlp_decode_step.restype = _i
        L.ttt_mlp_backward.argtypes = [ctypes.POINTER(MlpBackwardArgs), _vp]
        L.ttt_mlp_backward.restype = _i
        L.ttt_qkv_prologue.argtypes = [ctypes.POINTER(QkvPrologueArgs), _vp]
        L.ttt_qkv_prologue.restype = _i
        L.ttt_status_string.argtypes = [_i]
        L.ttt_status_string.restype = ctypes.c_char_p
        L.ttt_last_device_status.argtypes = [_vp]
        L.ttt_last_device_status.restype = _i
        L.ttt_version.argtypes = []
        L.ttt_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return library().ttt_status_string(code).decode()


def version() -> str:
    return library().ttt_version().decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libttt takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("libttt takes contiguous tensors only")
    return t.data_ptr()


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _io_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TTT_BF16
    if t.dtype == torch.float32:
        return TTT_F32
    raise ValueError(f"unsupported io dtype {t.dtype}")


def _check(code: int, what: str):
    if code != TTT_OK:
        raise TTTError(code, what)


def linear_forward(Q, K, V, eta, W0, b, *, eta_const=0.0, use_ln=False, c0=None, gamma=None, beta=None,
                   eps=1e-6, Z=None, W_out=None, c_out=None, flags=0, wait_timeout_ms=0, W_states=None,
                   c_states=None, outputs=True, stream=None):
    """TTT-Linear (optionally LN+residual) prefill; see ``ttt_linear_forward``.

    Q, K, V: [B,H,T,d] bf16 or fp32; eta: [B,H,T] fp32 or None (eta_const);
    W0: [H,d,d] (shared) or [B,H,d,d] fp32.  Returns (Z, W_out, c_out).
    W_states: optional [B,H,T/b,d,d] fp32 output, the state at every mini-batch
    start (for ``linear_backward``); with use_ln also c_states [B,H,T/b,d].
    outputs=False: Z is not computed (None is returned), only the state.
    """
    B, H, T, d = Q.shape
    dev = Q.device
    if not outputs:
        Z = None   # state only: the library skips the outputs
    elif Z is None:
        Z = torch.empty_like(Q)
    if W_out is None:
        W_out = torch.empty((B, H, d, d), device=dev, dtype=torch.float32)
    if use_ln and c_out is None:
        c_out = torch.empty((B, H, d), device=dev, dtype=torch.float32)
    W0_bstride = 0 if W0.dim() == 3 else H * d * d
    c0_bstride = H * d if (c0 is not None and c0.dim() == 3) else 0
    a = LinearArgs(B, H, T, d, b, _io_dtype(Q), _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), float(eta_const),
                   _ptr(W0), W0_bstride, _ptr(c0), c0_bstride, int(bool(use_ln)), _ptr(gamma), _ptr(beta),
                   float(eps), _ptr(Z), _ptr(W_out), _ptr(c_out), int(flags), int(wait_timeout_ms),
                   _ptr(W_states), _ptr(c_states))
    _check(library().ttt_linear_forward(ctypes.byref(a), _stream(stream)), "ttt_linear_forward")
    return Z, W_out, c_out


def linear_backward(Q, K, V, eta, W_states, b, *, dZ=None, dW_out=None, eta_const=0.0, dQ=None, dK=None,
                    dV=None, deta=None, dW0=None, flags=0, use_ln=False, c_states=None, gamma=None, beta=None,
                    eps=1e-6, dc_out=None, stream=None):
    """Outer-loop gradients of the TTT-Linear prefill (no LN); see
    ``ttt_linear_backward``.  W_states [B,H,T/b,d,d] comes from
    ``linear_forward(..., W_states=...)`` on the same inputs.  Returns
    (dQ, dK, dV, deta, dW0); deta is None when eta is None.  use_ln: the
    LN+residual model (c_states from the forward, gamma, beta, eps, optional
    dc_out); then returns (dQ, dK, dV, deta, dW0, dc0, dgamma, dbeta), the last
    three per unit [B,H,d]."""
    B, H, T, d = Q.shape
    dev = Q.device
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    if deta is None and eta is not None:
        deta = torch.empty((B, H, T), device=dev, dtype=torch.float32)
    dW0 = torch.empty((B, H, d, d), device=dev, dtype=torch.float32) if dW0 is None else dW0
    f32 = dict(device=dev, dtype=torch.float32)
    dc0 = torch.empty((B, H, d), **f32) if use_ln else None
    dgamma = torch.empty((B, H, d), **f32) if use_ln else None
    dbeta = torch.empty((B, H, d), **f32) if use_ln else None
    a = BackwardArgs(B, H, T, d, b, _io_dtype(Q), _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), float(eta_const),
                     _ptr(W_states), _ptr(dZ), _ptr(dW_out), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(deta), _ptr(dW0),
                     int(flags), int(bool(use_ln)), _ptr(c_states), _ptr(gamma), _ptr(beta), float(eps),
                     _ptr(dc_out), _ptr(dc0), _ptr(dgamma), _ptr(dbeta))
    _check(library().ttt_linear_backward(ctypes.byref(a), _stream(stream)), "ttt_linear_backward")
    if use_ln:
        return dQ, dK, dV, deta, dW0, dc0, dgamma, dbeta
    return dQ, dK, dV, deta, dW0


def mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b, *, eta_const=0.0, Z=None, W1_out=None, c1_out=None,
                W2_out=None, c2_out=None, flags=0, wait_timeout_ms=0, use_ln=False, gamma=None, beta=None,
                eps=1e-6, W_states=None, stream=None):
    """TTT-MLP prefill; see ``ttt_mlp_forward``.  Returns (Z, W1, c1, W2, c2).
    use_ln: LN+residual on the output layer with gamma, beta [H,d].
    W_states: [B,H,T/b,2dm+m+d] fp32 to receive the batch-start states (the
    checkpoints of ``mlp_backward``)."""
    B, H, T, d = Q.shape
    m = W1.shape[-1]
    dev = Q.device
    f32 = torch.float32
    Z = torch.empty_like(Q) if Z is None else Z
    W1_out = torch.empty((B, H, d, m), device=dev, dtype=f32) if W1_out is None else W1_out
    c1_out = torch.empty((B, H, m), device=dev, dtype=f32) if c1_out is None else c1_out
    W2_out = torch.empty((B, H, m, d), device=dev, dtype=f32) if W2_out is None else W2_out
    c2_out = torch.empty((B, H, d), device=dev, dtype=f32) if c2_out is None else c2_out
    per_seq = 1 if W1.dim() == 4 else 0
    a = MlpArgs(B, H, T, d, b, _io_dtype(Q), _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), float(eta_const),
                _ptr(W1), _ptr(c1), _ptr(W2), _ptr(c2), per_seq, _ptr(Z), _ptr(W1_out), _ptr(c1_out),
                _ptr(W2_out), _ptr(c2_out), int(flags), int(wait_timeout_ms), int(bool(use_ln)), _ptr(gamma),
                _ptr(beta), float(eps), _ptr(W_states))
    _check(library().ttt_mlp_forward(ctypes.byref(a), _stream(stream)), "ttt_mlp_forward")
    return Z, W1_out, c1_out, W2_out, c2_out


def linear_decode_step(W, q, k, v, eta, *, eta_const=0.0, z=None, use_ln=False, c=None, gamma=None, beta=None,
                       eps=1e-6, stream=None):
    """One decode token per unit; W [B,H,d,d] fp32 (and, with use_ln, the bias
    state c [B,H,d]) is updated in place.  Returns z."""
    B, H, d = q.shape
    z = torch.empty_like(q) if z is None else z
    a = DecodeArgs(B, H, d, _io_dtype(q), _ptr(W), _ptr(q), _ptr(k), _ptr(v), _ptr(eta), float(eta_const),
                   _ptr(z), int(bool(use_ln)), _ptr(c), _ptr(gamma), _ptr(beta), float(eps))
    _check(library().ttt_linear_decode_step(ctypes.byref(a), _stream(stream)), "ttt_linear_decode_step")
    return z


def mlp_decode_step(W1, c1, W2, c2, q, k, v, eta, *, eta_const=0.0, z=None, stream=None):
    """One TTT-MLP decode token per unit; W1 [B,H,d,4d], c1 [B,H,4d], W2 [B,H,4d,d]
    and c2 [B,H,d] (fp32) are updated in place.  Returns z."""
    B, H, d = q.shape
    z = torch.empty_like(q) if z is None else z
    a = MlpDecodeArgs(B, H, d, _io_dtype(q), _ptr(W1), _ptr(c1), _ptr(W2), _ptr(c2), _ptr(q), _ptr(k), _ptr(v),
                      _ptr(eta), float(eta_const), _ptr(z))
    _check(library().ttt_mlp_decode_step(ctypes.byref(a), _stream(stream)), "ttt_mlp_decode_step")
    return z


def mlp_backward(Q, K, V, eta, W_states, b, *, dZ=None, dW1_out=None, dc1_out=None, dW2_out=None, dc2_out=None,
                 eta_const=0.0, dQ=None, dK=None, dV=None, deta=None, want_deta=True, dW1=None, dc1=None, dW2=None,
                 dc2=None, flags=0, use_ln=False, gamma=None, beta=None, eps=1e-6, stream=None):
    """Outer-loop gradients of the TTT-MLP prefill; see ``ttt_mlp_backward``.
    Returns (dQ, dK, dV, deta, dW1, dc1, dW2, dc2), with use_ln also (dgamma,
    dbeta) [B,H,d]; deta is None when ``want_deta`` is False."""
    B, H, T, d = Q.shape
    m = 4 * d
    dev, f32 = Q.device, torch.float32
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(Q) if dK is None else dK
    dV = torch.empty_like(Q) if dV is None else dV
    if want_deta and deta is None:
        deta = torch.empty((B, H, T), device=dev, dtype=f32)
    dW1 = torch.empty((B, H, d, m), device=dev, dtype=f32) if dW1 is None else dW1
    dc1 = torch.empty((B, H, m), device=dev, dtype=f32) if dc1 is None else dc1
    dW2 = torch.empty((B, H, m, d), device=dev, dtype=f32) if dW2 is None else dW2
    dc2 = torch.empty((B, H, d), device=dev, dtype=f32) if dc2 is None else dc2
    dgamma = torch.empty((B, H, d), device=dev, dtype=f32) if use_ln else None
    dbeta = torch.empty((B, H, d), device=dev, dtype=f32) if use_ln else None
    a = MlpBackwardArgs(B, H, T, d, b, _io_dtype(Q), _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), float(eta_const),
                        _ptr(W_states), _ptr(dZ), _ptr(dW1_out), _ptr(dc1_out), _ptr(dW2_out), _ptr(dc2_out),
                        _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(deta), _ptr(dW1), _ptr(dc1), _ptr(dW2), _ptr(dc2),
                        int(flags), int(bool(use_ln)), _ptr(gamma), _ptr(beta), float(eps), _ptr(dgamma),
                        _ptr(dbeta))
    _check(library().ttt_mlp_backward(ctypes.byref(a), _stream(stream)), "ttt_mlp_backward")
    if use_ln:
        return dQ, dK, dV, deta, dW1, dc1, dW2, dc2, dgamma, dbeta
    return dQ, dK, dV, deta, dW1, dc1, dW2, dc2


def qkv_prologue(x, theta_q, theta_k, theta_v, theta_lr, eta_base, d, *, Q=None, K=None, V=None, eta=None,
                 flags=0, wait_timeout_ms=0, stream=None):
    """The views and the learning-rate gate from the layer input; see
    ``ttt_qkv_prologue``.  x [B,T,Dm] bf16; theta_q/k/v [H*d, Dm]; theta_lr
    [H, Dm] or None (no gate).  Returns (Q, K, V) [B,H,T,d] and eta [B,H,T]
    (None without the gate)."""
    B, T, Dm = x.shape
    H = theta_q.shape[0] // d
    dev = x.device
    Q = torch.empty((B, H, T, d), device=dev, dtype=x.dtype) if Q is None else Q
    K = torch.empty((B, H, T, d), device=dev, dtype=x.dtype) if K is None else K
    V = torch.empty((B, H, T, d), device=dev, dtype=x.dtype) if V is None else V
    if theta_lr is not None and eta is None:
        eta = torch.empty((B, H, T), device=dev, dtype=torch.float32)
    a = QkvPrologueArgs(B, T, Dm, H, d, _io_dtype(x), _ptr(x), _ptr(theta_q), _ptr(theta_k), _ptr(theta_v),
                        _ptr(theta_lr), float(eta_base), _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), int(flags),
                        int(wait_timeout_ms))
    _check(library().ttt_qkv_prologue(ctypes.byref(a), _stream(stream)), "ttt_qkv_prologue")
    return Q, K, V, eta


def last_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the device status (TTT_OK / TTT_ERR_TIMEOUT / ...)."""
    return library().ttt_last_device_status(_stream(stream))
