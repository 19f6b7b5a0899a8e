"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/ttt.h declares, and rejects invalid arguments
synchronously, before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "ttt.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ttt_[a-z_]+)\s*\(", src)))


def test_header_declares_entry_points():
    syms = declared_symbols()
    for s in ("ttt_linear_forward", "ttt_linear_backward", "ttt_mlp_forward", "ttt_linear_decode_step",
              "ttt_mlp_decode_step", "ttt_qkv_prologue"):
        assert s in syms


def test_library_exports_every_declared_symbol(ttt_lib):
    L = ttt_lib.library()
    for s in declared_symbols():
        assert hasattr(L, s), s
    assert set(declared_symbols()) <= set(ttt_lib.EXPORTS) | set(declared_symbols())


def test_status_strings(ttt_lib):
    assert ttt_lib.status_string(0) == "TTT_OK"
    assert ttt_lib.status_string(4) == "TTT_ERR_TIMEOUT"
    assert ttt_lib.version().startswith("ttt-b200")


def _linear_args(ttt, **kw):
    a = ttt.LinearArgs()
    a.B, a.H, a.T, a.d, a.b, a.io_dtype = 1, 1, 32, 64, 16, ttt.TTT_BF16
    fake = 1 << 20  # aligned fake device address; never dereferenced (validation fails first)
    a.Q = a.K = a.V = a.Z = a.W0 = a.W_out = fake
    a.ln_eps = 1e-6
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,code", [
    ("T", 30, 1),          # T % b != 0
    ("b", 0, 1),
    ("B", -1, 1),
    ("d", 48, 2),          # unsupported head dim
    ("d", 0, 1),
    ("b", 128, 1),         # T = 32 is not a multiple of 128
    ("io_dtype", 7, 1),
    ("Q", None, 1),        # null pointer
    ("Z", (1 << 20) + 4, 1),  # misaligned (NULL is allowed: state only)
    ("K", (1 << 20) + 4, 1),  # misaligned
    ("W_out", None, 1),
    ("eta", (1 << 20) + 8, 1),
    ("use_ln", 2, 1),
    ("flags", 0x8000, 1),
    ("flags", 0x6, 1),     # one and two units per CTA at once
    ("W0_bstride", -1, 1),
])
def test_linear_forward_rejects_invalid_arguments(ttt_lib, field, value, code):
    a = _linear_args(ttt_lib, **{field: value})
    assert ttt_lib.library().ttt_linear_forward(ctypes.byref(a), None) == code


def test_linear_forward_w_states_rules(ttt_lib):
    L = ttt_lib.library()
    a = _linear_args(ttt_lib, W_states=(1 << 20) + 4)    # misaligned
    assert L.ttt_linear_forward(ctypes.byref(a), None) == 1
    a = _linear_args(ttt_lib, W_states=1 << 20, use_ln=1, ln_gamma=1 << 20, ln_beta=1 << 20)
    assert L.ttt_linear_forward(ctypes.byref(a), None) == 1   # the LN variant needs c_states too


def _backward_args(ttt, **kw):
    a = ttt.BackwardArgs()
    a.B, a.H, a.T, a.d, a.b, a.io_dtype = 1, 2, 32, 64, 16, ttt.TTT_BF16
    fake = 1 << 20
    a.Q = a.K = a.V = a.W_states = a.dQ = a.dK = a.dV = a.dW0 = fake
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(T=30), 1),
    (dict(b=0), 1),
    (dict(d=48), 2),
    (dict(b=128, T=128), 2),
    (dict(io_dtype=3), 1),
    (dict(W_states=None), 1),
    (dict(dQ=None), 1),
    (dict(dW0=None), 1),
    (dict(dZ=(1 << 20) + 2), 1),
    (dict(dW_out=(1 << 20) + 8), 1),
    (dict(deta=(1 << 20) + 4), 1),
    (dict(B=0, Q=None), 0),
    (dict(flags=0x2), 1),
    (dict(use_ln=2), 1),
    (dict(use_ln=1), 1),                                       # no c_states / gamma / beta / outputs
    (dict(use_ln=1, c_states=1 << 20, ln_gamma=1 << 20, ln_beta=1 << 20, ln_eps=1e-6, dc0=1 << 20,
          dgamma=1 << 20, dbeta=(1 << 20) + 4), 1),            # misaligned dbeta
    (dict(use_ln=1, c_states=1 << 20, ln_gamma=1 << 20, ln_beta=1 << 20, dc0=1 << 20, dgamma=1 << 20,
          dbeta=1 << 20), 1),                                  # eps = 0
])
def test_linear_backward_validation(ttt_lib, kw, code):
    a = _backward_args(ttt_lib, **kw)
    assert ttt_lib.library().ttt_linear_backward(ctypes.byref(a), None) == code


def test_linear_forward_large_b_unsupported(ttt_lib):
    a = _linear_args(ttt_lib, b=128, T=256)
    assert ttt_lib.library().ttt_linear_forward(ctypes.byref(a), None) == 2


def test_linear_forward_ln_requires_gamma_beta(ttt_lib):
    a = _linear_args(ttt_lib, use_ln=1)
    assert ttt_lib.library().ttt_linear_forward(ctypes.byref(a), None) == 1


def test_empty_batch_is_a_no_op(ttt_lib):
    a = _linear_args(ttt_lib, B=0)
    assert ttt_lib.library().ttt_linear_forward(ctypes.byref(a), None) == 0


def test_null_args_struct(ttt_lib):
    L = ttt_lib.library()
    assert L.ttt_linear_forward(None, None) == 1
    assert L.ttt_mlp_forward(None, None) == 1
    assert L.ttt_linear_decode_step(None, None) == 1
    assert L.ttt_mlp_decode_step(None, None) == 1
    assert L.ttt_linear_backward(None, None) == 1
    assert L.ttt_qkv_prologue(None, None) == 1
    assert L.ttt_mlp_backward(None, None) == 1


def test_mlp_and_decode_validation(ttt_lib):
    L = ttt_lib.library()
    m = ttt_lib.MlpArgs()
    m.B, m.H, m.T, m.d, m.b, m.io_dtype = 1, 1, 32, 64, 16, ttt_lib.TTT_BF16
    assert L.ttt_mlp_forward(ctypes.byref(m), None) == 1   # null pointers
    m.T = 33
    assert L.ttt_mlp_forward(ctypes.byref(m), None) == 1
    dargs = ttt_lib.DecodeArgs()
    dargs.B, dargs.H, dargs.d, dargs.io_dtype = 2, 2, 64, ttt_lib.TTT_BF16
    assert L.ttt_linear_decode_step(ctypes.byref(dargs), None) == 1
    dargs.d = 24
    assert L.ttt_linear_decode_step(ctypes.byref(dargs), None) == 2


def _decode_args(ttt, **kw):
    a = ttt.DecodeArgs()
    a.B, a.H, a.d, a.io_dtype = 2, 2, 64, ttt.TTT_BF16
    fake = 1 << 20  # aligned fake device address; never dereferenced (validation fails first)
    a.W = a.q = a.k = a.v = a.z = fake
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(use_ln=2), 1),
    (dict(use_ln=1), 1),                                           # no c, gamma, beta
    (dict(use_ln=1, c=1 << 20, ln_gamma=1 << 20, ln_beta=1 << 20), 1),   # eps = 0
    (dict(use_ln=1, c=(1 << 20) + 4, ln_gamma=1 << 20, ln_beta=1 << 20, ln_eps=1e-6), 1),  # misaligned c
    (dict(use_ln=1, c=1 << 20, ln_gamma=None, ln_beta=1 << 20, ln_eps=1e-6), 1),
    (dict(use_ln=1, c=1 << 20, ln_gamma=1 << 20, ln_beta=1 << 20, ln_eps=1e-6, d=48), 2),
    (dict(B=0, use_ln=1), 0),                                      # empty: no-op before pointer checks
])
def test_ln_decode_validation(ttt_lib, kw, code):
    a = _decode_args(ttt_lib, **kw)
    assert ttt_lib.library().ttt_linear_decode_step(ctypes.byref(a), None) == code


def _mlp_decode_args(ttt, **kw):
    a = ttt.MlpDecodeArgs()
    a.B, a.H, a.d, a.io_dtype = 2, 2, 64, ttt.TTT_BF16
    fake = 1 << 20
    a.W1 = a.c1 = a.W2 = a.c2 = a.q = a.k = a.v = a.z = fake
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(W1=None), 1),
    (dict(c1=(1 << 20) + 4), 1),
    (dict(W2=None), 1),
    (dict(c2=None), 1),
    (dict(z=None), 1),
    (dict(eta=(1 << 20) + 8), 1),
    (dict(io_dtype=5), 1),
    (dict(d=48), 2),
    (dict(d=0), 1),
    (dict(B=-1), 1),
    (dict(B=0, W1=None), 0),
])
def test_mlp_decode_validation(ttt_lib, kw, code):
    a = _mlp_decode_args(ttt_lib, **kw)
    assert ttt_lib.library().ttt_mlp_decode_step(ctypes.byref(a), None) == code


def test_mlp_ln_validation(ttt_lib):
    L = ttt_lib.library()
    fake = 1 << 20
    m = ttt_lib.MlpArgs()
    m.B, m.H, m.T, m.d, m.b, m.io_dtype = 1, 1, 32, 64, 16, ttt_lib.TTT_BF16
    m.Q = m.K = m.V = m.Z = m.W1 = m.W2 = m.W1_out = m.W2_out = fake
    m.use_ln = 2
    assert L.ttt_mlp_forward(ctypes.byref(m), None) == 1
    m.use_ln = 1                     # no gamma / beta
    assert L.ttt_mlp_forward(ctypes.byref(m), None) == 1
    m.ln_gamma = m.ln_beta = fake    # eps = 0
    assert L.ttt_mlp_forward(ctypes.byref(m), None) == 1
    m.ln_eps = 1e-6
    m.ln_beta = fake + 4             # misaligned
    assert L.ttt_mlp_forward(ctypes.byref(m), None) == 1


def _mlp_backward_args(ttt, **kw):
    a = ttt.MlpBackwardArgs()
    a.B, a.H, a.T, a.d, a.b, a.io_dtype = 1, 2, 32, 64, 16, ttt.TTT_BF16
    fake = 1 << 20
    a.Q = a.K = a.V = a.W_states = a.dQ = a.dK = a.dV = a.dW1 = a.dc1 = a.dW2 = a.dc2 = fake
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(T=30), 1),
    (dict(b=0), 1),
    (dict(d=48), 2),
    (dict(b=32, T=64), 2),                       # the b x 4d intermediates exceed shared memory at d = 64
    (dict(io_dtype=3), 1),
    (dict(W_states=None), 1),
    (dict(dQ=None), 1),
    (dict(dW1=None), 1),
    (dict(dc2=(1 << 20) + 4), 1),
    (dict(dZ=(1 << 20) + 2), 1),
    (dict(dW2_out=(1 << 20) + 8), 1),
    (dict(deta=(1 << 20) + 4), 1),
    (dict(flags=0x2), 1),
    (dict(B=0, Q=None, dW1=None), 0),
    (dict(use_ln=2), 1),
    (dict(use_ln=1), 1),                                       # no gamma / beta / eps / dgamma / dbeta
    (dict(use_ln=1, ln_gamma=1 << 20, ln_beta=1 << 20, ln_eps=1e-6, dgamma=1 << 20,
          dbeta=(1 << 20) + 4), 1),                            # misaligned dbeta
    (dict(use_ln=1, ln_gamma=1 << 20, ln_beta=1 << 20, dgamma=1 << 20, dbeta=1 << 20), 1),   # eps = 0
    (dict(use_ln=1, ln_gamma=1 << 20, ln_beta=1 << 20, ln_eps=1e-6, dgamma=1 << 20, dbeta=1 << 20, b=32,
          T=64), 2),                                           # the LN variant's shared memory at d = 64
])
def test_mlp_backward_validation(ttt_lib, kw, code):
    a = _mlp_backward_args(ttt_lib, **kw)
    assert ttt_lib.library().ttt_mlp_backward(ctypes.byref(a), None) == code


def test_mlp_forward_states_rules(ttt_lib):
    L = ttt_lib.library()
    fake = 1 << 20
    m = ttt_lib.MlpArgs()
    m.B, m.H, m.T, m.d, m.b, m.io_dtype = 1, 1, 32, 64, 16, ttt_lib.TTT_BF16
    m.Q = m.K = m.V = m.Z = m.W1 = m.W2 = m.W1_out = m.W2_out = fake
    m.W_states = fake + 4                        # misaligned
    assert L.ttt_mlp_forward(ctypes.byref(m), None) == 1
    m.W_states = fake
    m.use_ln, m.ln_gamma, m.ln_beta, m.ln_eps = 1, fake, fake, 0.0
    assert L.ttt_mlp_forward(ctypes.byref(m), None) == 1   # the LN variant still needs eps > 0


def _prologue_args(ttt, **kw):
    a = ttt.QkvPrologueArgs()
    a.B, a.T, a.Dm, a.H, a.d, a.io_dtype = 2, 64, 768, 12, 64, ttt.TTT_BF16
    fake = 1 << 20
    a.x = a.theta_q = a.theta_k = a.theta_v = a.theta_lr = a.Q = a.K = a.V = a.eta = fake
    a.eta_base = 1.0
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), 1),
    (dict(T=-1), 1),
    (dict(Dm=0), 1),
    (dict(H=0), 1),
    (dict(d=0), 1),
    (dict(io_dtype=4), 1),
    (dict(io_dtype=0, flags=0x100), 2),          # the fp32 kernel has no stall hook
    (dict(d=48), 2),
    (dict(H=257), 2),                            # the gate tile holds at most 256 heads
    (dict(Dm=772), 2),                           # rows of x must be 16-byte multiples
    (dict(theta_lr=None), 1),                    # gate pointers come in pairs
    (dict(eta=None), 1),
    (dict(flags=0x2), 1),                        # only FORCE_SIMT and the stall hook are valid flags
    (dict(x=None), 1),
    (dict(theta_v=(1 << 20) + 2), 1),
    (dict(Q=None), 1),
    (dict(K=(1 << 20) + 8), 1),
    (dict(eta=(1 << 20) + 4), 1),
    (dict(B=0, x=None, Q=None), 0),              # nothing to do
    (dict(T=0, x=None, Q=None), 0),
])
def test_qkv_prologue_validation(ttt_lib, kw, code):
    a = _prologue_args(ttt_lib, **kw)
    assert ttt_lib.library().ttt_qkv_prologue(ctypes.byref(a), None) == code


def test_binding_refuses_cpu_tensors(ttt_lib):
    import torch
    x = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ttt_lib.linear_forward(x, x, x, None, torch.zeros(1, 64, 64), 16)
