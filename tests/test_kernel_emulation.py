"""The library's kernels' own source, run on the CPU under a host emulation of
the CUDA execution model (tests/emulation: one std::thread per CUDA thread,
__syncthreads as a barrier, shuffles, ldmatrix and mma through a per-warp
exchange with the PTX ISA's documented fragment layouts; for the tcgen05
kernels also mbarriers, 2-D TMA loads and stores, tensor memory and
tcgen05.mma, with asynchronous operations completing at issue), against the
float64 oracle.

This checks the source's index arithmetic, phase order and barrier placement
where no GPU is present.  Beyond parity: a deferred-completion mode (late
asynchronous copies, MMAs and TMEM accesses) and a serial scheduler (one
thread at a time, in index order) turn a missing wait or barrier into wrong
data; guards around every shared buffer and every array catch accesses
outside them; the stall hook checks that every wait ends.  It is not the GPU parity: the tests marked gpu run
the same kernels on the B200 through the C ABI, and the library itself has no
CPU path.

Covered: the TTT-MLP forward writing its batch-start states and the
outer-loop backward that reads them (fp32 CUDA cores); the TTT-Linear pair
on mma.sync (bf16, d = 64, b = 16) -- already verified on the B200, which
pins the emulated ldmatrix / mma semantics; and the LN+residual pair on
mma.sync; the TTT-MLP training pair on mma.sync; the fused prologue on fp32
CUDA cores and on tcgen05; and the TTT-Linear and TTT-MLP tensor-core
prefills (tcgen05, already verified on the B200, which pin the emulated
tcgen05 semantics) (paper digest
"论文速览 | TTT", sections 3.3, 3.4, 3.6, 3.7, 4.4, 4.6, 6.12).
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as O
from test_sequence_layers_head_b200 import workloads as WL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "emulation", "kernels_emu.cpp")


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("emu") / "kernels_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O1", "-fPIC", "-shared", "-I/usr/local/cuda/include", "-o", so, SRC,
                    "-lpthread"], check=True)
    return ctypes.CDLL(so)


# Arrays handed to the kernels come with 4 KB guard bands on both sides, filled
# with a pattern; every test checks afterwards that no kernel wrote into them
# (on the GPU, a write outside the caller's buffer).
_GUARD_BYTES = 4096
_guards = []


def _guarded(shape, dtype, fill):
    dtype = np.dtype(dtype)
    n = int(np.prod(shape))
    pad = _GUARD_BYTES // dtype.itemsize
    raw = np.empty(n + 2 * pad, dtype)
    raw.view(np.uint8)[:] = 0xA5
    raw[pad:pad + n] = fill
    _guards.append((raw, pad, n))
    return raw[pad:pad + n].reshape(shape)


def gzeros(shape, dtype=np.float64):
    return _guarded(shape, dtype, 0)


def gfull(shape, value, dtype):
    return _guarded(shape, dtype, value)


@pytest.fixture(autouse=True)
def no_out_of_bounds_write():
    """After each test: every guard band is intact."""
    _guards.clear()
    yield
    for raw, pad, n in _guards:
        b = raw.view(np.uint8)
        k = pad * raw.itemsize
        assert np.all(b[:k] == 0xA5) and np.all(b[k + n * raw.itemsize:] == 0xA5), "write outside the buffer"
    _guards.clear()


@pytest.fixture(autouse=True)
def no_shared_memory_overrun(request):
    """After each test: no kernel run touched its shared-memory buffer beyond
    the dynamic size the library launches it with (on the GPU, an access
    outside the CTA's allocation)."""
    yield
    for name in ("emu", "tc_emu", "lfr_emu", "mtc_emu"):
        if name in request.fixturenames:
            assert request.getfixturevalue(name).emu_smem_overruns() == 0, name


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def maxrel(x, y):
    return float(np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300)) if y.size else 0.0


def normwise(x, y):
    return float(np.linalg.norm((x - y).ravel()) / max(np.linalg.norm(y.ravel()), 1e-300)) if y.size else 0.0


CASES = [
    # B, H, T, d, b, io dtype, eta per token, upstream state gradients
    (1, 2, 32, 16, 16, WL.F32, True, True),
    (1, 1, 24, 16, 8, WL.F32, False, False),
    (2, 1, 20, 16, 4, WL.F32, True, True),
    (1, 1, 32, 32, 16, WL.F32, True, False),
    (1, 1, 32, 64, 16, WL.F32, True, True),
    (1, 1, 32, 64, 16, WL.BF16, True, True),
    (1, 1, 16, 16, 1, WL.F32, True, True),
    (1, 1, 0, 16, 16, WL.F32, True, True),
]


@pytest.mark.parametrize("B,H,T,d,b,io,per_token,upstream", CASES)
def test_mlp_forward_states_and_backward(emu, B, H, T, d, b, io, per_token, upstream):
    m = 4 * d
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=io, eta_mode="sigmoid", seed=31 + T + d + b)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(7 + d)
    # non-zero biases (the workloads start them at zero)
    c1 = (rng.standard_normal((H, m)) * 0.1).astype(np.float32)
    c2 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32)
    W1, W2 = raw["W1"], raw["W2"]
    eta = raw["eta"] if per_token else None
    eta_const = np.float32(0.02)
    dZd = rng.standard_normal((B, H, T, d))
    dZr, dZe = WL.store(dZd, io)
    ups = ([rng.standard_normal(s).astype(np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
           if upstream else [None] * 4)
    nb = T // b
    iot = np.uint16 if io == WL.BF16 else np.float32
    Z = gzeros((B, H, T, d), iot)
    outs = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
    states = gzeros((B, H, nb, 2 * d * m + m + d), np.float32)
    dQ, dK, dV = (gzeros((B, H, T, d), iot) for _ in range(3))
    deta = gzeros((B, H, T), np.float32)
    grads = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
    emu.emu_mlp_train.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + \
        [ctypes.c_void_p] * 23
    rc = emu.emu_mlp_train(1 if io == WL.BF16 else 0, B, H, T, d, b, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]),
                           _p(eta), eta_const, _p(W1), _p(c1), _p(W2), _p(c2), _p(dZr), *[_p(u) for u in ups],
                           _p(Z), *[_p(o) for o in outs], _p(states), _p(dQ), _p(dK), _p(dV), _p(deta),
                           *[_p(g) for g in grads])
    assert rc == 0

    f64 = lambda a: a.astype(np.float64)
    h = WL.bf16_bits_to_f64 if io == WL.BF16 else f64
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(eta_const))
    params = (f64(W1), f64(c1), f64(W2), f64(c2))
    ref_f = O.mlp_forward(ex["Q"], ex["K"], ex["V"], eta_e, *params, b)
    ref_b = O.mlp_backward(ex["Q"], ex["K"], ex["V"], eta_e, *params, b, dZ=dZe,
                           **{k: (None if u is None else f64(u))
                              for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    # the checkpoints: state i is the oracle's final state after the first i mini-batches
    for i in sorted({0, nb // 2, nb - 1} if nb else set()):
        t = i * b
        st = O.mlp_forward(ex["Q"][:, :, :t], ex["K"][:, :, :t], ex["V"][:, :, :t], eta_e[:, :, :t], *params, b)[1:]
        got = states[:, :, i]
        parts = np.split(got, [d * m, d * m + m, 2 * d * m + m], axis=-1)
        for g, r in zip(parts, st):
            assert maxrel(f64(g).reshape(r.shape), r) < 1e-4

    names = ["dQ", "dK", "dV", "deta", "dW1", "dc1", "dW2", "dc2"]
    gots = [h(dQ), h(dK), h(dV), f64(deta)] + [f64(g) for g in grads]
    for nm, got, ref in zip(names, gots, ref_b):
        if nm == "deta" and not per_token:
            continue
        if io == WL.BF16 and nm in ("dQ", "dK", "dV"):
            assert normwise(got, ref) < 2e-2, nm      # bf16 outputs: normwise bar
        else:
            assert maxrel(got, ref) < 1e-4, (nm, maxrel(got, ref))
    assert (normwise(h(Z), ref_f[0]) < 2e-2) if io == WL.BF16 else (maxrel(h(Z), ref_f[0]) < 1e-4)


@pytest.mark.parametrize("B,H,T,per_token,upstream", [(1, 2, 64, True, True), (2, 1, 48, False, False),
                                                     (1, 1, 16, True, True)])
def test_linear_training_on_mma_sync(emu, B, H, T, per_token, upstream):
    d, b = 64, 16
    inp = WL.random_case("linear", B, H, T, d, b, io_dtype=WL.BF16, eta_mode="sigmoid" if per_token else "const",
                         eta_const=0.0 if per_token else 0.05, seed=T + B)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(T)
    dZr, dZe = WL.store(rng.standard_normal((B, H, T, d)), WL.BF16)
    dW = rng.standard_normal((B, H, d, d)).astype(np.float32) if upstream else None
    nb = T // b
    Z = gzeros((B, H, T, d), np.uint16)
    W_out = gzeros((B, H, d, d), np.float32)
    states = gzeros((B, H, nb, d, d), np.float32)
    dQ, dK, dV = (gzeros((B, H, T, d), np.uint16) for _ in range(3))
    deta = gzeros((B, H, T), np.float32)
    dW0 = gzeros((B, H, d, d), np.float32)
    eta = raw["eta"] if per_token else None
    f = emu.emu_linear_train_mma
    f.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 4 + [ctypes.c_float, ctypes.c_void_p, ctypes.c_longlong] + \
        [ctypes.c_void_p] * 10
    assert f(B, H, T, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta), np.float32(inp.w.eta_const),
             _p(raw["W0"]), 0, _p(Z), _p(W_out), _p(states), _p(dZr), _p(dW), _p(dQ), _p(dK), _p(dV), _p(deta),
             _p(dW0)) == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(inp.w.eta_const)))
    Zr, Wr, _ = O.linear_forward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W0"], b)
    assert normwise(WL.bf16_bits_to_f64(Z), Zr) < 2e-2
    assert normwise(W_out.astype(np.float64), Wr) < 2e-2
    for i in range(nb):
        t = i * b
        Wi = O.linear_forward(ex["Q"][:, :, :t], ex["K"][:, :, :t], ex["V"][:, :, :t], eta_e[:, :, :t], ex["W0"],
                              b)[1]
        assert normwise(states[:, :, i].astype(np.float64), Wi) < 2e-2
    ref = O.linear_backward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W0"], b, dZ=dZe,
                            dW_out=None if dW is None else dW.astype(np.float64))
    gots = [WL.bf16_bits_to_f64(dQ), WL.bf16_bits_to_f64(dK), WL.bf16_bits_to_f64(dV), deta.astype(np.float64),
            dW0.astype(np.float64)]
    for nm, got, want in zip(("dQ", "dK", "dV", "deta", "dW0"), gots, ref):
        if nm == "deta" and not per_token:
            continue
        assert normwise(got, want) < 2e-2, (nm, normwise(got, want))


@pytest.mark.parametrize("B,H,T,per_token,upstream", [(1, 2, 64, True, True), (2, 1, 48, False, False),
                                                     (1, 1, 16, True, True)])
def test_ln_training_on_mma_sync(emu, B, H, T, per_token, upstream):
    d, b = 64, 16
    inp = WL.random_case("ln", B, H, T, d, b, io_dtype=WL.BF16, eta_mode="sigmoid" if per_token else "const",
                         eta_const=0.0 if per_token else 0.05, seed=5 + T)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(1 + T)
    c0 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32)
    dZr, dZe = WL.store(rng.standard_normal((B, H, T, d)), WL.BF16)
    dWo = rng.standard_normal((B, H, d, d)).astype(np.float32) if upstream else None
    dco = rng.standard_normal((B, H, d)).astype(np.float32) if upstream else None
    nb = T // b
    W_out, c_out = gzeros((B, H, d, d), np.float32), gzeros((B, H, d), np.float32)
    Ws, cs = gzeros((B, H, nb, d, d), np.float32), gzeros((B, H, nb, d), np.float32)
    dQ, dK, dV = (gzeros((B, H, T, d), np.uint16) for _ in range(3))
    deta = gzeros((B, H, T), np.float32)
    dW0 = gzeros((B, H, d, d), np.float32)
    dc0, dgam, dbet = (gzeros((B, H, d), np.float32) for _ in range(3))
    f = emu.emu_ln_train_mma
    f.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 4 + \
        [ctypes.c_float] + [ctypes.c_void_p] * 15
    eta = raw["eta"] if per_token else None
    assert f(B, H, T, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta), np.float32(inp.w.eta_const),
             _p(raw["W0"]), _p(c0), _p(raw["gamma"]), _p(raw["beta"]), np.float32(inp.w.ln_eps), _p(W_out),
             _p(c_out), _p(Ws), _p(cs), _p(dZr), _p(dWo), _p(dco), _p(dQ), _p(dK), _p(dV), _p(deta), _p(dW0),
             _p(dc0), _p(dgam), _p(dbet)) == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(inp.w.eta_const)))
    c0e = c0.astype(np.float64)
    _, Wr, cr = O.linear_forward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W0"], b, c0=c0e, gamma=ex["gamma"],
                                 beta=ex["beta"], use_ln=True, eps=inp.w.ln_eps)
    assert normwise(W_out.astype(np.float64), Wr) < 2e-2 and normwise(c_out.astype(np.float64), cr) < 2e-2
    for i in range(1, nb):
        t = i * b
        _, Wi, ci = O.linear_forward(ex["Q"][:, :, :t], ex["K"][:, :, :t], ex["V"][:, :, :t], eta_e[:, :, :t],
                                     ex["W0"], b, c0=c0e, gamma=ex["gamma"], beta=ex["beta"], use_ln=True,
                                     eps=inp.w.ln_eps)
        assert normwise(Ws[:, :, i].astype(np.float64), Wi) < 2e-2
        assert normwise(cs[:, :, i].astype(np.float64), ci) < 2e-2
    ref = O.linear_ln_backward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W0"], b, c0e, ex["gamma"], ex["beta"],
                               inp.w.ln_eps, dZ=dZe, dW_out=None if dWo is None else dWo.astype(np.float64),
                               dc_out=None if dco is None else dco.astype(np.float64))
    h = WL.bf16_bits_to_f64
    gots = [h(dQ), h(dK), h(dV), deta.astype(np.float64)] + [x.astype(np.float64) for x in (dW0, dc0, dgam, dbet)]
    for nm, got, want in zip(("dQ", "dK", "dV", "deta", "dW0", "dc0", "dgamma", "dbeta"), gots, ref):
        if nm == "deta" and not per_token:
            continue
        assert normwise(got, want) < 2e-2, (nm, normwise(got, want))


@pytest.mark.parametrize("B,T,Dm,H,d,gate,io", [(2, 20, 40, 3, 16, True, WL.F32), (1, 33, 264, 2, 64, True, WL.F32),
                                                (1, 17, 64, 7, 64, False, WL.F32), (2, 9, 24, 5, 32, True, WL.BF16)])
def test_prologue_on_cuda_cores(emu, B, T, Dm, H, d, gate, io):
    """The CUDA-core prologue (fp32 input, and bf16 with TTT_FLAG_FORCE_SIMT)
    against the oracle: two column blocks when 3 H d + H > 1024, ragged token
    blocks, no gate."""
    w, inp = WL.prologue_case(B, T, Dm, H, d, gate=gate, eta_base=0.5)
    e = inp["exact"]
    if io == WL.F32:
        raw = {k: v.astype(np.float32) for k, v in e.items()}
        iot = np.float32
    else:
        raw, iot = inp["raw"], np.uint16
    Q, K, V = (gzeros((B, H, T, d), iot) for _ in range(3))
    eta = gzeros((B, H, T), np.float32) if gate else None
    f = emu.emu_prologue_simt
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 5 + [ctypes.c_float] + [ctypes.c_void_p] * 4
    assert f(0 if io == WL.F32 else 1, B, T, Dm, H, d, _p(raw["x"]), _p(raw["theta_q"]), _p(raw["theta_k"]),
             _p(raw["theta_v"]), _p(raw["theta_lr"]) if gate else None, 0.5, _p(Q), _p(K), _p(V), _p(eta)) == 0
    ref = O.qkv_prologue(e["x"], e["theta_q"], e["theta_k"], e["theta_v"], e["theta_lr"], 0.5, d)
    h = (lambda a: a.astype(np.float64)) if io == WL.F32 else WL.bf16_bits_to_f64
    for got, want in zip((Q, K, V), ref[:3]):
        if io == WL.F32:
            assert maxrel(h(got), want) < 1e-4
        else:
            assert normwise(h(got), want) < 2e-2
    if gate:
        assert maxrel(eta.astype(np.float64), ref[3]) < 1e-4


@pytest.mark.parametrize("B,H,T,per_token,upstream", [(1, 2, 32, True, True), (1, 1, 48, False, False)])
def test_mlp_backward_on_mma_sync(emu, B, H, T, per_token, upstream):
    """The TTT-MLP backward on mma.sync (bf16, d = 64, b = 16) from the states
    the CUDA-core forward writes, against the oracle (bf16 bar)."""
    d, b, m = 64, 16, 256
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=WL.BF16, eta_mode="sigmoid" if per_token else "const",
                         eta_const=0.0 if per_token else 0.02, seed=41 + T)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(100 + T)
    c1 = (rng.standard_normal((H, m)) * 0.1).astype(np.float32)
    c2 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32)
    dZr, dZe = WL.store(rng.standard_normal((B, H, T, d)), WL.BF16)
    ups = ([rng.standard_normal(s).astype(np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
           if upstream else [None] * 4)
    nb = T // b
    Z = gzeros((B, H, T, d), np.uint16)
    outs = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
    states = gzeros((B, H, nb, 2 * d * m + m + d), np.float32)
    eta = raw["eta"] if per_token else None
    f = emu.emu_mlp_forward
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 10
    assert f(1, B, H, T, d, b, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta), np.float32(inp.w.eta_const),
             _p(raw["W1"]), _p(c1), _p(raw["W2"]), _p(c2), _p(Z), *[_p(o) for o in outs], _p(states)) == 0
    dQ, dK, dV = (gzeros((B, H, T, d), np.uint16) for _ in range(3))
    deta = gzeros((B, H, T), np.float32)
    grads = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
    g = emu.emu_mlp_backward_mma
    g.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 14
    assert g(B, H, T, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta), np.float32(inp.w.eta_const), _p(states),
             _p(dZr), *[_p(u) for u in ups], _p(dQ), _p(dK), _p(dV), _p(deta), *[_p(x) for x in grads]) == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(inp.w.eta_const)))
    ref = O.mlp_backward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W1"], c1.astype(np.float64), ex["W2"],
                         c2.astype(np.float64), b, dZ=dZe,
                         **{k: (None if u is None else u.astype(np.float64))
                            for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    h = WL.bf16_bits_to_f64
    gots = [h(dQ), h(dK), h(dV), deta.astype(np.float64)] + [x.astype(np.float64) for x in grads]
    for nm, got, want in zip(("dQ", "dK", "dV", "deta", "dW1", "dc1", "dW2", "dc2"), gots, ref):
        if nm == "deta" and not per_token:
            continue
        assert normwise(got, want) < 2e-2, (nm, normwise(got, want))


@pytest.mark.parametrize("B,H,T,per_token", [(1, 2, 48, True), (2, 1, 32, False), (1, 1, 0, True)])
def test_mlp_forward_states_on_mma_sync(emu, B, H, T, per_token):
    """The TTT-MLP forward writing its batch-start states on mma.sync (bf16, d = 64, b = 16): Z, the final
    state and every checkpoint against the oracle (bf16 bar)."""
    d, b, m = 64, 16, 256
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=WL.BF16, eta_mode="sigmoid" if per_token else "const",
                         eta_const=0.0 if per_token else 0.02, seed=61 + T)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(200 + T)
    c1 = (rng.standard_normal((H, m)) * 0.1).astype(np.float32)
    c2 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32)
    nb = T // b
    Z = gzeros((B, H, T, d), np.uint16)
    outs = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
    states = gzeros((B, H, max(nb, 1), 2 * d * m + m + d), np.float32)
    eta = raw["eta"] if per_token else None
    f = emu.emu_mlp_forward_mma
    f.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 10
    assert f(B, H, T, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta), np.float32(inp.w.eta_const), _p(raw["W1"]),
             _p(c1), _p(raw["W2"]), _p(c2), _p(Z), *[_p(o) for o in outs], _p(states)) == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(inp.w.eta_const)))
    params = (ex["W1"], c1.astype(np.float64), ex["W2"], c2.astype(np.float64))
    ref = O.mlp_forward(ex["Q"], ex["K"], ex["V"], eta_e, *params, b)
    if T:
        assert normwise(WL.bf16_bits_to_f64(Z), ref[0]) < 2e-2
    for got, want in zip(outs, ref[1:]):
        assert normwise(got.astype(np.float64), want) < 2e-2
    for i in range(nb):
        t = i * b
        st = O.mlp_forward(ex["Q"][:, :, :t], ex["K"][:, :, :t], ex["V"][:, :, :t], eta_e[:, :, :t], *params, b)[1:]
        parts = np.split(states[:, :, i], [d * m, d * m + m, 2 * d * m + m], axis=-1)
        for g, r in zip(parts, st):
            assert normwise(g.astype(np.float64).reshape(r.shape), r) < 2e-2


@pytest.fixture(scope="module")
def tc_emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("tcemu") / "tc_kernels_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O1", "-fPIC", "-shared", "-I/usr/local/cuda/include", "-o", so,
                    os.path.join(ROOT, "tests", "emulation", "tc_kernels_emu.cpp"), "-lpthread"], check=True)
    return ctypes.CDLL(so)


@pytest.mark.parametrize("B,T,Dm,H,d,gate,grid", [
    (1, 8, 64, 1, 16, True, 1),        # one tile of each kind
    (2, 200, 136, 5, 64, True, 3),     # ragged tokens and width, a partial column tile, persistent CTAs
    (3, 100, 72, 17, 16, True, 2),     # H not a multiple of 16 in the gate tile
    (2, 77, 64, 12, 64, False, 4),     # no gate
    (4, 33, 16, 7, 32, True, 1),       # width below one chunk
    (2, 64, 768, 12, 64, True, 7),     # the 12-head width
])
@pytest.mark.parametrize("deferred", [False, True])
def test_prologue_on_tcgen05(tc_emu, B, T, Dm, H, d, gate, grid, deferred):
    """The tcgen05 prologue kernel with the library's tile plan and tensor maps: every output written, the
    views within one bf16 rounding plus the fp32 accumulation bound, the gate within its bound, no
    emulated-hardware rule broken (TMA alignment, TMEM lane quadrant, MMA shape), no expired wait.  With
    `deferred`, the asynchronous operations complete late (loads overtaking MMAs, stores held until
    waited for): a missing or misplaced wait then shows as wrong data."""
    w, inp = WL.prologue_case(B, T, Dm, H, d, gate=gate, eta_base=0.5)
    r, e = inp["raw"], inp["exact"]
    Q, K, V = (gfull((B, H, T, d), 0x7FC0, np.uint16) for _ in range(3))   # NaN until written
    eta = gfull((B, H, T), np.nan, np.float32) if gate else None
    status = gzeros(1, np.int32)
    f = tc_emu.emu_prologue_tc
    f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 5 + [ctypes.c_float] + [ctypes.c_void_p] * 4 + \
        [ctypes.c_int, ctypes.c_void_p]
    tc_emu.emu_deferred(int(deferred))
    try:
        rc = f(B, T, Dm, H, d, _p(r["x"]), _p(r["theta_q"]), _p(r["theta_k"]), _p(r["theta_v"]),
               _p(r["theta_lr"]) if gate else None, 0.5, _p(Q), _p(K), _p(V), _p(eta), grid, _p(status))
    finally:
        tc_emu.emu_deferred(0)
    assert rc == 0 and status[0] == 0
    ref = O.qkv_prologue(e["x"], e["theta_q"], e["theta_k"], e["theta_v"], e["theta_lr"], 0.5, d)
    for got, want, nm in zip((Q, K, V), ref[:3], ("theta_q", "theta_k", "theta_v")):
        g = WL.bf16_bits_to_f64(got)
        S = (np.abs(e["x"]) @ np.abs(e[nm]).T).reshape(B, T, H, d).transpose(0, 2, 1, 3)
        assert np.all(np.isfinite(g))
        assert np.all(np.abs(g - want) <= 2.0 ** -8 * np.abs(want) + 2.0 ** -12 * S)
    if gate:
        S_lr = (np.abs(e["x"]) @ np.abs(e["theta_lr"]).T).transpose(0, 2, 1)
        assert np.all(np.isfinite(eta))
        assert np.all(np.abs(eta - ref[3]) <= 0.5 * (2.0 ** -12 * S_lr / 4 + 1e-6))


@pytest.mark.parametrize("B,H,T,d,b,io,per_token,upstream", [
    (1, 2, 32, 16, 16, WL.F32, True, True),
    (2, 1, 24, 16, 8, WL.F32, False, False),
    (1, 1, 32, 64, 16, WL.F32, True, True),
    (1, 1, 32, 64, 16, WL.BF16, True, True),
    (1, 1, 16, 16, 1, WL.F32, True, True),
])
def test_mlp_ln_forward_states_and_backward(emu, B, H, T, d, b, io, per_token, upstream):
    """TTT-MLP with LN+residual on fp32 CUDA cores: the forward writing its states and the backward
    (with dgamma, dbeta) against the oracle's reverse mode."""
    m = 4 * d
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=io, eta_mode="sigmoid", seed=5 + T + d)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(3 + d)
    c1 = (rng.standard_normal((H, m)) * 0.1).astype(np.float32)
    c2 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32)
    gam = (1 + rng.standard_normal((H, d)) * 0.2).astype(np.float32)
    bet = (rng.standard_normal((H, d)) * 0.2).astype(np.float32)
    dZr, dZe = WL.store(rng.standard_normal((B, H, T, d)), io)
    ups = ([rng.standard_normal(s).astype(np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
           if upstream else [None] * 4)
    nb = T // b
    iot = np.uint16 if io == WL.BF16 else np.float32
    states = gzeros((B, H, nb, 2 * d * m + m + d), np.float32)
    dQ, dK, dV = (gzeros((B, H, T, d), iot) for _ in range(3))
    deta = gzeros((B, H, T), np.float32)
    g = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d), (B, H, d), (B, H, d))]
    eta = raw["eta"] if per_token else None
    f = emu.emu_mlp_ln_train
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 6 + \
        [ctypes.c_float] + [ctypes.c_void_p] * 16
    assert f(1 if io == WL.BF16 else 0, B, H, T, d, b, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta),
             np.float32(0.02), _p(raw["W1"]), _p(c1), _p(raw["W2"]), _p(c2), _p(gam), _p(bet), np.float32(1e-6),
             _p(dZr), *[_p(u) for u in ups], _p(states), _p(dQ), _p(dK), _p(dV), _p(deta), *[_p(x) for x in g]) == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(0.02)))
    f64 = lambda a: a.astype(np.float64)
    ref = O.mlp_ln_backward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W1"], f64(c1), ex["W2"], f64(c2), b, f64(gam),
                            f64(bet), 1e-6, dZ=dZe,
                            **{k: (None if u is None else f64(u))
                               for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    h = WL.bf16_bits_to_f64 if io == WL.BF16 else f64
    gots = [h(dQ), h(dK), h(dV), f64(deta)] + [f64(x) for x in g]
    names = ("dQ", "dK", "dV", "deta", "dW1", "dc1", "dW2", "dc2", "dgamma", "dbeta")
    for nm, got, want in zip(names, gots, ref):
        if nm == "deta" and not per_token:
            continue
        if io == WL.BF16 and nm in ("dQ", "dK", "dV"):
            assert normwise(got, want) < 2e-2, nm
        else:
            assert maxrel(got, want) < 1e-4, (nm, maxrel(got, want))


@pytest.mark.parametrize("B,H,T,per_token,upstream", [(1, 2, 32, True, True), (1, 1, 48, False, False)])
def test_mlp_ln_backward_on_mma_sync(emu, B, H, T, per_token, upstream):
    """The TTT-MLP with LN+residual backward on mma.sync (bf16, d = 64, b = 16), from the states the
    CUDA-core LN forward writes, against the oracle (bf16 bar), dgamma and dbeta included."""
    d, b, m = 64, 16, 256
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=WL.BF16, eta_mode="sigmoid", seed=5 + T)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(3 + T)
    c1 = (rng.standard_normal((H, m)) * 0.1).astype(np.float32)
    c2 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32)
    gam = (1 + rng.standard_normal((H, d)) * 0.2).astype(np.float32)
    bet = (rng.standard_normal((H, d)) * 0.2).astype(np.float32)
    dZr, dZe = WL.store(rng.standard_normal((B, H, T, d)), WL.BF16)
    ups = ([rng.standard_normal(s).astype(np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
           if upstream else [None] * 4)
    nb = T // b
    Z = gzeros((B, H, T, d), np.uint16)
    outs = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
    states = gzeros((B, H, nb, 2 * d * m + m + d), np.float32)
    eta = raw["eta"] if per_token else None
    f = emu.emu_mlp_ln_forward
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 6 + \
        [ctypes.c_float] + [ctypes.c_void_p] * 6
    assert f(1, B, H, T, d, b, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta), np.float32(0.02), _p(raw["W1"]),
             _p(c1), _p(raw["W2"]), _p(c2), _p(gam), _p(bet), np.float32(1e-6), _p(Z), *[_p(o) for o in outs],
             _p(states)) == 0
    dQ, dK, dV = (gzeros((B, H, T, d), np.uint16) for _ in range(3))
    deta = gzeros((B, H, T), np.float32)
    g = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d), (B, H, d), (B, H, d))]
    bw = emu.emu_mlp_ln_backward_mma
    bw.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 8 + \
        [ctypes.c_float] + [ctypes.c_void_p] * 10
    assert bw(B, H, T, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta), np.float32(0.02), _p(states), _p(dZr),
              *[_p(u) for u in ups], _p(gam), _p(bet), np.float32(1e-6), _p(dQ), _p(dK), _p(dV), _p(deta),
              *[_p(x) for x in g]) == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(0.02)))
    f64 = lambda a: a.astype(np.float64)
    ref = O.mlp_ln_backward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W1"], f64(c1), ex["W2"], f64(c2), b, f64(gam),
                            f64(bet), 1e-6, dZ=dZe,
                            **{k: (None if u is None else f64(u))
                               for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    h = WL.bf16_bits_to_f64
    gots = [h(dQ), h(dK), h(dV), f64(deta)] + [f64(x) for x in g]
    names = ("dQ", "dK", "dV", "deta", "dW1", "dc1", "dW2", "dc2", "dgamma", "dbeta")
    for nm, got, want in zip(names, gots, ref):
        if nm == "deta" and not per_token:
            continue
        assert normwise(got, want) < 2e-2, (nm, normwise(got, want))


@pytest.mark.parametrize("B,H,T,per_token", [(1, 2, 48, True), (2, 1, 32, False)])
def test_mlp_ln_forward_states_on_mma_sync(emu, B, H, T, per_token):
    """TTT-MLP with LN+residual, the forward writing its batch-start states on mma.sync (bf16, d = 64,
    b = 16): Z, the final state and every checkpoint against the oracle (bf16 bar)."""
    d, b, m = 64, 16, 256
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=WL.BF16, eta_mode="sigmoid" if per_token else "const",
                         eta_const=0.0 if per_token else 0.02, seed=81 + T)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(300 + T)
    c1 = (rng.standard_normal((H, m)) * 0.1).astype(np.float32)
    c2 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32)
    gam = (1 + rng.standard_normal((H, d)) * 0.2).astype(np.float32)
    bet = (rng.standard_normal((H, d)) * 0.2).astype(np.float32)
    nb = T // b
    Z = gzeros((B, H, T, d), np.uint16)
    outs = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
    states = gzeros((B, H, nb, 2 * d * m + m + d), np.float32)
    eta = raw["eta"] if per_token else None
    f = emu.emu_mlp_ln_forward_mma
    f.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 6 + \
        [ctypes.c_float] + [ctypes.c_void_p] * 6
    assert f(B, H, T, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta), np.float32(inp.w.eta_const), _p(raw["W1"]),
             _p(c1), _p(raw["W2"]), _p(c2), _p(gam), _p(bet), np.float32(1e-6), _p(Z), *[_p(o) for o in outs],
             _p(states)) == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(inp.w.eta_const)))
    f64 = lambda a: a.astype(np.float64)
    params = (ex["W1"], f64(c1), ex["W2"], f64(c2))
    ln = dict(use_ln=True, gamma=f64(gam), beta=f64(bet))
    ref = O.mlp_forward(ex["Q"], ex["K"], ex["V"], eta_e, *params, b, **ln)
    assert normwise(WL.bf16_bits_to_f64(Z), ref[0]) < 2e-2
    for got, want in zip(outs, ref[1:]):
        assert normwise(f64(got), want) < 2e-2
    for i in range(nb):
        t = i * b
        st = O.mlp_forward(ex["Q"][:, :, :t], ex["K"][:, :, :t], ex["V"][:, :, :t], eta_e[:, :, :t], *params, b,
                           **ln)[1:]
        parts = np.split(states[:, :, i], [d * m, d * m + m, 2 * d * m + m], axis=-1)
        for g, r in zip(parts, st):
            assert normwise(f64(g).reshape(r.shape), r) < 2e-2


@pytest.fixture(scope="module")
def lfr_emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("lfr") / "tc_linear_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O1", "-fPIC", "-shared", "-I/usr/local/cuda/include", "-o", so,
                    os.path.join(ROOT, "tests", "emulation", "tc_linear_emu.cpp"), "-lpthread"], check=True)
    return ctypes.CDLL(so)


@pytest.mark.parametrize("ln,upc,B,H,T,per_token", [
    (False, 2, 1, 2, 64, True), (False, 1, 1, 1, 48, False), (False, 2, 1, 3, 80, True),
    (True, 2, 1, 2, 64, True), (True, 1, 2, 1, 48, False), (True, 2, 1, 3, 48, True),
    (False, 2, 1, 2, 256, False)])   # long enough that a stale state shows above the bar
@pytest.mark.parametrize("deferred", [False, True])
def test_linear_prefill_on_tcgen05(lfr_emu, ln, upc, B, H, T, per_token, deferred):
    """The TTT-Linear tensor-core prefill (B200-verified) under the emulated
    tcgen05 operations.  Its agreement with the oracle pins the emulation of
    the MMA operand descriptors (K-major and MN-major 128-byte swizzle, K-major
    without swizzle, A in tensor memory), the 32x32b TMEM loads and stores, the
    accumulator layout of the 16x256b load, stmatrix.trans and the 32- and
    64-byte swizzled TMA stores.  The state update W_T - W_0 is compared on its
    own: the full state is dominated by W_0.  `deferred` as in the prologue's test."""
    d, b = 64, 16
    inp = WL.random_case("ln" if ln else "linear", B, H, T, d, b, io_dtype=WL.BF16,
                         eta_mode="sigmoid" if per_token else "const", eta_const=0.0 if per_token else 0.05,
                         seed=3 + T)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(2 + T)
    c0 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32) if ln else None
    Z = gzeros((B, H, T, d), np.uint16)
    W_out = gzeros((B, H, d, d), np.float32)
    c_out = gzeros((B, H, d), np.float32) if ln else None
    status = gzeros(1, np.int32)
    eta = raw["eta"] if per_token else None
    f = lfr_emu.emu_linear_tc
    f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 4 + [ctypes.c_float, ctypes.c_void_p, ctypes.c_longlong,
                                                                ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p,
                                                                ctypes.c_void_p, ctypes.c_float] + \
        [ctypes.c_void_p] * 4
    lfr_emu.emu_deferred(int(deferred))
    try:
        rc = f(int(ln), upc, B, H, T, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta),
               np.float32(inp.w.eta_const), _p(raw["W0"]), 0, _p(c0), 0, _p(raw["gamma"]) if ln else None,
               _p(raw["beta"]) if ln else None, np.float32(inp.w.ln_eps if ln else 0.0), _p(Z), _p(W_out), _p(c_out),
               _p(status))
    finally:
        lfr_emu.emu_deferred(0)
    assert rc == 0 and status[0] == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(inp.w.eta_const)))
    if ln:
        c0e = c0.astype(np.float64)
        Zr, Wr, cr = O.linear_forward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W0"], b, c0=c0e, gamma=ex["gamma"],
                                      beta=ex["beta"], use_ln=True, eps=inp.w.ln_eps)
        c0b = np.broadcast_to(c0e, cr.shape)
        assert normwise(c_out.astype(np.float64) - c0b, cr - c0b) < 2e-2
    else:
        Zr, Wr, _ = O.linear_forward(ex["Q"], ex["K"], ex["V"], eta_e, ex["W0"], b)
    W0b = np.broadcast_to(ex["W0"], Wr.shape)
    assert normwise(WL.bf16_bits_to_f64(Z), Zr) < 2e-2
    assert normwise(W_out.astype(np.float64), Wr) < 2e-2
    assert normwise(W_out.astype(np.float64) - W0b, Wr - W0b) < 2e-2


@pytest.fixture(scope="module")
def mtc_emu(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("mtc") / "tc_mlp_emu.so")
    subprocess.run(["g++", "-std=c++20", "-O1", "-fPIC", "-shared", "-I/usr/local/cuda/include", "-o", so,
                    os.path.join(ROOT, "tests", "emulation", "tc_mlp_emu.cpp"), "-lpthread"], check=True)
    return ctypes.CDLL(so)


@pytest.mark.parametrize("ln,B,H,T,per_token,biases,per_seq", [
    (False, 1, 1, 32, True, True, False), (True, 1, 1, 32, True, True, False), (False, 2, 1, 48, False, True, False),
    (True, 1, 2, 48, True, False, False), (False, 1, 1, 16, True, True, False), (False, 2, 1, 32, True, True, True)])
@pytest.mark.parametrize("deferred", [False, True])
def test_mlp_prefill_on_tcgen05(mtc_emu, ln, B, H, T, per_token, biases, per_seq, deferred):
    """The TTT-MLP tensor-core prefill (B200-verified) under the emulated
    tcgen05 operations.  Its agreement with the oracle pins the emulation of
    the M = 64 accumulator layout (rows in lanes 0-15 of each quadrant), the
    MN-major A operand, the 16x128b TMEM store, the 16x256b x1 load and the x2
    ldmatrix / stmatrix forms.  Each parameter's update (final minus initial)
    is compared on its own.  `deferred` as in the prologue's test."""
    d, b, m = 64, 16, 256
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=WL.BF16, eta_mode="sigmoid" if per_token else "const",
                         eta_const=0.0 if per_token else 0.05, seed=11 + T + B)
    raw, ex = inp.raw, inp.exact
    rng = np.random.default_rng(5 + T)
    lead = (B, H) if per_seq else (H,)
    if per_seq:
        W1 = (raw["W1"][None] + 0.01 * rng.standard_normal((B,) + raw["W1"].shape)).astype(np.float32)
        W2 = (raw["W2"][None] + 0.01 * rng.standard_normal((B,) + raw["W2"].shape)).astype(np.float32)
    else:
        W1, W2 = raw["W1"], raw["W2"]
    c1 = (rng.standard_normal(lead + (m,)) * 0.1).astype(np.float32) if biases else gzeros(lead + (m,), np.float32)
    c2 = (rng.standard_normal(lead + (d,)) * 0.1).astype(np.float32) if biases else gzeros(lead + (d,), np.float32)
    gam = (1 + 0.1 * rng.standard_normal((H, d))).astype(np.float32)
    bet = (0.1 * rng.standard_normal((H, d))).astype(np.float32)
    Z = gzeros((B, H, T, d), np.uint16)
    outs = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
    status = gzeros(1, np.int32)
    eta = raw["eta"] if per_token else None
    f = mtc_emu.emu_mlp_tc
    f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 6 + \
        [ctypes.c_float] + [ctypes.c_void_p] * 6
    mtc_emu.emu_deferred(int(deferred))
    try:
        rc = f(int(ln), B, H, T, int(per_seq), _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(eta),
               np.float32(inp.w.eta_const), _p(W1), _p(c1), _p(W2), _p(c2), _p(gam) if ln else None,
               _p(bet) if ln else None, np.float32(1e-6), _p(Z), *[_p(o) for o in outs], _p(status))
    finally:
        mtc_emu.emu_deferred(0)
    assert rc == 0 and status[0] == 0
    eta_e = ex["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(inp.w.eta_const)))
    f64 = lambda a: a.astype(np.float64)
    ref = O.mlp_forward(ex["Q"], ex["K"], ex["V"], eta_e, f64(W1), f64(c1), f64(W2), f64(c2), b, use_ln=ln,
                        gamma=f64(gam), beta=f64(bet), eps=1e-6)
    assert normwise(WL.bf16_bits_to_f64(Z), ref[0]) < 2e-2
    for nm, got, want, init in zip(("W1", "c1", "W2", "c2"), outs, ref[1:], (W1, c1, W2, c2)):
        i0 = np.broadcast_to(f64(init), want.shape)
        assert normwise(f64(got), want) < 2e-2, nm
        if biases or nm[0] == "W":
            assert normwise(f64(got) - i0, want - i0) < 2e-2, (nm, normwise(f64(got) - i0, want - i0))


@pytest.mark.parametrize("kind", ["prologue", "linear", "linear_one_unit", "mlp", "mlp_ln"])
def test_tcgen05_stall_hook_times_out_and_every_thread_exits(tc_emu, lfr_emu, mtc_emu, kind):
    """The stall hook (the MMA issuer waits on a barrier nothing arrives on)
    with a 20 ms wait limit: the run returns, with kStatusTimeout recorded and
    no emulated-hardware rule broken, so every wait of the kernel's other
    roles ends once the abort flag is up and every thread reaches the end
    (a wait that never ended would hang this test).  The same path runs on the
    B200 in the tests marked gpu."""
    stall, limit = 0x100, 20_000_000
    status = gzeros(1, np.int32)
    if kind == "prologue":
        B, T, Dm, H, d = 2, 200, 136, 5, 64
        w, inp = WL.prologue_case(B, T, Dm, H, d, gate=True, eta_base=0.5)
        r = inp["raw"]
        Q, K, V = (gzeros((B, H, T, d), np.uint16) for _ in range(3))
        eta = gzeros((B, H, T), np.float32)
        tc_emu.emu_prologue_tc_knobs.argtypes = [ctypes.c_uint, ctypes.c_ulonglong]
        tc_emu.emu_prologue_tc_knobs(stall, limit)
        f = tc_emu.emu_prologue_tc
        f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 5 + [ctypes.c_float] + [ctypes.c_void_p] * 4 + \
            [ctypes.c_int, ctypes.c_void_p]
        try:
            rc = f(B, T, Dm, H, d, _p(r["x"]), _p(r["theta_q"]), _p(r["theta_k"]), _p(r["theta_v"]),
                   _p(r["theta_lr"]), 0.5, _p(Q), _p(K), _p(V), _p(eta), 3, _p(status))
        finally:
            tc_emu.emu_prologue_tc_knobs(0, 120_000_000_000)
    elif kind.startswith("linear"):
        B, H, T, d = 1, 3, 64, 64
        inp = WL.random_case("linear", B, H, T, d, 16, io_dtype=WL.BF16, eta_mode="sigmoid", seed=9)
        raw = inp.raw
        Z = gzeros((B, H, T, d), np.uint16)
        W_out = gzeros((B, H, d, d), np.float32)
        lfr_emu.emu_linear_tc_knobs.argtypes = [ctypes.c_uint, ctypes.c_ulonglong]
        lfr_emu.emu_linear_tc_knobs(stall, limit)
        f = lfr_emu.emu_linear_tc
        f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 4 + \
            [ctypes.c_float, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p,
             ctypes.c_void_p, ctypes.c_float] + [ctypes.c_void_p] * 4
        try:
            rc = f(0, 1 if kind.endswith("one_unit") else 2, B, H, T, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]),
                   _p(raw["eta"]), 0.0, _p(raw["W0"]), 0, None, 0, None, None, 0.0, _p(Z), _p(W_out), None,
                   _p(status))
        finally:
            lfr_emu.emu_linear_tc_knobs(0, 120_000_000_000)
    else:
        B, H, T, d, m = 1, 2, 48, 64, 256
        inp = WL.random_case("mlp", B, H, T, d, 16, io_dtype=WL.BF16, eta_mode="sigmoid", seed=9)
        raw = inp.raw
        gam, bet = np.ones((H, d), np.float32), gzeros((H, d), np.float32)
        Z = gzeros((B, H, T, d), np.uint16)
        outs = [gzeros(s, np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
        mtc_emu.emu_mlp_tc_knobs.argtypes = [ctypes.c_uint, ctypes.c_ulonglong]
        mtc_emu.emu_mlp_tc_knobs(stall, limit)
        f = mtc_emu.emu_mlp_tc
        f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 6 + \
            [ctypes.c_float] + [ctypes.c_void_p] * 6
        ln = kind == "mlp_ln"
        try:
            rc = f(int(ln), B, H, T, 0, _p(raw["Q"]), _p(raw["K"]), _p(raw["V"]), _p(raw["eta"]), 0.0,
                   _p(raw["W1"]), _p(raw["c1"]), _p(raw["W2"]), _p(raw["c2"]), _p(gam) if ln else None,
                   _p(bet) if ln else None, np.float32(1e-6), _p(Z), *[_p(o) for o in outs], _p(status))
        finally:
            mtc_emu.emu_mlp_tc_knobs(0, 120_000_000_000)
    assert rc == 0
    assert status[0] & 1


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("name,args", [
    ("test_mlp_backward_on_mma_sync", (1, 1, 32, True, True)),
    ("test_mlp_ln_backward_on_mma_sync", (1, 1, 32, True, True)),
    ("test_mlp_forward_states_on_mma_sync", (1, 1, 32, True)),
    ("test_mlp_ln_forward_states_on_mma_sync", (1, 1, 32, True)),
    ("test_ln_training_on_mma_sync", (1, 1, 32, True, True)),
    ("test_mlp_forward_states_and_backward", (1, 1, 32, 16, 16, WL.F32, True, True)),
    ("test_mlp_ln_forward_states_and_backward", (1, 1, 32, 16, 16, WL.F32, True, True)),
    ("test_prologue_on_cuda_cores", (2, 20, 40, 3, 16, True, WL.F32)),
])
def test_serial_schedules(emu, name, args, mode):
    """The kernels not yet run on the B200 under the serial scheduler
    (emu_core.h): one thread at a time, handing on only at a barrier, a warp
    collective or a spin, the lowest (1) or highest (2) ready thread first, so
    that one warp runs to its next block-wide barrier before the others move.
    A missing __syncthreads (a read before the write it needs, or a write into
    a tile others still read) then gives wrong data deterministically; no run
    may end with every thread blocked."""
    emu.emu_serial(mode)
    try:
        globals()[name](emu, *args)
    finally:
        emu.emu_serial(0)
    assert emu.emu_sched_errors() == 0


@pytest.mark.parametrize("mode", [1, 2])
def test_serial_schedules_tcgen05_prologue(tc_emu, mode):
    """The tcgen05 prologue (not yet run on the B200) under the serial
    scheduler, as above, both with completion at issue and deferred."""
    for deferred in (False, True):
        tc_emu.emu_serial(mode)
        try:
            test_prologue_on_tcgen05(tc_emu, 2, 40, 136, 5, 64, True, 2, deferred)
        finally:
            tc_emu.emu_serial(0)
        assert tc_emu.emu_sched_errors() == 0


@pytest.mark.parametrize("mode", [1, 2])
def test_serial_schedules_tcgen05_verified(lfr_emu, mtc_emu, mode):
    """The two B200-verified tensor-core prefills under the serial scheduler
    with deferred completion: a check of the checker (no false alarm on
    kernels known to be right)."""
    for lib, run in ((lfr_emu, lambda: test_linear_prefill_on_tcgen05(lfr_emu, True, 2, 1, 2, 32, True, True)),
                     (mtc_emu, lambda: test_mlp_prefill_on_tcgen05(mtc_emu, False, 1, 1, 32, True, True, False,
                                                                   True))):
        lib.emu_serial(mode)
        try:
            run()
        finally:
            lib.emu_serial(0)
        assert lib.emu_sched_errors() == 0
