"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Small cases span several mini-batches, odd unit counts (the tensor-core
kernel pairs units per CTA) and every inner model; the full-size workloads
are checked on sampled units that the oracle recomputes one by one.
Tolerances are the problem statement's: max relative error <= 1e-4 for fp32
workloads, normwise <= 2e-2 on Z and on the final state for bf16 inputs with
fp32 state.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from test_sequence_layers_head_b200 import workloads as WL
from tests.gpu_util import assert_close, normwise, poison_like, to_dev, to_host

pytestmark = pytest.mark.gpu


def run_linear(ttt, inp, use_ln=False, flags=0, eta_none=False):
    r, w = inp.raw, inp.w
    Q, K, V = to_dev(r["Q"]), to_dev(r["K"]), to_dev(r["V"])
    eta = None if eta_none else to_dev(r["eta"])
    W0 = to_dev(r["W0"])
    kw = {}
    if use_ln:
        kw = dict(c0=to_dev(r["c0"]), gamma=to_dev(r["gamma"]), beta=to_dev(r["beta"]), eps=w.ln_eps)
    B, H, T, d = Q.shape
    Z = poison_like(Q)
    Wout = torch.full((B, H, d, d), float("nan"), device="cuda")
    cout = torch.full((B, H, d), float("nan"), device="cuda") if use_ln else None
    ttt.linear_forward(Q, K, V, eta, W0, w.b, eta_const=w.eta_const, use_ln=use_ln, Z=Z, W_out=Wout,
                       c_out=cout, flags=flags, **kw)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == ttt.TTT_OK
    return to_host(Z), to_host(Wout), (to_host(cout) if use_ln else None)


def oracle_linear(inp, use_ln=False):
    e, w = inp.exact, inp.w
    kw = dict(c0=e["c0"], gamma=e["gamma"], beta=e["beta"], eps=w.ln_eps) if use_ln else {}
    return O.linear_forward(e["Q"], e["K"], e["V"], e["eta"], e["W0"], w.b, use_ln=use_ln, **kw)


def check_linear(ttt, inp, use_ln=False, flags=0):
    Zg, Wg, cg = run_linear(ttt, inp, use_ln, flags)
    Zo, Wo, co = oracle_linear(inp, use_ln)
    ez = assert_close("Z", Zg, Zo, inp.w.io_dtype)
    ew = assert_close("W_out", Wg, Wo, inp.w.io_dtype)
    if use_ln:
        assert_close("c_out", cg, co, inp.w.io_dtype)
    return ez, ew


# ---------------------------------------------------------------------------
# TTT-Linear, tensor-core kernel (bf16, d = 64, b = 16)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,T", [(1, 1, 16), (1, 2, 48), (1, 3, 160), (2, 5, 64), (3, 3, 256)])
@pytest.mark.parametrize("use_ln", [False, True])
@pytest.mark.parametrize("layout", ["one", "two"])
def test_linear_tc_small(ttt_lib, B, H, T, use_ln, layout):
    """Both CTA layouts of the tensor-core kernel (one or two units per CTA)."""
    inp = WL.random_case("ln" if use_ln else "linear", B, H, T, 64, 16, seed=B * 100 + H * 10 + T)
    flags = ttt_lib.FLAG_ONE_UNIT_PER_CTA if layout == "one" else ttt_lib.FLAG_TWO_UNITS_PER_CTA
    ez, ew = check_linear(ttt_lib, inp, use_ln, flags)
    # the bf16-operand error is well below the tolerance at these sizes
    assert ez < 1e-2 and ew < 1e-2, (ez, ew)


@pytest.mark.parametrize("use_ln", [False, True])
def test_linear_tc_layouts_agree(ttt_lib, use_ln):
    """One and two units per CTA run the same products in the same order (the
    LN feature sums differ only in their summation order, which flips the
    bf16 rounding of a few Z elements: Z is compared at 2e-3, a fraction of
    one bf16 ulp (2^-8), the fp32 state at 1e-4)."""
    inp = WL.random_case("ln" if use_ln else "linear", 2, 3, 224, 64, 16, seed=29)
    Z1, W1, c1 = run_linear(ttt_lib, inp, use_ln, flags=ttt_lib.FLAG_ONE_UNIT_PER_CTA)
    Z2, W2, c2 = run_linear(ttt_lib, inp, use_ln, flags=ttt_lib.FLAG_TWO_UNITS_PER_CTA)
    if use_ln:
        assert normwise(Z1, Z2) < 2e-3 and normwise(W1, W2) < 1e-4 and normwise(c1, c2) < 1e-4
    else:
        assert np.array_equal(Z1, Z2) and np.array_equal(W1, W2)


@pytest.mark.parametrize("use_ln", [False, True])
def test_linear_tc_matches_simt(ttt_lib, use_ln):
    """The tensor-core and the fp32 CUDA-core kernels agree on the same inputs."""
    inp = WL.random_case("ln" if use_ln else "linear", 2, 3, 128, 64, 16, seed=5)
    Zt, Wt, _ = run_linear(ttt_lib, inp, use_ln)
    Zs, Ws, _ = run_linear(ttt_lib, inp, use_ln, flags=ttt_lib.FLAG_FORCE_SIMT)
    assert normwise(Zt, Zs) < 1e-2 and normwise(Wt, Ws) < 1e-2


def test_linear_tc_constant_eta_and_per_sequence_W0(ttt_lib):
    w = WL.Workload("c", "linear", 2, 2, 96, 64, 16, WL.BF16, "const", 0.02, 11)
    inp = WL.make_inputs(w, threads=1)
    # per-sequence initial state [B,H,d,d]
    rng = np.random.default_rng(3)
    W0 = rng.standard_normal((2, 2, 64, 64)) / 8.0
    raw, ex = WL.store(W0, WL.F32)
    inp.raw["W0"], inp.exact["W0"] = raw, ex
    Zg, Wg, _ = run_linear(ttt_lib, inp, eta_none=True)
    e = inp.exact
    Zo, Wo, _ = O.linear_forward(e["Q"], e["K"], e["V"], np.full((2, 2, 96), np.float32(0.02)), e["W0"], 16)
    assert_close("Z", Zg, Zo, WL.BF16)
    assert_close("W_out", Wg, Wo, WL.BF16)


def test_linear_tc_theorem1(ttt_lib):
    """W0 = 0, eta = 1, b = T = 16: causal linear attention (section 4.1)."""
    w = WL.Workload("t1", "linear", 1, 2, 16, 64, 16, WL.BF16, "const", 1.0, 13)
    inp = WL.make_inputs(w, threads=1)
    inp.raw["W0"] = np.zeros((2, 64, 64), np.float32)
    inp.exact["W0"] = np.zeros((2, 64, 64))
    Zg, _, _ = run_linear(ttt_lib, inp, eta_none=True)
    q, k, v = (inp.exact[n][0] for n in "QKV")
    ref = np.einsum("hts,hsd->htd", np.tril(np.einsum("htd,hsd->hts", q, k)), v)
    assert normwise(Zg[0], ref) < 1e-2


def test_linear_tc_eta_zero(ttt_lib):
    w = WL.Workload("z", "linear", 1, 3, 64, 64, 16, WL.BF16, "const", 0.0, 17)
    inp = WL.make_inputs(w, threads=1)
    Zg, Wg, _ = run_linear(ttt_lib, inp, eta_none=True)
    assert np.array_equal(Wg, np.broadcast_to(inp.exact["W0"][None], Wg.shape))
    Zo = np.einsum("bhtd,hde->bhte", inp.exact["Q"], inp.exact["W0"])
    assert normwise(Zg, Zo) < 1e-2


@pytest.mark.parametrize("use_ln", [False, True])
def test_linear_tc_chunked_calls(ttt_lib, use_ln):
    """forward(T1) then forward(T2) from its final state equals forward(T1+T2)."""
    inp = WL.random_case("ln" if use_ln else "linear", 1, 3, 96, 64, 16, seed=23)
    r = inp.raw
    dev = {k: to_dev(v) for k, v in r.items()}
    kw = dict(gamma=dev["gamma"], beta=dev["beta"]) if use_ln else {}
    Zf, Wf, cf = ttt_lib.linear_forward(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], 16, use_ln=use_ln,
                                        c0=dev.get("c0"), **kw)
    T1 = 48
    sl = lambda t, a, b: t[:, :, a:b].contiguous()
    Za, Wa, ca = ttt_lib.linear_forward(sl(dev["Q"], 0, T1), sl(dev["K"], 0, T1), sl(dev["V"], 0, T1),
                                        sl(dev["eta"], 0, T1), dev["W0"], 16, use_ln=use_ln, c0=dev.get("c0"),
                                        **kw)
    Zb, Wb, cb = ttt_lib.linear_forward(sl(dev["Q"], T1, 96), sl(dev["K"], T1, 96), sl(dev["V"], T1, 96),
                                        sl(dev["eta"], T1, 96), Wa, 16, use_ln=use_ln, c0=ca, **kw)
    torch.cuda.synchronize()
    # the resumed call starts its look-ahead from the bf16 copy of the stored
    # state, so the two routes agree to rounding, not bit for bit
    Zc = to_host(torch.cat([Za, Zb], 2))
    assert normwise(Zc, to_host(Zf)) < 5e-3
    assert normwise(to_host(Wb), to_host(Wf)) < 5e-3
    Zo, Wo, _ = oracle_linear(inp, use_ln)
    assert_close("Z (chunked)", Zc, Zo, WL.BF16)
    assert_close("W_out (chunked)", to_host(Wb), Wo, WL.BF16)


# ---------------------------------------------------------------------------
# TTT-Linear, fp32 CUDA-core kernel
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d,b,io,use_ln", [(64, 16, WL.BF16, False), (32, 4, WL.F32, False),
                                         (16, 1, WL.F32, False), (64, 8, WL.BF16, True)])
def test_state_only_forward(ttt_lib, d, b, io, use_ln):
    """Z = NULL (the state-only half of the mini-batch size study): W_out (and
    c_out) equal those of the same fp32 kernel with outputs, bit for bit, and
    the oracle's within the tolerance."""
    inp = WL.random_case("ln" if use_ln else "linear", 2, 3, 64, d, b, io_dtype=io, seed=d + b)
    r, w = inp.raw, inp.w
    Q, K, V, eta, W0 = (to_dev(r[n]) for n in ("Q", "K", "V", "eta", "W0"))
    kw = dict(c0=to_dev(r["c0"]), gamma=to_dev(r["gamma"]), beta=to_dev(r["beta"]), eps=w.ln_eps) if use_ln else {}
    _, Wa, ca = ttt_lib.linear_forward(Q, K, V, eta, W0, b, use_ln=use_ln, flags=ttt_lib.FLAG_FORCE_SIMT, **kw)
    Zb, Wb, cb = ttt_lib.linear_forward(Q, K, V, eta, W0, b, use_ln=use_ln, outputs=False, **kw)
    torch.cuda.synchronize()
    assert Zb is None
    assert torch.equal(Wa, Wb)
    if use_ln:
        assert torch.equal(ca, cb)
    _, Wo, co = oracle_linear(inp, use_ln)
    assert_close("W_out", to_host(Wb), Wo, io)


def test_linear_d16_f32_workload(ttt_lib):
    """The fp32 workload (d = 16, T = 256, eta = 0.1): max relative error <= 1e-4."""
    w = WL.WORKLOADS["linear_d16_T256_f32"]
    inp = WL.make_inputs(w, threads=1)
    Zg, Wg, _ = run_linear(ttt_lib, inp, eta_none=True)
    e = inp.exact
    Zo, Wo, _ = O.linear_forward(e["Q"], e["K"], e["V"], np.full(e["eta"].shape, np.float32(0.1)), e["W0"], 16)
    assert_close("Z", Zg, Zo, WL.F32)
    assert_close("W_out", Wg, Wo, WL.F32)


@pytest.mark.parametrize("d,b,T,io", [(16, 1, 37, WL.F32), (32, 8, 64, WL.F32), (64, 64, 128, WL.F32),
                                      (32, 16, 96, WL.BF16), (16, 4, 0, WL.F32)])
@pytest.mark.parametrize("use_ln", [False, True])
def test_linear_simt_shapes(ttt_lib, d, b, T, io, use_ln):
    if T % b:
        pytest.skip("T must be a multiple of b")
    inp = WL.random_case("ln" if use_ln else "linear", 2, 2, T, d, b, io_dtype=io, seed=d + b + T)
    check_linear(ttt_lib, inp, use_ln)


# ---------------------------------------------------------------------------
# TTT-MLP
# ---------------------------------------------------------------------------

def run_mlp(ttt, inp, flags=0):
    r, w = inp.raw, inp.w
    args = [to_dev(r[n]) for n in ("Q", "K", "V", "eta", "W1", "c1", "W2", "c2")]
    out = ttt.mlp_forward(*args, w.b, eta_const=w.eta_const, flags=flags)
    torch.cuda.synchronize()
    return [to_host(x) for x in out]


def check_mlp(ttt, inp, flags=0):
    got = run_mlp(ttt, inp, flags)
    e = inp.exact
    ref = O.mlp_forward(e["Q"], e["K"], e["V"], e["eta"], e["W1"], e["c1"], e["W2"], e["c2"], inp.w.b)
    errs = [assert_close(n, g, o, inp.w.io_dtype) for n, g, o in zip(("Z", "W1", "c1", "W2", "c2"), got, ref)]
    return errs


@pytest.mark.parametrize("d,b,T,io", [(16, 16, 64, WL.F32), (32, 8, 48, WL.F32), (16, 4, 32, WL.BF16)])
def test_mlp_simt_shapes(ttt_lib, d, b, T, io):
    inp = WL.random_case("mlp", 2, 2, T, d, b, io_dtype=io, eta_mode="const", eta_const=0.05, seed=d * b)
    check_mlp(ttt_lib, inp)


@pytest.mark.parametrize("B,H,T", [(1, 1, 16), (1, 2, 64), (2, 3, 128)])
def test_mlp_d64_bf16(ttt_lib, B, H, T):
    inp = WL.random_case("mlp", B, H, T, 64, 16, io_dtype=WL.BF16, eta_mode="const", eta_const=1 / 64,
                         seed=B + H + T)
    check_mlp(ttt_lib, inp)


@pytest.mark.parametrize("d,b,T,io", [(16, 16, 64, WL.F32), (32, 4, 48, WL.F32), (64, 16, 64, WL.BF16),
                                      (16, 1, 12, WL.F32)])
def test_mlp_ln_matches_oracle(ttt_lib, d, b, T, io):
    """TTT-MLP with LN+residual on the output layer (fp32 CUDA-core kernel)."""
    inp = WL.random_case("mlp", 2, 3, T, d, b, io_dtype=io, eta_mode="sigmoid", seed=d + b + T)
    rng = np.random.default_rng(d + 3 * b)
    gr, ge = WL.store(1 + rng.standard_normal((3, d)) * 0.14, WL.F32)
    br, be = WL.store(rng.standard_normal((3, d)) * 0.14, WL.F32)
    r, e = inp.raw, inp.exact
    dev = {k: to_dev(r[k]) for k in ("Q", "K", "V", "eta", "W1", "c1", "W2", "c2")}
    out = ttt_lib.mlp_forward(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W1"], dev["c1"], dev["W2"], dev["c2"],
                              b, Z=poison_like(dev["Q"]), use_ln=True, gamma=to_dev(gr), beta=to_dev(br))
    torch.cuda.synchronize()
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK
    ref = O.mlp_forward(e["Q"], e["K"], e["V"], e["eta"], e["W1"], e["c1"], e["W2"], e["c2"], b, use_ln=True,
                        gamma=ge, beta=be)
    for name, g, o in zip(("Z", "W1", "c1", "W2", "c2"), out, ref):
        assert_close(name, to_host(g), o, io)


@pytest.mark.parametrize("B,H,T,eta_mode", [(2, 4, 256, "sigmoid"), (1, 3, 48, "const"), (3, 1, 16, "sigmoid")])
def test_mlp_ln_tensor_core(ttt_lib, B, H, T, eta_mode):
    """bf16, d = 64, b = 16 with LN+residual runs on the tensor-core MLP kernel:
    against the oracle, and against the fp32 CUDA-core kernel on the same inputs."""
    d, b = 64, 16
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=WL.BF16, eta_mode=eta_mode, eta_const=1 / 64,
                         seed=5 * T + H)
    rng = np.random.default_rng(T + B)
    gr, ge = WL.store(1 + rng.standard_normal((H, d)) * 0.14, WL.F32)
    br, be = WL.store(rng.standard_normal((H, d)) * 0.14, WL.F32)
    r, e = inp.raw, inp.exact
    dev = {k: to_dev(r[k]) for k in ("Q", "K", "V", "eta", "W1", "c1", "W2", "c2")}
    args = (dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W1"], dev["c1"], dev["W2"], dev["c2"], b)
    tc = ttt_lib.mlp_forward(*args, Z=poison_like(dev["Q"]), use_ln=True, gamma=to_dev(gr), beta=to_dev(br))
    ft = ttt_lib.mlp_forward(*args, use_ln=True, gamma=to_dev(gr), beta=to_dev(br), flags=ttt_lib.FLAG_FORCE_SIMT)
    torch.cuda.synchronize()
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK
    ref = O.mlp_forward(e["Q"], e["K"], e["V"], e["eta"], e["W1"], e["c1"], e["W2"], e["c2"], b, use_ln=True,
                        gamma=ge, beta=be)
    for name, g, f, o in zip(("Z", "W1", "c1", "W2", "c2"), tc, ft, ref):
        assert_close(name, to_host(g), o, WL.BF16)
        assert normwise(to_host(g), to_host(f)) < 1e-2, name


def test_mlp_tc_matches_simt(ttt_lib):
    """The tensor-core and the fp32 CUDA-core MLP kernels agree on the same inputs."""
    inp = WL.random_case("mlp", 1, 3, 96, 64, 16, io_dtype=WL.BF16, eta_mode="const", eta_const=1 / 64, seed=41)
    a = run_mlp(ttt_lib, inp)
    b = run_mlp(ttt_lib, inp, flags=ttt_lib.FLAG_FORCE_SIMT)
    for x, y in zip(a, b):
        assert normwise(x, y) < 1e-2


def test_mlp_tc_sigmoid_eta_and_biases(ttt_lib):
    """Per-token eta and non-zero initial biases through the tensor-core MLP kernel."""
    inp = WL.random_case("mlp", 2, 2, 64, 64, 16, io_dtype=WL.BF16, eta_mode="sigmoid", seed=43)
    rng = np.random.default_rng(5)
    for nm, shape in (("c1", (2, 256)), ("c2", (2, 64))):
        raw, ex = WL.store(rng.standard_normal(shape) * 0.1, WL.F32)
        inp.raw[nm], inp.exact[nm] = raw, ex
    check_mlp(ttt_lib, inp)


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d,io", [(64, WL.BF16), (32, WL.F32), (16, WL.BF16)])
def test_decode_steps(ttt_lib, d, io):
    w = WL.Workload("dec", "linear", 3, 5, 1, d, 1, io, "sigmoid", 0.0, 31)
    rng = np.random.default_rng(d)
    W = rng.standard_normal((3, 5, d, d)) / np.sqrt(d)
    Wd = torch.tensor(W, dtype=torch.float32, device="cuda")
    Wo = Wd.double().cpu().numpy()
    for step in range(6):
        raw, ex = WL.make_decode_tokens(w, step)
        q, k, v, eta = (to_dev(raw[n]) for n in ("q", "k", "v", "eta"))
        z = ttt_lib.linear_decode_step(Wd, q, k, v, eta)
        Wo, zo = O.linear_decode_step(Wo, ex["q"], ex["k"], ex["v"], ex["eta"])
        torch.cuda.synchronize()
        if io == WL.F32:
            assert_close("z", to_host(z), zo, io)
        else:
            assert normwise(to_host(z), zo) < 1e-2
        assert normwise(to_host(Wd), Wo) < 1e-5


def _f32_state(rng, shape, scale, offset=0.0):
    """fp32 device tensor and the same values in float64 for the oracle."""
    raw, ex = WL.store(offset + rng.standard_normal(shape) * scale, WL.F32)
    return to_dev(raw), ex


@pytest.mark.parametrize("d,io", [(64, WL.BF16), (32, WL.F32), (16, WL.BF16), (64, WL.F32)])
def test_ln_decode_steps(ttt_lib, d, io):
    """LN+residual decode (b = 1 primal step) against the oracle's forward with
    T = b = 1 from the same state; W and c carried over six steps."""
    B, H = 3, 5
    w = WL.Workload("dec", "ln", B, H, 1, d, 1, io, "sigmoid", 0.0, 37)
    rng = np.random.default_rng(100 + d)
    Wd, Wo = _f32_state(rng, (B, H, d, d), 1 / np.sqrt(d))
    cd, co = _f32_state(rng, (B, H, d), 0.1)
    gd, go = _f32_state(rng, (H, d), np.sqrt(0.02), offset=1.0)
    bd, bo = _f32_state(rng, (H, d), np.sqrt(0.02))
    for step in range(6):
        raw, ex = WL.make_decode_tokens(w, step)
        q, k, v, eta = (to_dev(raw[n]) for n in ("q", "k", "v", "eta"))
        z = ttt_lib.linear_decode_step(Wd, q, k, v, eta, use_ln=True, c=cd, gamma=gd, beta=bd, eps=1e-6)
        Z, Wo, co = O.linear_forward(ex["q"][:, :, None], ex["k"][:, :, None], ex["v"][:, :, None],
                                     ex["eta"][:, :, None], Wo, 1, c0=co, gamma=go, beta=bo, use_ln=True, eps=1e-6)
        zo = Z[:, :, 0]
        torch.cuda.synchronize()
        if io == WL.F32:
            assert_close("z", to_host(z), zo, io)
        else:
            assert normwise(to_host(z), zo) < 1e-2
        assert normwise(to_host(Wd), Wo) < 1e-5
        assert normwise(to_host(cd), co) < 1e-5
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK


@pytest.mark.parametrize("d,io", [(64, WL.BF16), (64, WL.F32), (32, WL.F32), (16, WL.BF16)])
def test_mlp_decode_steps(ttt_lib, d, io):
    """TTT-MLP decode (b = 1 primal step) against the oracle's MLP forward with
    T = b = 1 from the same per-sequence state; the four state tensors carried
    over six steps."""
    B, H, m = 3, 5, 4 * d
    w = WL.Workload("dec", "mlp", B, H, 1, d, 1, io, "sigmoid", 0.0, 41)
    rng = np.random.default_rng(200 + d)
    W1d, W1o = _f32_state(rng, (B, H, d, m), 1 / np.sqrt(d))
    c1d, c1o = _f32_state(rng, (B, H, m), 0.1)
    W2d, W2o = _f32_state(rng, (B, H, m, d), 1 / np.sqrt(m))
    c2d, c2o = _f32_state(rng, (B, H, d), 0.1)
    for step in range(6):
        raw, ex = WL.make_decode_tokens(w, step)
        q, k, v, eta = (to_dev(raw[n]) for n in ("q", "k", "v", "eta"))
        z = ttt_lib.mlp_decode_step(W1d, c1d, W2d, c2d, q, k, v, eta)
        Z, W1o, c1o, W2o, c2o = O.mlp_forward(ex["q"][:, :, None], ex["k"][:, :, None], ex["v"][:, :, None],
                                              ex["eta"][:, :, None], W1o, c1o, W2o, c2o, 1)
        zo = Z[:, :, 0]
        torch.cuda.synchronize()
        if io == WL.F32:
            assert_close("z", to_host(z), zo, io)
        else:
            assert normwise(to_host(z), zo) < 1e-2
        for nm, g, o in (("W1", W1d, W1o), ("c1", c1d, c1o), ("W2", W2d, W2o), ("c2", c2d, c2o)):
            assert normwise(to_host(g), o) < 1e-5, nm
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK


def test_mlp_decode_eta_zero_is_a_forward(ttt_lib):
    """eta = 0: the state is returned bit for bit and z = f(q; state)."""
    B, H, d, m = 2, 3, 64, 256
    rng = np.random.default_rng(7)
    W1d, W1o = _f32_state(rng, (B, H, d, m), 1 / np.sqrt(d))
    c1d, c1o = _f32_state(rng, (B, H, m), 0.1)
    W2d, W2o = _f32_state(rng, (B, H, m, d), 1 / np.sqrt(m))
    c2d, c2o = _f32_state(rng, (B, H, d), 0.1)
    before = [t.clone() for t in (W1d, c1d, W2d, c2d)]
    qr, qe = WL.store(rng.standard_normal((B, H, d)) / 8, WL.F32)
    q = to_dev(qr)
    z = ttt_lib.mlp_decode_step(W1d, c1d, W2d, c2d, q, q, q, None, eta_const=0.0)
    torch.cuda.synchronize()
    for a, b in zip(before, (W1d, c1d, W2d, c2d)):
        assert torch.equal(a, b)
    zo = O.mlp_forward(qe[:, :, None], qe[:, :, None], qe[:, :, None], np.zeros((B, H, 1)), W1o, c1o, W2o, c2o,
                       1)[0][:, :, 0]
    assert_close("z", to_host(z), zo, WL.F32)


# ---------------------------------------------------------------------------
# full-size workloads, sampled units
# ---------------------------------------------------------------------------

def sampled_parity(ttt, w, units, flags=0):
    inp = WL.make_inputs(w, want_exact=False)
    r = inp.raw
    dev = {k: to_dev(v) for k, v in r.items()}
    B, H = w.B, w.H
    if w.kind == "mlp":
        out = ttt.mlp_forward(dev["Q"], dev["K"], dev["V"], None, dev["W1"], dev["c1"], dev["W2"], dev["c2"], w.b,
                              eta_const=w.eta_const, flags=flags)
    else:
        ln = w.kind == "ln"
        kw = dict(c0=dev["c0"], gamma=dev["gamma"], beta=dev["beta"], eps=w.ln_eps) if ln else {}
        out = ttt.linear_forward(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], w.b, use_ln=ln, flags=flags,
                                 **kw)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == ttt.TTT_OK
    del dev
    errs = []
    for u in units:
        n, h = divmod(u, H)
        one = WL.make_unit_inputs(w, u)
        e = one.exact
        if w.kind == "mlp":
            ref = O.mlp_forward(e["Q"], e["K"], e["V"], np.full(e["eta"].shape, w.eta_const), e["W1"], e["c1"],
                                e["W2"], e["c2"], w.b)
            names = ("Z", "W1", "c1", "W2", "c2")
        else:
            ln = w.kind == "ln"
            kw = dict(c0=e["c0"], gamma=e["gamma"], beta=e["beta"], eps=w.ln_eps) if ln else {}
            ref = O.linear_forward(e["Q"], e["K"], e["V"], e["eta"], e["W0"], w.b, use_ln=ln, **kw)
            names = ("Z", "W_out", "c_out")[: 3 if ln else 2]
        for nm, g, o in zip(names, out, ref):
            errs.append(assert_close(f"{nm}[unit {u}]", to_host(g[n, h]), o[0, 0], w.io_dtype))
    return max(errs)


@pytest.mark.slow
@pytest.mark.parametrize("name,units", [
    ("linear_B8_H12_T2048", [0, 1, 47, 95]),
    ("ln_B4_H32_T8192", [0, 77, 127]),
    ("mlp_B2_H32_T8192", [0, 63]),
    ("linear_B16_H32_T32768_decode1024", [0, 257, 511]),
])
def test_full_size_sampled(ttt_lib, name, units):
    sampled_parity(ttt_lib, WL.WORKLOADS[name], units)


@pytest.mark.slow
def test_long_decode_after_prefill(ttt_lib):
    """Decode phase of the long-context workload (all 16 x 32 units, 1024
    steps) starting from a prefill's final state; every step's z and the
    final state are compared with the oracle.  The prefill is shortened to
    T = 256 here so that the oracle stays cheap; the full-length prefill is
    covered by test_full_size_sampled."""
    w = WL.scaled(WL.WORKLOADS["linear_B16_H32_T32768_decode1024"], T=256)
    inp = WL.make_inputs(w)
    dev = {k: to_dev(v) for k, v in inp.raw.items()}
    _, Wd, _ = ttt_lib.linear_forward(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], 16)
    e = inp.exact
    _, Wo, _ = O.linear_forward(e["Q"], e["K"], e["V"], e["eta"], e["W0"], 16)
    Wo = to_host(Wd)   # continue the oracle from the GPU prefill state to isolate the decode error
    worst = 0.0
    for step in range(w.decode_steps):
        raw, ex = WL.make_decode_tokens(w, step)
        z = ttt_lib.linear_decode_step(Wd, *(to_dev(raw[n]) for n in ("q", "k", "v", "eta")))
        Wo, zo = O.linear_decode_step(Wo, ex["q"], ex["k"], ex["v"], ex["eta"])
        worst = max(worst, normwise(to_host(z), zo))
    torch.cuda.synchronize()
    assert worst < 2e-2
    assert normwise(to_host(Wd), Wo) < 2e-2
