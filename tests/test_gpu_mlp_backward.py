"""Parity of the TTT-MLP training path through the C ABI with the float64
oracle: the forward writing the batch-start states (W_states) and the
outer-loop backward reading them (ttt_mlp_backward), against the oracle's
forward on prefixes and its reverse-mode differentiation of the primal loop
(paper digest "论文速览 | TTT", sections 3.4, 3.7, 6.12).

Tolerances are the forward's: max relative error <= 1e-4 per tensor for fp32
inputs; normwise <= 2e-2 per tensor for bf16 inputs.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from test_sequence_layers_head_b200 import workloads as WL
from tests.gpu_util import maxrel, normwise, to_dev, to_host

pytestmark = [pytest.mark.gpu,
              pytest.mark.skip(reason="TTT-MLP backward kernel: first supervised B200 run pending")]


def _run(ttt, inp, c1, c2, dz, ups, per_token):
    r, w = inp.raw, inp.w
    Q, K, V = to_dev(r["Q"]), to_dev(r["K"]), to_dev(r["V"])
    eta = to_dev(r["eta"]) if per_token else None
    W1, W2 = to_dev(r["W1"]), to_dev(r["W2"])
    c1d, c2d = to_dev(c1), to_dev(c2)
    B, H, T, d = Q.shape
    m = 4 * d
    states = torch.full((B, H, T // w.b, 2 * d * m + m + d), float("nan"), device="cuda")
    ttt.mlp_forward(Q, K, V, eta, W1, c1d, W2, c2d, w.b, eta_const=w.eta_const, W_states=states)
    nan = lambda t: torch.full_like(t, float("nan"))
    out = ttt.mlp_backward(Q, K, V, eta, states, w.b, dZ=None if dz[0] is None else to_dev(dz[0]),
                           **{k: (None if u is None else to_dev(u))
                              for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)},
                           eta_const=w.eta_const, dQ=nan(Q), dK=nan(K), dV=nan(V), want_deta=per_token)
    torch.cuda.synchronize()
    assert ttt.last_device_status() == ttt.TTT_OK
    return to_host(states), [None if g is None else to_host(g) for g in out]


def _case(B, H, T, d, b, io, per_token, upstream, with_dz=True, seed=0):
    m = 4 * d
    inp = WL.random_case("mlp", B, H, T, d, b, io_dtype=io, eta_mode="sigmoid" if per_token else "const",
                         eta_const=0.0 if per_token else 0.02, seed=41 + seed)
    rng = np.random.default_rng(100 + seed)
    c1 = (rng.standard_normal((H, m)) * 0.1).astype(np.float32)
    c2 = (rng.standard_normal((H, d)) * 0.1).astype(np.float32)
    dz = WL.store(rng.standard_normal((B, H, T, d)), io) if with_dz else (None, None)
    ups = ([rng.standard_normal(s).astype(np.float32) for s in ((B, H, d, m), (B, H, m), (B, H, m, d), (B, H, d))]
           if upstream else [None] * 4)
    return inp, c1, c2, dz, ups


def _check(inp, c1, c2, dz, ups, per_token, states, grads):
    e, w = inp.exact, inp.w
    f64 = lambda a: a.astype(np.float64)
    B, H, T, d = e["Q"].shape
    eta = e["eta"] if per_token else np.full((B, H, T), np.float64(np.float32(w.eta_const)))
    params = (e["W1"], f64(c1), e["W2"], f64(c2))
    ref = O.mlp_backward(e["Q"], e["K"], e["V"], eta, *params, w.b, dZ=dz[1],
                         **{k: (None if u is None else f64(u))
                            for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    m = 4 * d
    nb = T // w.b
    for i in sorted({0, nb // 2, nb - 1} if nb else set()):
        t = i * w.b
        st = O.mlp_forward(e["Q"][:, :, :t], e["K"][:, :, :t], e["V"][:, :, :t], eta[:, :, :t], *params, w.b)[1:]
        parts = np.split(states[:, :, i], [d * m, d * m + m, 2 * d * m + m], axis=-1)
        for g, r in zip(parts, st):
            if w.io_dtype == WL.BF16:
                assert normwise(g.reshape(r.shape), r) <= 2e-2
            else:
                assert maxrel(g.reshape(r.shape), r) <= 1e-4
    for nm, got, want in zip(["dQ", "dK", "dV", "deta", "dW1", "dc1", "dW2", "dc2"], grads, ref):
        if got is None:
            continue
        if w.io_dtype == WL.BF16:
            # bf16 workloads: the normwise bar on every output (bf16 d = 64, b = 16 runs on mma.sync with
            # bf16 operands)
            assert normwise(got, want) <= 2e-2, (nm, normwise(got, want))
        else:
            assert maxrel(got, want) <= 1e-4, (nm, maxrel(got, want))


@pytest.mark.parametrize("B,H,T,d,b,io,per_token,upstream", [
    (1, 2, 64, 16, 16, WL.F32, True, True),
    (2, 1, 48, 16, 4, WL.F32, False, False),
    (1, 2, 32, 32, 8, WL.F32, True, True),
    (1, 1, 16, 16, 1, WL.F32, True, True),
    (2, 2, 64, 64, 16, WL.F32, True, True),
    (2, 3, 128, 64, 16, WL.BF16, True, True),
])
def test_mlp_backward_matches_oracle(ttt_lib, B, H, T, d, b, io, per_token, upstream):
    inp, c1, c2, dz, ups = _case(B, H, T, d, b, io, per_token, upstream, seed=T + d + b)
    states, grads = _run(ttt_lib, inp, c1, c2, dz, ups, per_token)
    _check(inp, c1, c2, dz, ups, per_token, states, grads)


def test_mlp_backward_state_gradients_only(ttt_lib):
    """No dZ: only the final-state gradients flow back."""
    inp, c1, c2, dz, ups = _case(1, 2, 48, 16, 16, WL.F32, True, True, with_dz=False, seed=3)
    states, grads = _run(ttt_lib, inp, c1, c2, dz, ups, True)
    _check(inp, c1, c2, dz, ups, True, states, grads)


def test_mlp_backward_empty_sequence(ttt_lib):
    """T = 0: the gradients of the initial state are the upstream ones."""
    from test_sequence_layers_head_b200 import ttt
    d, m = 16, 64
    rng = np.random.default_rng(9)
    ups = [rng.standard_normal(s).astype(np.float32) for s in ((1, 2, d, m), (1, 2, m), (1, 2, m, d), (1, 2, d))]
    Q = torch.empty((1, 2, 0, d), device="cuda")
    out = ttt.mlp_backward(Q, Q, Q, None, None, 16, eta_const=0.1, want_deta=False,
                           **{k: to_dev(u) for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    torch.cuda.synchronize()
    for g, u in zip(out[4:], ups):
        assert np.array_equal(to_host(g), u.astype(np.float64))


def test_mlp_backward_full_size_sampled(ttt_lib):
    """The TTT-MLP workload at full size (B=2, H=32, T=8192): the whole batch on
    the GPU; the first and last units against the oracle on that unit alone."""
    w = WL.WORKLOADS["mlp_B2_H32_T8192"]
    inp = WL.make_inputs(w, want_exact=False)
    r = inp.raw
    Q, K, V = to_dev(r["Q"]), to_dev(r["K"]), to_dev(r["V"])
    B, H, T, d = w.B, w.H, w.T, w.d
    m = 4 * d
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    dZ = torch.randn(B, H, T, d, generator=g, device="cuda").to(torch.bfloat16)
    states = torch.empty((B, H, T // w.b, 2 * d * m + m + d), device="cuda")
    ttt_lib.mlp_forward(Q, K, V, None, to_dev(r["W1"]), to_dev(r["c1"]), to_dev(r["W2"]), to_dev(r["c2"]), w.b,
                        eta_const=w.eta_const, W_states=states)
    out = ttt_lib.mlp_backward(Q, K, V, None, states, w.b, dZ=dZ, eta_const=w.eta_const, want_deta=False)
    torch.cuda.synchronize()
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK
    for t in out:
        if t is not None:
            assert bool(torch.isfinite(t).all())
    dz_host = to_host(dZ)
    for unit in (0, w.units - 1):
        n, h = divmod(unit, H)
        ui = WL.make_unit_inputs(w, unit)
        e = ui.exact
        eta = np.full((1, 1, T), np.float64(np.float32(w.eta_const)))
        ref = O.mlp_backward(e["Q"], e["K"], e["V"], eta, e["W1"], e["c1"], e["W2"], e["c2"], w.b,
                             dZ=dz_host[n:n + 1, h:h + 1])
        for nm, k in (("dQ", 0), ("dK", 1), ("dV", 2)):
            assert normwise(out[k][n:n + 1, h:h + 1].float().cpu().numpy().astype(np.float64), ref[k]) <= 2e-2, nm
        for nm, k in (("dW1", 4), ("dc1", 5), ("dW2", 6), ("dc2", 7)):
            got = out[k][n:n + 1, h:h + 1].cpu().numpy().astype(np.float64)
            assert normwise(got, ref[k]) <= 2e-2, nm


def test_mlp_backward_tensor_cores_match_cuda_cores(ttt_lib):
    """bf16, d = 64, b = 16 runs on mma.sync; TTT_FLAG_FORCE_SIMT runs the same
    call on the fp32 CUDA-core kernel: both against the oracle, and each other."""
    inp, c1, c2, dz, ups = _case(2, 2, 64, 64, 16, WL.BF16, True, True, seed=17)
    r, w = inp.raw, inp.w
    Q, K, V, eta = (to_dev(r[n]) for n in ("Q", "K", "V", "eta"))
    B, H, T, d = Q.shape
    m = 4 * d
    states = torch.empty((B, H, T // 16, 2 * d * m + m + d), device="cuda")
    ttt_lib.mlp_forward(Q, K, V, eta, to_dev(r["W1"]), to_dev(c1), to_dev(r["W2"]), to_dev(c2), 16, W_states=states)
    kw = dict(dZ=to_dev(dz[0]), **{k: to_dev(u) for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    tc = ttt_lib.mlp_backward(Q, K, V, eta, states, 16, **kw)
    simt = ttt_lib.mlp_backward(Q, K, V, eta, states, 16, flags=ttt_lib.FLAG_FORCE_SIMT, **kw)
    torch.cuda.synchronize()
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK
    for a, b_ in zip(tc, simt):
        assert normwise(to_host(a), to_host(b_)) <= 2e-2
    _check(inp, c1, c2, dz, ups, True, to_host(states), [to_host(g) for g in tc])


@pytest.mark.parametrize("B,H,T,d,b,io", [(1, 2, 64, 16, 16, WL.F32), (2, 2, 64, 64, 16, WL.BF16),
                                          (1, 1, 32, 32, 4, WL.F32)])
def test_mlp_ln_training_matches_oracle(ttt_lib, B, H, T, d, b, io):
    """TTT-MLP with LN+residual on the output layer: the forward writes its states (fp32 CUDA cores),
    the backward returns the eight gradients plus dgamma, dbeta; all against the oracle's reverse mode."""
    m = 4 * d
    inp, c1, c2, dz, ups = _case(B, H, T, d, b, io, True, True, seed=50 + T + d)
    r, e, w = inp.raw, inp.exact, inp.w
    rng = np.random.default_rng(T + d)
    gam = (1 + rng.standard_normal((H, d)) * 0.2).astype(np.float32)
    bet = (rng.standard_normal((H, d)) * 0.2).astype(np.float32)
    Q, K, V, eta = (to_dev(r[n]) for n in ("Q", "K", "V", "eta"))
    states = torch.full((B, H, T // b, 2 * d * m + m + d), float("nan"), device="cuda")
    ttt_lib.mlp_forward(Q, K, V, eta, to_dev(r["W1"]), to_dev(c1), to_dev(r["W2"]), to_dev(c2), b, use_ln=True,
                        gamma=to_dev(gam), beta=to_dev(bet), W_states=states)
    out = ttt_lib.mlp_backward(Q, K, V, eta, states, b, dZ=to_dev(dz[0]), use_ln=True, gamma=to_dev(gam),
                               beta=to_dev(bet), **{k: to_dev(u) for k, u in
                                                    zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    torch.cuda.synchronize()
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK
    f64 = lambda a: a.astype(np.float64)
    ref = O.mlp_ln_backward(e["Q"], e["K"], e["V"], e["eta"], e["W1"], f64(c1), e["W2"], f64(c2), b, f64(gam),
                            f64(bet), dZ=dz[1], **{k: f64(u) for k, u in
                                                   zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    for nm, got, want in zip(("dQ", "dK", "dV", "deta", "dW1", "dc1", "dW2", "dc2", "dgamma", "dbeta"), out, ref):
        g = to_host(got)
        if io == WL.BF16:
            assert normwise(g, want) <= 2e-2, nm
        else:
            assert maxrel(g, want) <= 1e-4, (nm, maxrel(g, want))


def test_mlp_ln_backward_tensor_cores_match_cuda_cores(ttt_lib):
    """With LN+residual, bf16 d = 64 b = 16 runs the backward on mma.sync and TTT_FLAG_FORCE_SIMT on fp32
    CUDA cores: the two agree within the bf16 bar on every gradient, dgamma and dbeta included."""
    d, b, m = 64, 16, 256
    inp, c1, c2, dz, ups = _case(2, 2, 64, d, b, WL.BF16, True, True, seed=71)
    r = inp.raw
    rng = np.random.default_rng(72)
    gam = to_dev((1 + rng.standard_normal((2, d)) * 0.2).astype(np.float32))
    bet = to_dev((rng.standard_normal((2, d)) * 0.2).astype(np.float32))
    Q, K, V, eta = (to_dev(r[n]) for n in ("Q", "K", "V", "eta"))
    states = torch.empty((2, 2, 64 // b, 2 * d * m + m + d), device="cuda")
    ttt_lib.mlp_forward(Q, K, V, eta, to_dev(r["W1"]), to_dev(c1), to_dev(r["W2"]), to_dev(c2), b, use_ln=True,
                        gamma=gam, beta=bet, W_states=states)
    kw = dict(dZ=to_dev(dz[0]), use_ln=True, gamma=gam, beta=bet,
              **{k: to_dev(u) for k, u in zip(("dW1_out", "dc1_out", "dW2_out", "dc2_out"), ups)})
    tc = ttt_lib.mlp_backward(Q, K, V, eta, states, b, **kw)
    simt = ttt_lib.mlp_backward(Q, K, V, eta, states, b, flags=ttt_lib.FLAG_FORCE_SIMT, **kw)
    torch.cuda.synchronize()
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK
    for a, b_ in zip(tc, simt):
        assert normwise(to_host(a), to_host(b_)) <= 2e-2
