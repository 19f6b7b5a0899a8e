"""Pins of the oracle's outer-loop backward (TTT-Linear, no LN).

The backward is reverse-mode differentiation of the primal mini-batch loop
(paper digest "论文速览 | TTT", section 3.4: the outer loop's gradients pass
through the inner loop's updates of W; sections 3.5-3.6 define those
updates).  It is pinned against central finite differences of the forward
oracle, which is itself pinned elsewhere, and against the closed form at
eta = 0, where the layer reduces to Z = Q W0 and W_out = W0.
"""
import numpy as np
import pytest

from oracle import oracle as O


def _case(B, H, T, d, shared_w0, seed):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    K = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    V = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    eta = 0.2 + 0.3 * rng.random((B, H, T))
    W0 = rng.standard_normal((H, d, d) if shared_w0 else (B, H, d, d)) / np.sqrt(d)
    dZ = rng.standard_normal((B, H, T, d))
    dW = rng.standard_normal((B, H, d, d))
    return Q, K, V, eta, W0, dZ, dW


def _loss(Q, K, V, eta, W0, b, dZ, dW):
    Z, W_out, _ = O.linear_forward(Q, K, V, eta, W0, b, threads=1)
    return float(np.sum(Z * dZ) + np.sum(W_out * dW))


@pytest.mark.parametrize("B,H,T,d,b,shared", [
    (1, 2, 5, 3, 2, True),     # ragged last mini-batch
    (2, 1, 6, 2, 3, False),    # per-sequence W0
    (1, 1, 4, 3, 1, True),     # b = 1: the sequential delta rule
    (1, 1, 4, 2, 4, True),     # one mini-batch, b = T
])
def test_backward_matches_finite_differences(B, H, T, d, b, shared):
    Q, K, V, eta, W0, dZ, dW = _case(B, H, T, d, shared, seed=10 * T + d + b)
    dQ, dK, dV, deta, dW0 = O.linear_backward(Q, K, V, eta, W0, b, dZ=dZ, dW_out=dW, threads=1)
    if shared:
        dW0 = dW0.sum(axis=0)
    grads = {"Q": dQ, "K": dK, "V": dV, "eta": deta, "W0": dW0}
    inputs = {"Q": Q, "K": K, "V": V, "eta": eta, "W0": W0}
    h = 1e-6
    for name, x in inputs.items():
        g = grads[name]
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = _loss(*inputs.values(), b, dZ, dW)
            x[idx] = keep - h
            lm = _loss(*inputs.values(), b, dZ, dW)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - g)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-7, (name, err)


def test_backward_at_zero_eta_is_the_linear_map():
    """eta = 0: Z = Q W0 and W_out = W0, so dQ = dZ W0^T, dW0 = Q^T dZ + dW_out,
    dK = dV = 0; deta_t = -<D_t, k_t^T e_t> with e_t = k_t W0 - v_t and D_t the
    state gradient after token t (dW_out plus the outputs at t and later)."""
    B, H, T, d, b = 1, 1, 6, 4, 3
    Q, K, V, eta, W0, dZ, dW = _case(B, H, T, d, True, seed=3)
    eta = np.zeros_like(eta)
    dQ, dK, dV, deta, dW0 = O.linear_backward(Q, K, V, eta, W0, b, dZ=dZ, dW_out=dW, threads=1)
    W = W0[0]
    q, k, v, dz = Q[0, 0], K[0, 0], V[0, 0], dZ[0, 0]
    np.testing.assert_allclose(dQ[0, 0], dz @ W.T, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dW0[0, 0], q.T @ dz + dW[0, 0], rtol=0, atol=1e-13)
    assert np.all(dK == 0) and np.all(dV == 0)
    e = k @ W - v
    for t in range(T):
        D = dW[0, 0] + q[t:].T @ dz[t:]
        assert abs(deta[0, 0, t] + k[t] @ D @ e[t]) < 1e-12


def test_backward_without_upstream_gradients_is_zero():
    Q, K, V, eta, W0, _, _ = _case(1, 2, 4, 3, True, seed=5)
    out = O.linear_backward(Q, K, V, eta, W0, 2, threads=1)
    for g in out:
        assert np.all(g == 0)


# ---------------------------------------------------------------------------
# LN+residual: f(x) = x + gamma LN(x W + c) + beta (section 4.4); the outer
# loop also trains the LN parameters and the initial bias
# ---------------------------------------------------------------------------

def _ln_case(B, H, T, d, shared, seed):
    Q, K, V, eta, W0, dZ, dW = _case(B, H, T, d, shared, seed)
    rng = np.random.default_rng(seed + 1)
    c0 = rng.standard_normal((H, d) if shared else (B, H, d)) * 0.2
    gamma = 1 + rng.standard_normal((H, d)) * 0.3
    beta = rng.standard_normal((H, d)) * 0.3
    dc = rng.standard_normal((B, H, d))
    return Q, K, V, eta, W0, c0, gamma, beta, dZ, dW, dc


def _ln_loss(Q, K, V, eta, W0, c0, gamma, beta, b, dZ, dW, dc):
    Z, W_out, c_out = O.linear_forward(Q, K, V, eta, W0, b, c0=c0, gamma=gamma, beta=beta, use_ln=True, threads=1)
    return float(np.sum(Z * dZ) + np.sum(W_out * dW) + np.sum(c_out * dc))


@pytest.mark.parametrize("B,H,T,d,b,shared", [
    (1, 2, 5, 3, 2, True),     # ragged last mini-batch
    (2, 1, 6, 3, 3, False),    # per-sequence W0 and c0
    (1, 1, 4, 3, 1, True),     # b = 1
    (1, 1, 4, 4, 4, True),     # one mini-batch
])
def test_ln_backward_matches_finite_differences(B, H, T, d, b, shared):
    Q, K, V, eta, W0, c0, gamma, beta, dZ, dW, dc = _ln_case(B, H, T, d, shared, seed=100 + 10 * T + d + b)
    g = O.linear_ln_backward(Q, K, V, eta, W0, b, c0, gamma, beta, dZ=dZ, dW_out=dW, dc_out=dc, threads=1)
    dQ, dK, dV, deta, dW0, dc0, dgamma, dbeta = g
    if shared:
        dW0, dc0 = dW0.sum(axis=0), dc0.sum(axis=0)
    grads = {"Q": dQ, "K": dK, "V": dV, "eta": deta, "W0": dW0, "c0": dc0, "gamma": dgamma.sum(axis=0),
             "beta": dbeta.sum(axis=0)}
    inputs = {"Q": Q, "K": K, "V": V, "eta": eta, "W0": W0, "c0": c0, "gamma": gamma, "beta": beta}
    # the LN makes the loss strongly curved in some directions (the central difference's error
    # falls as h^2 there), so a smaller step than for the linear model
    h = 1e-7
    for name, x in inputs.items():
        gr = grads[name]
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = _ln_loss(*inputs.values(), b, dZ, dW, dc)
            x[idx] = keep - h
            lm = _ln_loss(*inputs.values(), b, dZ, dW, dc)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - gr)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-6, (name, err)


# ---------------------------------------------------------------------------
# TTT-MLP, f(x) = GELU(x W1 + c1) W2 + c2 (section 4.4): the outer loop also
# trains the initial parameters of both layers
# ---------------------------------------------------------------------------

def _mlp_case(B, H, T, d, m, shared, seed):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.standard_normal((B, H, T, d)) / np.sqrt(d) for _ in range(3))
    eta = 0.2 + 0.3 * rng.random((B, H, T))
    pre = (H,) if shared else (B, H)
    W1 = rng.standard_normal(pre + (d, m)) / np.sqrt(d)
    c1 = rng.standard_normal(pre + (m,)) * 0.2
    W2 = rng.standard_normal(pre + (m, d)) / np.sqrt(m)
    c2 = rng.standard_normal(pre + (d,)) * 0.2
    up = [rng.standard_normal((B, H, T, d)), rng.standard_normal((B, H, d, m)), rng.standard_normal((B, H, m)),
          rng.standard_normal((B, H, m, d)), rng.standard_normal((B, H, d))]
    return Q, K, V, eta, W1, c1, W2, c2, up


def _mlp_loss(Q, K, V, eta, W1, c1, W2, c2, b, up):
    out = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b, threads=1)
    return float(sum(np.sum(o * u) for o, u in zip(out, up)))


@pytest.mark.parametrize("B,H,T,d,m,b,shared", [
    (1, 2, 5, 2, 6, 2, True),     # ragged last mini-batch
    (2, 1, 4, 3, 5, 2, False),    # per-sequence parameters
    (1, 1, 4, 2, 4, 1, True),     # b = 1
    (1, 1, 3, 3, 4, 3, True),     # one mini-batch
])
def test_mlp_backward_matches_finite_differences(B, H, T, d, m, b, shared):
    Q, K, V, eta, W1, c1, W2, c2, up = _mlp_case(B, H, T, d, m, shared, seed=200 + 10 * T + d + m + b)
    g = O.mlp_backward(Q, K, V, eta, W1, c1, W2, c2, b, *up, threads=1)
    dQ, dK, dV, deta, dW1, dc1, dW2, dc2 = g
    if shared:
        dW1, dc1, dW2, dc2 = (x.sum(axis=0) for x in (dW1, dc1, dW2, dc2))
    grads = {"Q": dQ, "K": dK, "V": dV, "eta": deta, "W1": dW1, "c1": dc1, "W2": dW2, "c2": dc2}
    inputs = {"Q": Q, "K": K, "V": V, "eta": eta, "W1": W1, "c1": c1, "W2": W2, "c2": c2}
    h = 1e-6
    for name, x in inputs.items():
        gr = grads[name]
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = _mlp_loss(*inputs.values(), b, up)
            x[idx] = keep - h
            lm = _mlp_loss(*inputs.values(), b, up)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - gr)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-6, (name, err)


def test_gelu_second_derivative():
    """GELU'' used by the MLP backward, against central differences of GELU'."""
    from scipy.special import erf
    x = np.linspace(-4, 4, 81)
    g1 = lambda t: 0.5 * (1 + erf(t / np.sqrt(2))) + t * np.exp(-0.5 * t * t) / np.sqrt(2 * np.pi)
    h = 1e-5
    fd = (g1(x + h) - g1(x - h)) / (2 * h)
    g2 = np.exp(-0.5 * x * x) / np.sqrt(2 * np.pi) * (2 - x * x)
    assert np.max(np.abs(fd - g2)) < 1e-8


# ---------------------------------------------------------------------------
# TTT-MLP with LN+residual on the output layer, f(x) = x + gamma LN(GELU(x W1 +
# c1) W2 + c2) + beta (section 4.4): the outer loop also trains gamma and beta
# ---------------------------------------------------------------------------

def _mlp_ln_loss(Q, K, V, eta, W1, c1, W2, c2, gamma, beta, b, up):
    out = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b, threads=1, use_ln=True, gamma=gamma, beta=beta)
    return float(sum(np.sum(o * u) for o, u in zip(out, up)))


@pytest.mark.parametrize("B,H,T,d,m,b,shared", [
    (1, 2, 5, 3, 6, 2, True),     # ragged last mini-batch
    (2, 1, 4, 3, 5, 2, False),    # per-sequence parameters
    (1, 1, 4, 3, 4, 1, True),     # b = 1
    (1, 1, 3, 4, 4, 3, True),     # one mini-batch
])
def test_mlp_ln_backward_matches_finite_differences(B, H, T, d, m, b, shared):
    Q, K, V, eta, W1, c1, W2, c2, up = _mlp_case(B, H, T, d, m, shared, seed=300 + 10 * T + d + m + b)
    rng = np.random.default_rng(T + d)
    gamma = 1 + rng.standard_normal((H, d)) * 0.3
    beta = rng.standard_normal((H, d)) * 0.3
    g = O.mlp_ln_backward(Q, K, V, eta, W1, c1, W2, c2, b, gamma, beta, dZ=up[0], dW1_out=up[1], dc1_out=up[2],
                          dW2_out=up[3], dc2_out=up[4], threads=1)
    dQ, dK, dV, deta, dW1, dc1, dW2, dc2, dgamma, dbeta = g
    if shared:
        dW1, dc1, dW2, dc2 = (x.sum(axis=0) for x in (dW1, dc1, dW2, dc2))
    grads = {"Q": dQ, "K": dK, "V": dV, "eta": deta, "W1": dW1, "c1": dc1, "W2": dW2, "c2": dc2,
             "gamma": dgamma.sum(axis=0), "beta": dbeta.sum(axis=0)}
    inputs = {"Q": Q, "K": K, "V": V, "eta": eta, "W1": W1, "c1": c1, "W2": W2, "c2": c2, "gamma": gamma,
              "beta": beta}
    h = 1e-7   # the LN's curvature, as for the linear model with LN
    for name, x in inputs.items():
        gr = grads[name]
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = _mlp_ln_loss(*inputs.values(), b, up)
            x[idx] = keep - h
            lm = _mlp_ln_loss(*inputs.values(), b, up)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - gr)) / max(np.max(np.abs(fd)), 1e-12)
        assert err < 1e-6, (name, err)


def test_mlp_ln_backward_at_zero_eta():
    """eta = 0: the state never moves, so dZ reaches only the outputs of the initial state and the
    final-state gradients pass straight through to the initial state (plus the outputs' terms)."""
    Q, K, V, eta, W1, c1, W2, c2, up = _mlp_case(1, 1, 4, 3, 5, True, seed=7)
    eta[:] = 0.0
    rng = np.random.default_rng(8)
    gamma = 1 + rng.standard_normal((1, 3)) * 0.3
    beta = rng.standard_normal((1, 3)) * 0.3
    g = O.mlp_ln_backward(Q, K, V, eta, W1, c1, W2, c2, 2, gamma, beta, dZ=None, dW1_out=up[1], dc1_out=up[2],
                          dW2_out=up[3], dc2_out=up[4], threads=1)
    for got, u in zip(g[4:8], up[1:]):
        assert np.array_equal(got, u)
    for x in (g[0], g[1], g[2]):
        assert not np.any(x)
