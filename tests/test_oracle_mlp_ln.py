"""Pins of the oracle's TTT-MLP with LN+residual on the output layer,
f(x) = x + gamma LN(GELU(x W1 + c1) W2 + c2) + beta: the form the pages give
for TTT-MLP in practice (paper digest "论文速览 | TTT", section 4.4; the dual
form of section 3.7 with the LN backward in place of the residual E).

The same independent routes as the other models' pins: a matrix dual form
written from the pages, finite differences of the reconstruction loss for
the one-mini-batch state change, and the output rule.
"""
import numpy as np
import pytest
from scipy.special import erf

from oracle import oracle as O
from tests.test_oracle_pins import fd_grad, gelu, ln_rows, rel

RNG = np.random.default_rng(4321)


def f_mlp_ln(X, W1, c1, W2, c2, gamma, beta, eps=1e-6):
    return X + gamma * ln_rows(gelu(X @ W1 + c1) @ W2 + c2, eps) + beta


def make(B, H, T, d, m, eta_scale=0.3):
    Q, K, V = (RNG.standard_normal((B, H, T, d)) / np.sqrt(d) for _ in range(3))
    eta = np.abs(RNG.standard_normal((B, H, T))) * eta_scale
    W1 = RNG.standard_normal((H, d, m)) / np.sqrt(d)
    c1 = RNG.standard_normal((H, m)) * 0.1
    W2 = RNG.standard_normal((H, m, d)) / np.sqrt(m)
    c2 = RNG.standard_normal((H, d)) * 0.1
    gamma = 1 + RNG.standard_normal((H, d)) * 0.2
    beta = RNG.standard_normal((H, d)) * 0.2
    return Q, K, V, eta, W1, c1, W2, c2, gamma, beta


def dual_mlp_ln_unit(Q, K, V, eta, W1, c1, W2, c2, gamma, beta, b, eps=1e-6):
    """Per mini-batch at the batch-start weights: Y = GELU(K W1 + c1) W2 + c2,
    Delta2 = the LN+residual backward at Y, D1 = (Delta2 W2^T) * GELU'(A); the
    outputs through tril(Q K^T + 1) on layer 1 and tril(Hq Hk^T + 1) on layer 2
    and the output LN; the updates with Delta2 in place of E."""
    T, d = Q.shape
    W1, c1, W2, c2 = W1.copy(), c1.copy(), W2.copy(), c2.copy()
    Z = np.empty_like(Q)
    Phi = lambda x: 0.5 * (1 + erf(x / np.sqrt(2)))
    phi = lambda x: np.exp(-0.5 * x * x) / np.sqrt(2 * np.pi)
    for t0 in range(0, T, b):
        sl = slice(t0, min(t0 + b, T))
        Qb, Kb, Vb, eb = Q[sl], K[sl], V[sl], eta[sl]
        A = Kb @ W1 + c1
        Hk = gelu(A)
        Y = Hk @ W2 + c2
        mu = Y.mean(1, keepdims=True)
        r = 1.0 / np.sqrt(((Y - mu) ** 2).mean(1, keepdims=True) + eps)
        Xh = (Y - mu) * r
        G = gamma * (Kb + gamma * Xh + beta - Vb)
        D2 = r * (G - G.mean(1, keepdims=True) - Xh * (G * Xh).mean(1, keepdims=True))
        D1 = (D2 @ W2.T) * (Phi(A) + A * phi(A))
        S1 = np.tril(Qb @ Kb.T + 1.0)
        Aq = Qb @ W1 + c1 - (S1 * eb[None, :]) @ D1
        Hq = gelu(Aq)
        S2 = np.tril(Hq @ Hk.T + 1.0)
        Zpre = Hq @ W2 + c2 - (S2 * eb[None, :]) @ D2
        Z[sl] = Qb + gamma * ln_rows(Zpre, eps) + beta
        W1 = W1 - Kb.T @ (eb[:, None] * D1)
        c1 = c1 - eb @ D1
        W2 = W2 - Hk.T @ (eb[:, None] * D2)
        c2 = c2 - eb @ D2
    return Z, W1, c1, W2, c2


@pytest.mark.parametrize("d,b,T", [(2, 1, 3), (3, 2, 7), (4, 4, 8), (3, 16, 35), (4, 2, 10)])
def test_primal_equals_dual_mlp_ln(d, b, T):
    m = 4 * d
    Q, K, V, eta, W1, c1, W2, c2, gamma, beta = make(1, 2, T, d, m)
    out = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b, use_ln=True, gamma=gamma, beta=beta)
    for h in range(2):
        ref = dual_mlp_ln_unit(Q[0, h], K[0, h], V[0, h], eta[0, h], W1[h], c1[h], W2[h], c2[h], gamma[h],
                               beta[h], b)
        for got, want in zip(out, ref):
            assert rel(got[0, h], want) < 1e-10


def test_fd_gradient_mlp_ln():
    """One mini-batch (b = T): the state change equals eta-weighted gradient
    steps of 1/2 ||f(k_t) - v_t||^2 summed over the batch, each at the
    batch-start weights (section 3.5), checked by central differences."""
    d, m, T = 3, 12, 5
    Q, K, V, eta, W1, c1, W2, c2, gamma, beta = make(1, 1, T, d, m, eta_scale=0.5)
    _, W1o, c1o, W2o, c2o = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, T, use_ln=True, gamma=gamma, beta=beta)
    P = [W1[0].copy(), c1[0].copy(), W2[0].copy(), c2[0].copy()]
    k, v, e = K[0, 0], V[0, 0], eta[0, 0]

    def loss():
        R = f_mlp_ln(k, *P, gamma[0], beta[0]) - v
        return 0.5 * np.sum(e[:, None] * R * R)

    g = fd_grad(loss, P)
    assert rel(W1[0] - W1o[0, 0], g[0]) < 1e-7
    assert rel(c1[0] - c1o[0, 0], g[1]) < 1e-7
    assert rel(W2[0] - W2o[0, 0], g[2]) < 1e-7
    assert rel(c2[0] - c2o[0, 0], g[3]) < 1e-7


def test_output_uses_state_after_own_token_mlp_ln():
    """z_t = f(q_t; state after token t) (section 3.1): the state from the
    forward on the prefix ending at t."""
    d, m, T, b = 3, 12, 6, 4
    Q, K, V, eta, W1, c1, W2, c2, gamma, beta = make(1, 1, T, d, m)
    Z = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b, use_ln=True, gamma=gamma, beta=beta)[0]
    for t in range(T):
        s = slice(0, t + 1)
        _, W1t, c1t, W2t, c2t = O.mlp_forward(Q[:, :, s], K[:, :, s], V[:, :, s], eta[:, :, s], W1, c1, W2, c2, b,
                                              use_ln=True, gamma=gamma, beta=beta)
        want = f_mlp_ln(Q[0, 0, t], W1t[0, 0], c1t[0, 0], W2t[0, 0], c2t[0, 0], gamma[0], beta[0])
        assert rel(Z[0, 0, t], want) < 1e-12


def test_plain_mlp_unchanged_by_the_ln_option():
    Q, K, V, eta, W1, c1, W2, c2, gamma, beta = make(1, 2, 8, 3, 12)
    a = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, 4)
    b = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, 4, use_ln=False, gamma=gamma, beta=beta)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
