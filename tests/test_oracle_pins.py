"""Pins of the float64 oracle against what the paper and the mathematics fix.

Paper: "Learning to (Learn at Test Time): RNNs with Expressive Hidden States"
(paper digest "论文速览 | TTT", equinox-blog).  Each test names the passage it
follows.  None of them re-types the oracle's own loop: they use independent
routes to the same numbers (the dual form, the sequential delta rule, finite
differences of the loss, linear attention, closed forms and invariants), so
that a dropped term, a wrong sign or index, a transposed operand or an
off-by-one in the causal mask inside the oracle fails at least one of them.
"""
import numpy as np
import pytest
from scipy.special import erf

from oracle import oracle as O

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------------------
# textbook forward definitions (no gradient code): f(x) for the three models
# ---------------------------------------------------------------------------

def gelu(x):
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def ln_rows(Y, eps):
    mu = Y.mean(-1, keepdims=True)
    var = ((Y - mu) ** 2).mean(-1, keepdims=True)
    return (Y - mu) / np.sqrt(var + eps)


def f_linear(X, W, c=None, use_ln=False, gamma=None, beta=None, eps=1e-6):
    Y = X @ W
    if not use_ln:
        return Y
    return X + gamma * ln_rows(Y + c, eps) + beta


def f_mlp(X, W1, c1, W2, c2):
    return gelu(X @ W1 + c1) @ W2 + c2


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


def make_linear(B, H, T, d, use_ln=False, eta_scale=0.3):
    Q, K, V = (rand(B, H, T, d, scale=1 / np.sqrt(d)) for _ in range(3))
    eta = np.abs(rand(B, H, T)) * eta_scale
    W0 = rand(H, d, d, scale=1 / np.sqrt(d))
    extra = {}
    if use_ln:
        extra = dict(c0=rand(H, d, scale=0.1), gamma=1 + rand(H, d, scale=0.2), beta=rand(H, d, scale=0.2))
    return Q, K, V, eta, W0, extra


def make_mlp(B, H, T, d, m, eta_scale=0.3):
    Q, K, V = (rand(B, H, T, d, scale=1 / np.sqrt(d)) for _ in range(3))
    eta = np.abs(rand(B, H, T)) * eta_scale
    W1 = rand(H, d, m, scale=1 / np.sqrt(d))
    c1 = rand(H, m, scale=0.1)
    W2 = rand(H, m, d, scale=1 / np.sqrt(m))
    c2 = rand(H, d, scale=0.1)
    return Q, K, V, eta, W1, c1, W2, c2


# ---------------------------------------------------------------------------
# P1: dual form (sections 3.6 and 3.7) written in matrix form
# ---------------------------------------------------------------------------

def dual_linear_unit(Q, K, V, eta, W, b, c=None, use_ln=False, gamma=None, beta=None, eps=1e-6):
    """Dual form per mini-batch, half-loss convention (eta_here = 2 eta_pages).

    linear:  E = K W - V,  Z = Q W - (tril(Q K^T) * eta_s) E,  W <- W - K^T diag(eta) E
    LN:      Delta from one batch forward/backward through LN at the batch-start
             state; the bias enters the causal matrix as tril(Q K^T + 1).
    """
    T, d = Q.shape
    W = W.copy()
    c = np.zeros(d) if c is None else c.copy()
    Z = np.empty_like(Q)
    for t0 in range(0, T, b):
        sl = slice(t0, min(t0 + b, T))
        Qb, Kb, Vb, eb = Q[sl], K[sl], V[sl], eta[sl]
        if not use_ln:
            E = Kb @ W - Vb
            S = np.tril(Qb @ Kb.T)
            Z[sl] = Qb @ W - (S * eb[None, :]) @ E
            W = W - Kb.T @ (eb[:, None] * E)
        else:
            Y = Kb @ W + c
            mu = Y.mean(1, keepdims=True)
            r = 1.0 / np.sqrt(((Y - mu) ** 2).mean(1, keepdims=True) + eps)
            Xh = (Y - mu) * r
            G = gamma * (Kb + gamma * Xh + beta - Vb)
            Delta = r * (G - G.mean(1, keepdims=True) - Xh * (G * Xh).mean(1, keepdims=True))
            S = np.tril(Qb @ Kb.T + 1.0)
            Yq = Qb @ W + c - (S * eb[None, :]) @ Delta
            Z[sl] = Qb + gamma * ln_rows(Yq, eps) + beta
            W = W - Kb.T @ (eb[:, None] * Delta)
            c = c - eb @ Delta
    return Z, W, c


def dual_mlp_unit(Q, K, V, eta, W1, c1, W2, c2, b):
    """Dual form for the two-layer MLP (section 3.7): one batch forward/backward
    at the batch-start weights, then the output pass with causal masks
    tril(Q K^T + 1) for layer 1 and tril(H_q H_k^T + 1) for layer 2."""
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
        E = Hk @ W2 + c2 - Vb
        D1 = (E @ W2.T) * (Phi(A) + A * phi(A))
        S1 = np.tril(Qb @ Kb.T + 1.0)
        Aq = Qb @ W1 + c1 - (S1 * eb[None, :]) @ D1
        Hq = gelu(Aq)
        S2 = np.tril(Hq @ Hk.T + 1.0)
        Z[sl] = Hq @ W2 + c2 - (S2 * eb[None, :]) @ E
        W1 = W1 - Kb.T @ (eb[:, None] * D1)
        c1 = c1 - eb @ D1
        W2 = W2 - Hk.T @ (eb[:, None] * E)
        c2 = c2 - eb @ E
    return Z, W1, c1, W2, c2


CASES = [(d, b, T) for d in (2, 3, 4, 8) for b in (1, 2, 4, 16) for T in (b, 2 * b, 5 * b, 5 * b + 3)]


@pytest.mark.parametrize("d,b,T", CASES)
@pytest.mark.parametrize("use_ln", [False, True])
def test_primal_equals_dual_linear(d, b, T, use_ln):
    Q, K, V, eta, W0, ex = make_linear(1, 2, T, d, use_ln)
    Z, Wo, co = O.linear_forward(Q, K, V, eta, W0, b, use_ln=use_ln, **ex)
    for h in range(2):
        Zd, Wd, cd = dual_linear_unit(Q[0, h], K[0, h], V[0, h], eta[0, h], W0[h], b,
                                      c=ex["c0"][h] if use_ln else None, use_ln=use_ln,
                                      gamma=ex["gamma"][h] if use_ln else None,
                                      beta=ex["beta"][h] if use_ln else None)
        assert rel(Z[0, h], Zd) < 1e-10
        assert rel(Wo[0, h], Wd) < 1e-10
        if use_ln:
            assert rel(co[0, h], cd) < 1e-10


@pytest.mark.parametrize("d,b,T", [c for c in CASES if c[0] in (2, 3, 4)])
def test_primal_equals_dual_mlp(d, b, T):
    m = 4 * d
    Q, K, V, eta, W1, c1, W2, c2 = make_mlp(1, 2, T, d, m)
    Z, W1o, c1o, W2o, c2o = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b)
    for h in range(2):
        Zd, W1d, c1d, W2d, c2d = dual_mlp_unit(Q[0, h], K[0, h], V[0, h], eta[0, h], W1[h], c1[h], W2[h],
                                               c2[h], b)
        for x, y in ((Z[0, h], Zd), (W1o[0, h], W1d), (c1o[0, h], c1d), (W2o[0, h], W2d),
                     (c2o[0, h], c2d)):
            assert rel(x, y) < 1e-10


# ---------------------------------------------------------------------------
# P2: b = 1 is the sequential delta rule (section 2.6: DeltaNet is TTT-Linear
# with b = 1 and no LN/residual; section 3.1: update, then output)
# ---------------------------------------------------------------------------

def delta_rule(Q, K, V, eta, W):
    W = W.copy()
    Z = np.empty_like(Q)
    for t in range(Q.shape[0]):
        W = W - eta[t] * np.outer(K[t], K[t] @ W - V[t])
        Z[t] = Q[t] @ W
    return Z, W


@pytest.mark.parametrize("d,T", [(2, 7), (4, 33), (16, 64)])
def test_b1_is_delta_rule(d, T):
    Q, K, V, eta, W0, _ = make_linear(2, 1, T, d)
    Z, Wo, _ = O.linear_forward(Q, K, V, eta, W0, 1)
    for n in range(2):
        Zr, Wr = delta_rule(Q[n, 0], K[n, 0], V[n, 0], eta[n, 0], W0[0])
        assert rel(Z[n, 0], Zr) < 1e-12
        assert rel(Wo[n, 0], Wr) < 1e-12


def test_decode_step_is_delta_rule():
    d, steps = 8, 5
    W = rand(3, 2, d, d, scale=1 / np.sqrt(d))
    Wr = W.copy()
    for _ in range(steps):
        q, k, v = (rand(3, 2, d, scale=1 / np.sqrt(d)) for _ in range(3))
        eta = np.abs(rand(3, 2)) * 0.5
        W, z = O.linear_decode_step(W, q, k, v, eta)
        for n in range(3):
            for h in range(2):
                Zr, Wn = delta_rule(q[n, h][None], k[n, h][None], v[n, h][None], eta[n, h][None], Wr[n, h])
                Wr[n, h] = Wn
                assert rel(z[n, h], Zr[0]) < 1e-12
    assert rel(W, Wr) < 1e-12


# ---------------------------------------------------------------------------
# P3: finite differences of the reconstruction loss (sections 3.3, 3.5):
# after ONE mini-batch, W_b = W_0 - grad_W sum_t eta_t 1/2 ||f(k_t; W_0) - v_t||^2
# ---------------------------------------------------------------------------

def fd_grad(loss, params, h=1e-6):
    grads = []
    for p in params:
        g = np.zeros_like(p)
        it = np.nditer(p, flags=["multi_index"])
        for _ in it:
            ix = it.multi_index
            old = p[ix]
            p[ix] = old + h
            lp = loss()
            p[ix] = old - h
            lm = loss()
            p[ix] = old
            g[ix] = (lp - lm) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("use_ln", [False, True])
def test_fd_gradient_linear(use_ln):
    d, T = 4, 6
    Q, K, V, eta, W0, ex = make_linear(1, 1, T, d, use_ln, eta_scale=0.5)
    Z, Wo, co = O.linear_forward(Q, K, V, eta, W0, T, use_ln=use_ln, **ex)
    W = W0[0].copy()
    c = ex["c0"][0].copy() if use_ln else np.zeros(d)
    g = ex["gamma"][0] if use_ln else None
    be = ex["beta"][0] if use_ln else None
    k, v, e = K[0, 0], V[0, 0], eta[0, 0]

    def loss():
        R = f_linear(k, W, c, use_ln, g, be) - v
        return 0.5 * np.sum(e[:, None] * R * R)

    params = [W, c] if use_ln else [W]
    grads = fd_grad(loss, params)
    assert rel(W0[0] - Wo[0, 0], grads[0]) < 1e-7
    if use_ln:
        assert rel(ex["c0"][0] - co[0, 0], grads[1]) < 1e-7


def test_fd_gradient_mlp():
    d, m, T = 3, 12, 5
    Q, K, V, eta, W1, c1, W2, c2 = make_mlp(1, 1, T, d, m, eta_scale=0.5)
    Z, W1o, c1o, W2o, c2o = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, T)
    P = [W1[0].copy(), c1[0].copy(), W2[0].copy(), c2[0].copy()]
    k, v, e = K[0, 0], V[0, 0], eta[0, 0]

    def loss():
        R = f_mlp(k, *P) - v
        return 0.5 * np.sum(e[:, None] * R * R)

    g = fd_grad(loss, P)
    assert rel(W1[0] - W1o[0, 0], g[0]) < 1e-7
    assert rel(c1[0] - c1o[0, 0], g[1]) < 1e-7
    assert rel(W2[0] - W2o[0, 0], g[2]) < 1e-7
    assert rel(c2[0] - c2o[0, 0], g[3]) < 1e-7


# ---------------------------------------------------------------------------
# output rule: z_t = f(q_t; W_t) with W_t the state after token t itself
# (section 3.1, update then output; causal mask includes the diagonal)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["linear", "ln", "mlp"])
def test_output_uses_state_after_own_token(kind):
    d, b, T = 3, 4, 11
    if kind == "mlp":
        Q, K, V, eta, W1, c1, W2, c2 = make_mlp(1, 1, T, d, 4 * d)
        Z = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b)[0]
        for t in range(T):
            _, W1t, c1t, W2t, c2t = O.mlp_forward(Q[:, :, :t + 1], K[:, :, :t + 1], V[:, :, :t + 1],
                                                  eta[:, :, :t + 1], W1, c1, W2, c2, b)
            assert rel(Z[0, 0, t], f_mlp(Q[0, 0, t], W1t[0, 0], c1t[0, 0], W2t[0, 0], c2t[0, 0])) < 1e-12
    else:
        use_ln = kind == "ln"
        Q, K, V, eta, W0, ex = make_linear(1, 1, T, d, use_ln)
        Z = O.linear_forward(Q, K, V, eta, W0, b, use_ln=use_ln, **ex)[0]
        for t in range(T):
            _, Wt, ct = O.linear_forward(Q[:, :, :t + 1], K[:, :, :t + 1], V[:, :, :t + 1], eta[:, :, :t + 1],
                                         W0, b, use_ln=use_ln, **ex)
            zt = f_linear(Q[0, 0, t], Wt[0, 0], ct[0, 0], use_ln, ex.get("gamma", [None])[0],
                          ex.get("beta", [None])[0])
            assert rel(Z[0, 0, t], zt) < 1e-12


# ---------------------------------------------------------------------------
# P4: Theorem 1 (section 4.1): linear model, batch GD (b = T), W0 = 0 and
# eta = 1/2 in the full-loss form (eta = 1 in the half-loss form) is causal
# linear attention z_t = sum_{s<=t} (q_t . k_s) v_s
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d,T", [(4, 9), (16, 16), (8, 40)])
def test_theorem1_linear_attention(d, T):
    Q, K, V, _, _, _ = make_linear(1, 1, T, d)
    Z, _, _ = O.linear_forward(Q, K, V, np.ones((1, 1, T)), np.zeros((1, d, d)), T)
    q, k, v = Q[0, 0], K[0, 0], V[0, 0]
    ref = np.array([sum((q[t] @ k[s]) * v[s] for s in range(t + 1)) for t in range(T)])
    assert rel(Z[0, 0], ref) < 1e-12


# ---------------------------------------------------------------------------
# P5: eta = 0 leaves the state untouched
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["linear", "ln", "mlp"])
def test_eta_zero(kind):
    d, T = 4, 20
    if kind == "mlp":
        Q, K, V, eta, W1, c1, W2, c2 = make_mlp(2, 2, T, d, 16)
        Z, W1o, c1o, W2o, c2o = O.mlp_forward(Q, K, V, 0 * eta, W1, c1, W2, c2, 4)
        assert np.array_equal(W1o, np.broadcast_to(W1, W1o.shape))
        assert np.array_equal(W2o, np.broadcast_to(W2, W2o.shape))
        for h in range(2):
            assert rel(Z[:, h], f_mlp(Q[:, h], W1[h], c1[h], W2[h], c2[h])) < 1e-13
    else:
        use_ln = kind == "ln"
        Q, K, V, eta, W0, ex = make_linear(2, 2, T, d, use_ln)
        Z, Wo, co = O.linear_forward(Q, K, V, 0 * eta, W0, 4, use_ln=use_ln, **ex)
        assert np.array_equal(Wo, np.broadcast_to(W0, Wo.shape))
        for h in range(2):
            zr = f_linear(Q[:, h], W0[h], ex["c0"][h] if use_ln else None, use_ln,
                          ex["gamma"][h] if use_ln else None, ex["beta"][h] if use_ln else None)
            assert rel(Z[:, h], zr) < 1e-13


# ---------------------------------------------------------------------------
# closed form for d = 1, b = 2 (worked by hand from sections 3.1 and 3.5):
#   g_t = k_t (k_t w - v_t) at the batch start w
#   w_1 = w - eta_1 g_1, z_1 = q_1 w_1;  w_2 = w_1 - eta_2 g_2, z_2 = q_2 w_2
# ---------------------------------------------------------------------------

def test_scalar_closed_form():
    w, k1, k2, v1, v2, q1, q2, e1, e2 = 0.7, 1.5, -0.5, 0.25, 2.0, 3.0, -1.0, 0.1, 0.3
    g1 = k1 * (k1 * w - v1)
    g2 = k2 * (k2 * w - v2)          # taken at w, not at w_1
    w1 = w - e1 * g1
    w2 = w1 - e2 * g2
    Q = np.array([q1, q2]).reshape(1, 1, 2, 1)
    K = np.array([k1, k2]).reshape(1, 1, 2, 1)
    V = np.array([v1, v2]).reshape(1, 1, 2, 1)
    eta = np.array([e1, e2]).reshape(1, 1, 2)
    Z, Wo, _ = O.linear_forward(Q, K, V, eta, np.full((1, 1, 1), w), 2)
    assert abs(Z[0, 0, 0, 0] - q1 * w1) < 1e-15
    assert abs(Z[0, 0, 1, 0] - q2 * w2) < 1e-15
    assert abs(Wo[0, 0, 0, 0] - w2) < 1e-15
    # with b = 1 the second gradient is taken at w_1 instead
    Z1, Wo1, _ = O.linear_forward(Q, K, V, eta, np.full((1, 1, 1), w), 1)
    assert abs(Wo1[0, 0, 0, 0] - (w1 - e2 * k2 * (k2 * w1 - v2))) < 1e-15


# ---------------------------------------------------------------------------
# P6: resumable state: forward(T1) then forward(T2) from its final state
# equals forward(T1 + T2) when T1 is a multiple of b
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["linear", "ln", "mlp"])
def test_chunked_calls(kind):
    d, b, T1, T2 = 4, 4, 12, 9
    T = T1 + T2
    if kind == "mlp":
        Q, K, V, eta, W1, c1, W2, c2 = make_mlp(1, 2, T, d, 16)
        full = O.mlp_forward(Q, K, V, eta, W1, c1, W2, c2, b)
        a = O.mlp_forward(Q[:, :, :T1], K[:, :, :T1], V[:, :, :T1], eta[:, :, :T1], W1, c1, W2, c2, b)
        s = O.mlp_forward(Q[:, :, T1:], K[:, :, T1:], V[:, :, T1:], eta[:, :, T1:], *a[1:], b)
        assert rel(np.concatenate([a[0], s[0]], 2), full[0]) < 1e-12
        for x, y in zip(s[1:], full[1:]):
            assert rel(x, y) < 1e-12
    else:
        use_ln = kind == "ln"
        Q, K, V, eta, W0, ex = make_linear(1, 2, T, d, use_ln)
        full = O.linear_forward(Q, K, V, eta, W0, b, use_ln=use_ln, **ex)
        a = O.linear_forward(Q[:, :, :T1], K[:, :, :T1], V[:, :, :T1], eta[:, :, :T1], W0, b,
                             use_ln=use_ln, **ex)
        ex2 = dict(ex)
        if use_ln:
            ex2["c0"] = a[2]
        s = O.linear_forward(Q[:, :, T1:], K[:, :, T1:], V[:, :, T1:], eta[:, :, T1:], a[1], b,
                             use_ln=use_ln, **ex2)
        assert rel(np.concatenate([a[0], s[0]], 2), full[0]) < 1e-12
        assert rel(s[1], full[1]) < 1e-12


# ---------------------------------------------------------------------------
# P7: TTT-Linear without LN: output columns evolve independently, so
# permuting the columns of W0 and V permutes the columns of Z and W_out
# ---------------------------------------------------------------------------

def test_column_permutation():
    d, T, b = 6, 24, 4
    Q, K, V, eta, W0, _ = make_linear(1, 1, T, d)
    perm = RNG.permutation(d)
    Z, Wo, _ = O.linear_forward(Q, K, V, eta, W0, b)
    Zp, Wop, _ = O.linear_forward(Q, K, V[..., perm], eta, W0[..., perm], b)
    assert rel(Zp, Z[..., perm]) < 1e-13
    assert rel(Wop, Wo[..., perm]) < 1e-13


def test_shared_vs_per_sequence_W0():
    d, T, b = 4, 8, 4
    Q, K, V, eta, W0, _ = make_linear(3, 2, T, d)
    a = O.linear_forward(Q, K, V, eta, W0, b)
    full = np.broadcast_to(W0, (3, 2, d, d)).copy()
    c = O.linear_forward(Q, K, V, eta, full, b)
    assert np.array_equal(a[0], c[0]) and np.array_equal(a[1], c[1])
