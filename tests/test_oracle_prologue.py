"""Pins of the oracle's prologue: the multi-view projections q = theta_Q x,
k = theta_K x, v = theta_V x (paper digest "论文速览 | TTT", section 3.3) and
the learnable learning rate eta(x) = eta_base sigmoid(theta_lr^T x)
(section 4.6), computed from the layer input.

The pins do not restate the oracle's sums:
  - a one-hot input e_k selects column k of each view matrix, head h's rows
    h*d .. h*d+d-1, at the token's own place in the [B, H, T, d] layout;
  - the views are linear in x (with the one-hot values this fixes them);
  - the gate takes the sigmoid's closed-form values sigmoid(0) = 1/2,
    sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4, saturates at eta_base, and
    eta(u) + eta(-u) = eta_base.
"""
import numpy as np
import pytest

from oracle import oracle as O

RNG = np.random.default_rng(9090)


def views(H, d, Dm):
    return [RNG.standard_normal((H * d, Dm)) for _ in range(3)], RNG.standard_normal((H, Dm))


@pytest.mark.parametrize("B,T,Dm,H,d", [(1, 1, 1, 1, 1), (2, 5, 7, 3, 4), (3, 4, 20, 2, 6), (1, 9, 12, 4, 3)])
def test_one_hot_input_selects_view_columns(B, T, Dm, H, d):
    (tq, tk, tv), tl = views(H, d, Dm)
    kidx = RNG.integers(0, Dm, size=(B, T))
    x = np.zeros((B, T, Dm))
    for n in range(B):
        for t in range(T):
            x[n, t, kidx[n, t]] = 1.0
    Q, K, V, _ = O.qkv_prologue(x, tq, tk, tv, tl, 1.0, d)
    for n in range(B):
        for t in range(T):
            c = kidx[n, t]
            for h in range(H):
                assert np.array_equal(Q[n, h, t], tq[h * d:(h + 1) * d, c])
                assert np.array_equal(K[n, h, t], tk[h * d:(h + 1) * d, c])
                assert np.array_equal(V[n, h, t], tv[h * d:(h + 1) * d, c])


def test_views_are_linear_in_the_input():
    B, T, Dm, H, d = 2, 6, 9, 3, 4
    (tq, tk, tv), tl = views(H, d, Dm)
    x1, x2 = RNG.standard_normal((B, T, Dm)), RNG.standard_normal((B, T, Dm))
    a, b = 0.7, -1.3
    o1 = O.qkv_prologue(x1, tq, tk, tv, tl, 1.0, d)
    o2 = O.qkv_prologue(x2, tq, tk, tv, tl, 1.0, d)
    o = O.qkv_prologue(a * x1 + b * x2, tq, tk, tv, tl, 1.0, d)
    for i in range(3):
        assert np.allclose(o[i], a * o1[i] + b * o2[i], rtol=0, atol=1e-12)
    # a zero input gives zero views and the gate's midpoint
    z = O.qkv_prologue(np.zeros((B, T, Dm)), tq, tk, tv, tl, 0.3, d)
    for i in range(3):
        assert not np.any(z[i])
    assert np.all(z[3] == 0.15)


def test_gate_closed_forms_per_head():
    """Head h's gate reads row h of theta_lr: with x = e_0 the logit is
    theta_lr[h, 0], set to 0, ln 3, -ln 3 and a large value on four heads."""
    H, d, Dm, T = 4, 2, 5, 3
    (tq, tk, tv), _ = views(H, d, Dm)
    tl = np.zeros((H, Dm))
    tl[:, 0] = [0.0, np.log(3.0), -np.log(3.0), 60.0]
    tl[:, 1:] = RNG.standard_normal((H, Dm - 1))    # not read: x is zero there
    x = np.zeros((1, T, Dm))
    x[0, :, 0] = 1.0
    eta_base = 0.25
    eta = O.qkv_prologue(x, tq, tk, tv, tl, eta_base, d)[3]
    want = eta_base * np.array([0.5, 0.75, 0.25, 1.0])
    for t in range(T):
        assert np.allclose(eta[0, :, t], want, rtol=1e-14, atol=0)


def test_gate_symmetry_and_range():
    B, T, Dm, H, d = 2, 7, 6, 3, 2
    (tq, tk, tv), tl = views(H, d, Dm)
    x = RNG.standard_normal((B, T, Dm))
    eta_base = 1.0 / 64
    e1 = O.qkv_prologue(x, tq, tk, tv, tl, eta_base, d)[3]
    e2 = O.qkv_prologue(-x, tq, tk, tv, tl, eta_base, d)[3]
    assert np.allclose(e1 + e2, eta_base, rtol=0, atol=1e-15)
    assert np.all(e1 > 0) and np.all(e1 < eta_base)
    # the gate is monotone in the logit: doubling theta_lr moves eta away from the midpoint
    e3 = O.qkv_prologue(x, tq, tk, tv, 2 * tl, eta_base, d)[3]
    assert np.all(np.abs(e3 - eta_base / 2) >= np.abs(e1 - eta_base / 2))


def test_views_feed_the_inner_loop_unchanged():
    """The prologue's outputs are the inner loop's inputs as they stand: the
    forward on them equals the forward on views built from one-hot columns."""
    B, T, Dm, H, d, b = 1, 8, 6, 2, 3, 4
    (tq, tk, tv), tl = views(H, d, Dm)
    kidx = RNG.integers(0, Dm, size=T)
    x = np.zeros((B, T, Dm))
    x[0, np.arange(T), kidx] = 1.0
    Q, K, V, eta = O.qkv_prologue(x, tq, tk, tv, tl, 0.2, d)
    Qc = np.stack([np.stack([tq[h * d:(h + 1) * d, kidx[t]] for t in range(T)]) for h in range(H)])[None]
    Kc = np.stack([np.stack([tk[h * d:(h + 1) * d, kidx[t]] for t in range(T)]) for h in range(H)])[None]
    Vc = np.stack([np.stack([tv[h * d:(h + 1) * d, kidx[t]] for t in range(T)]) for h in range(H)])[None]
    W0 = RNG.standard_normal((H, d, d)) / np.sqrt(d)
    a = O.linear_forward(Q, K, V, eta, W0, b)
    c = O.linear_forward(Qc, Kc, Vc, eta, W0, b)
    for x1, x2 in zip(a, c):
        if x1 is not None:
            assert np.array_equal(x1, x2)


def test_rejects_bad_shapes():
    (tq, tk, tv), tl = views(2, 3, 4)
    with pytest.raises(ValueError):
        O.qkv_prologue(np.zeros((1, 2, 5)), tq, tk, tv, tl, 1.0, 3)   # Dm mismatch
    with pytest.raises(ValueError):
        O.qkv_prologue(np.zeros((1, 2, 4)), tq, tk, tv, tl, 1.0, 2)   # d mismatch
