"""Parity of the fused prologue (ttt_qkv_prologue) with the float64 oracle:
the three views (paper digest "论文速览 | TTT", section 3.3) and the
learning-rate gate (section 4.6) from the layer input, on seeded inputs.

Tolerances, from the arithmetic: the GPU multiplies the stored bf16 values
exactly and accumulates in fp32 over Dm terms, then rounds each view once to
bf16.  Per element, with S = sum_k |x_k| |theta_k|:
    |Q_gpu - Q| <= 2^-8 |Q| + 2^-12 S
(2^-8: one bf16 rounding; 2^-12 >= Dm * 2^-24 for Dm <= 4096 bounds the fp32
accumulation).  The gate's logit carries the same accumulation error and the
sigmoid's slope is at most 1/4, so
    |eta_gpu - eta| <= eta_base (2^-12 S_lr / 4 + 1e-6) .
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from test_sequence_layers_head_b200 import workloads as WL
from tests.gpu_util import TOL_BF16_NORMWISE, maxrel, normwise, to_dev, to_host

pytestmark = [pytest.mark.gpu,
              pytest.mark.skip(reason="prologue kernel: first supervised B200 run pending")]


def view_bounds(x, theta, H, d):
    """S[n, h, t, j] = sum_k |x[n,t,k]| |theta[h d + j, k]|."""
    B, T, _ = x.shape
    S = np.abs(x) @ np.abs(theta).T
    return S.reshape(B, T, H, d).transpose(0, 2, 1, 3)


def check_views(got, ref, S):
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * S
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (worst, got[worst], ref[worst], bound[worst])


def check_eta(got, ref, S_lr, eta_base):
    assert np.all(np.isfinite(got))
    bound = eta_base * (2.0 ** -12 * S_lr / 4 + 1e-6)
    assert np.all(np.abs(got - ref) <= bound)


def run_gpu(w, inp, flags=0, wait_ms=0):
    r = inp["raw"]
    dev = {nm: to_dev(v) for nm, v in r.items()}
    B, H, T, d = w.B, w.H, w.T, w.d
    Q, K, V = (torch.full((B, H, T, d), float("nan"), device="cuda", dtype=torch.bfloat16) for _ in range(3))
    eta = torch.full((B, H, T), float("nan"), device="cuda") if w.gate else None
    from test_sequence_layers_head_b200 import ttt
    ttt.qkv_prologue(dev["x"], dev["theta_q"], dev["theta_k"], dev["theta_v"],
                     dev["theta_lr"] if w.gate else None, w.eta_base, d, Q=Q, K=K, V=V, eta=eta, flags=flags,
                     wait_timeout_ms=wait_ms)
    torch.cuda.synchronize()
    return Q, K, V, eta


CASES = [
    # B, T, Dm, H, d, gate: ragged token tiles (T * B not a multiple of 128), a model
    # width that is not a multiple of 64, view widths with a partial 256-column
    # tile, H not a multiple of 16 for the gate, every head dim
    (2, 200, 136, 5, 64, True),
    (1, 1, 8, 1, 16, True),
    (3, 100, 72, 17, 16, True),
    (2, 77, 64, 12, 64, False),
    (4, 33, 16, 7, 32, True),
    (1, 129, 2048, 2, 64, True),
    (2, 384, 768, 12, 64, True),
]


@pytest.mark.parametrize("B,T,Dm,H,d,gate", CASES)
def test_prologue_parity(ttt_lib, B, T, Dm, H, d, gate):
    w, inp = WL.prologue_case(B, T, Dm, H, d, gate=gate, eta_base=0.5)
    Q, K, V, eta = run_gpu(w, inp)
    e = inp["exact"]
    ref = O.qkv_prologue(e["x"], e["theta_q"], e["theta_k"], e["theta_v"], e["theta_lr"], w.eta_base, d)
    for got, want, nm in zip((Q, K, V), ref[:3], ("theta_q", "theta_k", "theta_v")):
        check_views(to_host(got), want, view_bounds(e["x"], e[nm], H, d))
    if gate:
        S_lr = (np.abs(e["x"]) @ np.abs(e["theta_lr"]).T).transpose(0, 2, 1)
        check_eta(to_host(eta), ref[3], S_lr, w.eta_base)
    assert ttt_lib.last_device_status() == 0


@pytest.mark.parametrize("name", list(WL.PROLOGUE_WORKLOADS))
def test_prologue_full_size_sampled(ttt_lib, name):
    """Full-size launch; 48 sampled tokens (whole blocks regenerated on the
    host) checked against the oracle, every output finite."""
    w = WL.PROLOGUE_WORKLOADS[name]
    inp = WL.make_prologue_inputs(w, want_exact=False)
    Q, K, V, eta = run_gpu(w, inp)
    for t in (Q, K, V, eta):
        assert bool(torch.isfinite(t).all())
    e = inp["exact"]
    rng = np.random.default_rng(5)
    picks = sorted({(int(rng.integers(w.B)), int(rng.integers(w.T))) for _ in range(48)} | {(w.B - 1, w.T - 1)})
    xs = np.stack([WL.store(WL.prologue_x_block(w, n, t // WL.PRO_BLOCK), WL.BF16)[1][t % WL.PRO_BLOCK]
                   for n, t in picks])[None]
    ref = O.qkv_prologue(xs, e["theta_q"], e["theta_k"], e["theta_v"], e["theta_lr"], w.eta_base, w.d)
    idx_n = torch.tensor([n for n, _ in picks], device="cuda")
    idx_t = torch.tensor([t for _, t in picks], device="cuda")
    for got, want, nm in zip((Q, K, V), ref[:3], ("theta_q", "theta_k", "theta_v")):
        g = to_host(got[idx_n, :, idx_t, :]).transpose(1, 0, 2)[None]   # [1, H, S, d]
        check_views(g, want, view_bounds(xs, e[nm], w.H, w.d))
    S_lr = (np.abs(xs) @ np.abs(e["theta_lr"]).T).transpose(0, 2, 1)
    check_eta(to_host(eta[idx_n, :, idx_t]).T[None], ref[3], S_lr, w.eta_base)


def test_prologue_then_forward(ttt_lib):
    """The prologue's outputs drive the tensor-core TTT-Linear forward as they
    stand: GPU prologue -> GPU forward against oracle prologue -> bf16
    storage -> oracle forward (normwise, the bf16 bar)."""
    from test_sequence_layers_head_b200 import ttt
    w, inp = WL.prologue_case(2, 256, 768, 12, 64, gate=True, eta_base=1.0 / 64)
    Q, K, V, eta = run_gpu(w, inp)
    e = inp["exact"]
    W0 = np.random.default_rng(3).standard_normal((w.H, w.d, w.d)) / np.sqrt(w.d)
    W0_dev = torch.from_numpy(W0.astype(np.float32)).cuda()
    Z, W_out, _ = ttt.linear_forward(Q, K, V, eta, W0_dev, 16)
    torch.cuda.synchronize()
    Qr, Kr, Vr, er = O.qkv_prologue(e["x"], e["theta_q"], e["theta_k"], e["theta_v"], e["theta_lr"],
                                    w.eta_base, w.d)
    Qs, Ks, Vs = (WL.store(a, WL.BF16)[1] for a in (Qr, Kr, Vr))
    es = WL.store(er, WL.F32)[1]
    Zr, Wr, _ = O.linear_forward(Qs, Ks, Vs, es, W0.astype(np.float32).astype(np.float64), 16)
    assert normwise(to_host(Z), Zr) <= TOL_BF16_NORMWISE
    assert normwise(to_host(W_out), Wr) <= TOL_BF16_NORMWISE


def test_prologue_stall_reports_timeout(ttt_lib):
    """A wait that nothing ends expires (about 0.2 s), the call reports
    TTT_ERR_TIMEOUT, and the context still serves a normal call."""
    from test_sequence_layers_head_b200 import ttt
    w, inp = WL.prologue_case(1, 256, 128, 4, 64)
    run_gpu(w, inp, flags=ttt.FLAG_TEST_STALL, wait_ms=200)
    assert ttt_lib.last_device_status() == ttt.TTT_ERR_TIMEOUT
    Q, K, V, eta = run_gpu(w, inp)
    e = inp["exact"]
    ref = O.qkv_prologue(e["x"], e["theta_q"], e["theta_k"], e["theta_v"], e["theta_lr"], w.eta_base, w.d)
    check_views(to_host(Q), ref[0], view_bounds(e["x"], e["theta_q"], w.H, w.d))
    assert ttt_lib.last_device_status() == 0


@pytest.mark.parametrize("B,T,Dm,H,d,gate", [(2, 20, 40, 3, 16, True), (1, 33, 264, 2, 64, True),
                                             (1, 256, 768, 12, 64, True)])
def test_prologue_fp32_on_cuda_cores(ttt_lib, B, T, Dm, H, d, gate):
    """fp32 input runs on the CUDA-core kernel: max relative error <= 1e-4."""
    from test_sequence_layers_head_b200 import ttt
    w, inp = WL.prologue_case(B, T, Dm, H, d, gate=gate, eta_base=0.5)
    e = inp["exact"]
    dev = {k: torch.from_numpy(v.astype(np.float32)).cuda() for k, v in e.items()}
    Q, K, V, eta = ttt.qkv_prologue(dev["x"], dev["theta_q"], dev["theta_k"], dev["theta_v"],
                                    dev["theta_lr"] if gate else None, 0.5, d)
    torch.cuda.synchronize()
    ref = O.qkv_prologue(e["x"], e["theta_q"], e["theta_k"], e["theta_v"], e["theta_lr"], 0.5, d)
    for got, want in zip((Q, K, V), ref[:3]):
        assert maxrel(to_host(got), want) <= 1e-4
    if gate:
        assert maxrel(to_host(eta), ref[3]) <= 1e-4


def test_prologue_tensor_cores_match_cuda_cores_at_full_width(ttt_lib):
    """bf16 at the 32-head width (Dm = 2048): the tcgen05 kernel against the
    CUDA-core kernel (TTT_FLAG_FORCE_SIMT) on every output, within two bf16
    roundings."""
    from test_sequence_layers_head_b200 import ttt
    w, inp = WL.prologue_case(2, 512, 2048, 32, 64, gate=True)
    dev = {k: to_dev(v) for k, v in inp["raw"].items()}
    a = ttt.qkv_prologue(dev["x"], dev["theta_q"], dev["theta_k"], dev["theta_v"], dev["theta_lr"], w.eta_base, 64)
    b = ttt.qkv_prologue(dev["x"], dev["theta_q"], dev["theta_k"], dev["theta_v"], dev["theta_lr"], w.eta_base, 64,
                         flags=ttt.FLAG_FORCE_SIMT)
    torch.cuda.synchronize()
    for x, y in zip(a[:3], b[:3]):
        x, y = to_host(x), to_host(y)
        assert np.all(np.abs(x - y) <= 2.0 ** -7 * np.abs(y) + 1e-3)
    assert maxrel(to_host(a[3]), to_host(b[3])) <= 1e-3
