"""Seeded synthetic workloads for the TTT inner-loop forward.

This module holds the shapes of the five workloads and the seeded random
generators that produce their inputs.  It holds none of the method's
arithmetic: it only draws numbers, rounds them to the storage dtype and
packs them.  Both the CUDA path (through the Python binding) and the float64
oracle consume exactly what these generators return, so the two sides see the
same inputs bit for bit.

Recipe (the shapes and value distributions follow the problem statement of
"Learning to (Learn at Test Time): RNNs with Expressive Hidden States",
section 3 (mini-batch TTT, dual form) and section 4.4-4.6 (TTT-Linear,
TTT-MLP, LN+residual, learnable W0 and per-token learning rate)):

* generator: numpy ``PCG64``; every (sequence, head) unit has its own stream
  keyed by ``(seed, stream_id, unit)`` so that any single unit can be
  regenerated on the host without drawing the others;
* values are drawn in float64 and rounded once to the storage dtype
  (round-to-nearest-even to bf16 or fp32);
* ``N(0, s)`` means variance ``s``;
* per-token learning rate ``eta_t = (1/64) * sigmoid(u_t)``, ``u_t ~ N(0,1)``;
* per-head parameters (W0, LN gamma/beta, MLP weights) are drawn from the
  head's own stream and broadcast over the batch of sequences.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "linear", "ln" or "mlp"
    B: int
    H: int
    T: int
    d: int
    b: int
    io_dtype: str        # storage dtype of Q, K, V and Z
    eta_mode: str        # "const" or "sigmoid"
    eta_const: float
    seed: int
    decode_steps: int = 0
    ln_eps: float = 1e-6

    @property
    def units(self) -> int:
        return self.B * self.H

    @property
    def hidden(self) -> int:
        return 4 * self.d


# The five workloads of the problem statement, named by what they are.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("linear_d16_T256_f32", "linear", 1, 1, 256, 16, 16, F32, "const", 0.1, 20260000),
        Workload("linear_B8_H12_T2048", "linear", 8, 12, 2048, 64, 16, BF16, "sigmoid", 0.0, 20260001),
        Workload("ln_B4_H32_T8192", "ln", 4, 32, 8192, 64, 16, BF16, "sigmoid", 0.0, 20260002),
        Workload("mlp_B2_H32_T8192", "mlp", 2, 32, 8192, 64, 16, BF16, "const", 1.0 / 64.0, 20260003),
        Workload("linear_B16_H32_T32768_decode1024", "linear", 16, 32, 32768, 64, 16, BF16, "sigmoid",
                 0.0, 20260004, decode_steps=1024),
    ]
}
WORKLOAD_ORDER = list(WORKLOADS)


def scaled(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(w, **kw)


# ----------------------------------------------------------------------------
# rounding helpers (storage formats only)
# ----------------------------------------------------------------------------

def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    u = x.view(np.uint64)
    # bf16 keeps 7 explicit mantissa bits; float64 has 52 -> drop 45 bits.
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    r = (u + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f32 = r.view(np.float64).astype(np.float32)      # exact: value has <= 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def store(x: np.ndarray, dtype: str):
    """Round float64 ``x`` to the storage dtype.

    Returns ``(raw, exact)``: ``raw`` is what goes to the device (uint16 bf16
    bits or float32), ``exact`` its exact value in float64 for the oracle.
    """
    if dtype == BF16:
        raw = round_to_bf16_bits(x)
        return raw, bf16_bits_to_f64(raw)
    raw = np.ascontiguousarray(x, dtype=np.float32)
    return raw, raw.astype(np.float64)


def _sigmoid(u):
    return 1.0 / (1.0 + np.exp(-u))


# stream ids: one independent PCG64 stream per (purpose, unit or head)
_S_TOKENS, _S_HEAD, _S_DECODE = 1, 2, 3


def _rng(seed: int, stream: int, index: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream, index]))


def unit_tokens(w: Workload, unit: int, T: Optional[int] = None):
    """Q, K, V and u (eta logits) of one (sequence, head) unit, float64 draws."""
    T = w.T if T is None else T
    g = _rng(w.seed, _S_TOKENS, unit)
    sd = np.sqrt(1.0 / w.d)
    Q = g.standard_normal((T, w.d)) * sd
    K = g.standard_normal((T, w.d)) * sd
    V = g.standard_normal((T, w.d)) * sd
    u = g.standard_normal(T)
    return Q, K, V, u


def head_params(w: Workload, head: int) -> dict:
    """Per-head parameters (shared over the batch of sequences), float64 draws."""
    g = _rng(w.seed, _S_HEAD, head)
    d = w.d
    out = {}
    if w.kind in ("linear", "ln"):
        out["W0"] = g.standard_normal((d, d)) * np.sqrt(1.0 / d)
        if w.kind == "ln":
            out["c0"] = np.zeros(d)
            out["gamma"] = 1.0 + g.standard_normal(d) * np.sqrt(0.02)
            out["beta"] = g.standard_normal(d) * np.sqrt(0.02)
    else:
        hdim = w.hidden
        out["W1"] = g.standard_normal((d, hdim)) * np.sqrt(1.0 / d)
        out["c1"] = np.zeros(hdim)
        out["W2"] = g.standard_normal((hdim, d)) * np.sqrt(1.0 / hdim)
        out["c2"] = np.zeros(d)
    return out


def eta_from_logits(w: Workload, u: np.ndarray) -> np.ndarray:
    if w.eta_mode == "const":
        return np.full(u.shape, w.eta_const)
    return _sigmoid(u) / 64.0


@dataclasses.dataclass
class Inputs:
    """Device-ready raw arrays plus their exact float64 values."""
    w: Workload
    raw: dict      # name -> numpy array in storage format (uint16 bf16 bits or float32)
    exact: dict    # name -> float64 array with the exact stored values


def _fill_units(w: Workload, units, T, dtype, raw, exact, want_exact):
    for n_unit in units:
        Q, K, V, u = unit_tokens(w, n_unit, T)
        for nm, x in (("Q", Q), ("K", K), ("V", V)):
            r, e = store(x, dtype)
            raw[nm][n_unit] = r
            if want_exact:
                exact[nm][n_unit] = e
        er, ee = store(eta_from_logits(w, u), F32)
        raw["eta"][n_unit] = er
        if want_exact:
            exact["eta"][n_unit] = ee


def make_inputs(w: Workload, want_exact: bool = True, threads: int = 8, T: Optional[int] = None) -> Inputs:
    """All inputs of workload ``w`` (prefill part).

    Q, K, V: ``[B,H,T,d]``; eta: ``[B,H,T]`` float32; per-head parameters
    ``[H,...]`` float32.  ``want_exact=False`` skips the float64 copies (used
    by the benchmark for the big workloads).
    """
    T = w.T if T is None else T
    U, d = w.units, w.d
    io = np.uint16 if w.io_dtype == BF16 else np.float32
    raw = {nm: np.empty((U, T, d), io) for nm in ("Q", "K", "V")}
    raw["eta"] = np.empty((U, T), np.float32)
    exact = {}
    if want_exact:
        exact = {nm: np.empty((U, T, d)) for nm in ("Q", "K", "V")}
        exact["eta"] = np.empty((U, T))
    chunks = [list(range(i, U, threads)) for i in range(min(threads, U))]
    with ThreadPoolExecutor(max_workers=len(chunks)) as ex:
        list(ex.map(lambda us: _fill_units(w, us, T, w.io_dtype, raw, exact, want_exact), chunks))
    for nm in list(raw):
        raw[nm] = raw[nm].reshape((w.B, w.H) + raw[nm].shape[1:])
    for nm in list(exact):
        exact[nm] = exact[nm].reshape((w.B, w.H) + exact[nm].shape[1:])
    heads = [head_params(w, h) for h in range(w.H)]
    for nm in heads[0]:
        r, e = store(np.stack([hp[nm] for hp in heads]), F32)
        raw[nm] = r
        exact[nm] = e
    return Inputs(w, raw, exact)


def make_unit_inputs(w: Workload, unit: int, T: Optional[int] = None) -> Inputs:
    """Inputs of one unit only (for sampled parity checks at full size).

    Arrays have B=H=1 layout; per-head parameters are those of ``unit % H``.
    """
    T = w.T if T is None else T
    Q, K, V, u = unit_tokens(w, unit, T)
    raw, exact = {}, {}
    for nm, x in (("Q", Q), ("K", K), ("V", V)):
        r, e = store(x, w.io_dtype)
        raw[nm], exact[nm] = r[None, None], e[None, None]
    r, e = store(eta_from_logits(w, u), F32)
    raw["eta"], exact["eta"] = r[None, None], e[None, None]
    hp = head_params(w, unit % w.H)
    for nm, x in hp.items():
        r, e = store(x, F32)
        raw[nm], exact[nm] = r[None], e[None]
    return Inputs(w, raw, exact)


def make_decode_tokens(w: Workload, step: int):
    """q, k, v ``[B,H,d]`` (storage dtype) and eta ``[B,H]`` of decode step ``step``."""
    g = _rng(w.seed, _S_DECODE, step)
    sd = np.sqrt(1.0 / w.d)
    shape = (w.B, w.H, w.d)
    q = g.standard_normal(shape) * sd
    k = g.standard_normal(shape) * sd
    v = g.standard_normal(shape) * sd
    u = g.standard_normal((w.B, w.H))
    out_raw, out_exact = {}, {}
    for nm, x in (("q", q), ("k", k), ("v", v)):
        out_raw[nm], out_exact[nm] = store(x, w.io_dtype)
    out_raw["eta"], out_exact["eta"] = store(eta_from_logits(w, u), F32)
    return out_raw, out_exact


def random_case(kind: str, B: int, H: int, T: int, d: int, b: int, io_dtype: str = BF16,
                eta_mode: str = "sigmoid", eta_const: float = 0.0, seed: int = 7) -> Inputs:
    """A small ad-hoc case with the same distributions (parity tests)."""
    w = Workload(f"{kind}_case", kind, B, H, T, d, b, io_dtype, eta_mode, eta_const, seed)
    return make_inputs(w, threads=1)


# ----------------------------------------------------------------------------
# the fused prologue: layer input and the view / gate weights
# ----------------------------------------------------------------------------
# Recipe: x ~ N(0, 1) per element (a normalised layer input); theta_q, theta_k,
# theta_v ~ N(0, 1/(Dm d)), so each view element has variance 1/d like the
# inner-loop workloads' Q, K, V; theta_lr ~ N(0, 1/Dm), so the gate's logits
# are ~ N(0, 1) like their u_t and eta_base = 1/64 reproduces their
# eta_t = (1/64) sigmoid(u_t).  All values are rounded once to bf16.  x is
# drawn in blocks of 128 tokens, one stream per (sequence, block), so any
# block can be regenerated alone.

_S_PRO_X, _S_PRO_THETA = 4, 5
PRO_BLOCK = 128


@dataclasses.dataclass(frozen=True)
class PrologueWorkload:
    name: str
    B: int
    T: int
    Dm: int
    H: int
    d: int
    gate: bool
    eta_base: float
    seed: int

    @property
    def tokens(self) -> int:
        return self.B * self.T


# the two model widths of the inner-loop workloads: 12 heads of 64 (width 768)
# and 32 heads of 64 (width 2048), at their batch and sequence sizes
PROLOGUE_WORKLOADS = {
    w.name: w
    for w in [
        PrologueWorkload("prologue_B8_T2048_Dm768_H12", 8, 2048, 768, 12, 64, True, 1.0 / 64.0, 20260011),
        PrologueWorkload("prologue_B16_T32768_Dm2048_H32", 16, 32768, 2048, 32, 64, True, 1.0 / 64.0, 20260014),
    ]
}


def prologue_x_block(w: PrologueWorkload, n: int, blk: int) -> np.ndarray:
    """Rows PRO_BLOCK*blk .. of sequence n of the layer input, float64 draws."""
    rows = min(PRO_BLOCK, w.T - PRO_BLOCK * blk)
    return _rng(w.seed, _S_PRO_X, n * 1_000_003 + blk).standard_normal((rows, w.Dm))


def prologue_theta(w: PrologueWorkload) -> dict:
    """theta_q, theta_k, theta_v [H*d, Dm] and theta_lr [H, Dm], float64 draws."""
    g = _rng(w.seed, _S_PRO_THETA, 0)
    sd = np.sqrt(1.0 / (w.Dm * w.d))
    out = {nm: g.standard_normal((w.H * w.d, w.Dm)) * sd for nm in ("theta_q", "theta_k", "theta_v")}
    out["theta_lr"] = g.standard_normal((w.H, w.Dm)) * np.sqrt(1.0 / w.Dm)
    return out


def make_prologue_inputs(w: PrologueWorkload, want_exact: bool = True, threads: int = 8) -> dict:
    """{"raw": ..., "exact": ...}: x [B, T, Dm] and the theta matrices as bf16
    bits (raw) and their exact float64 values (exact; skipped for x when
    want_exact is False)."""
    nblk = (w.T + PRO_BLOCK - 1) // PRO_BLOCK
    raw = {"x": np.empty((w.B, w.T, w.Dm), np.uint16)}
    exact = {"x": np.empty((w.B, w.T, w.Dm))} if want_exact else {}

    def fill(jobs):
        for n, blk in jobs:
            r, e = store(prologue_x_block(w, n, blk), BF16)
            s = slice(PRO_BLOCK * blk, PRO_BLOCK * blk + r.shape[0])
            raw["x"][n, s] = r
            if want_exact:
                exact["x"][n, s] = e

    jobs = [(n, blk) for n in range(w.B) for blk in range(nblk)]
    parts = [jobs[i::threads] for i in range(min(threads, len(jobs)))]
    if parts:
        with ThreadPoolExecutor(max_workers=len(parts)) as ex:
            list(ex.map(fill, parts))
    for nm, x in prologue_theta(w).items():
        raw[nm], exact[nm] = store(x, BF16)
    return {"raw": raw, "exact": exact}


def prologue_case(B: int, T: int, Dm: int, H: int, d: int, gate: bool = True, eta_base: float = 1.0 / 64.0,
                  seed: int = 11) -> tuple:
    """A small ad-hoc prologue case with the same distributions (parity tests)."""
    w = PrologueWorkload(f"prologue_case_B{B}_T{T}_Dm{Dm}_H{H}_d{d}", B, T, Dm, H, d, gate, eta_base, seed)
    return w, make_prologue_inputs(w, threads=1)
