"""Benchmark of the TTT inner-loop forward on B200.

Default workload: the long-context TTT-Linear prefill (B=16 sequences,
H=32 heads, d=64, T=32768 tokens, mini-batch b=16, bf16 Q/K/V/Z, fp32
state), the largest single-GPU configuration.  One step = one call of
ttt_linear_forward over the whole batch (every row of the hot path:
TMA loads, the key-side residual, the causal outputs, the in-place state
update and the final-state store).

Prints ONE JSON line:
  value       prefill tokens/s per layer (B*T / time, all heads), summed over
              ranks (weak scaling: every rank runs its own B=16 batch)
  roofline    the prefill kernel against HBM bandwidth (algorithmic bytes:
              Q, K, V, Z bf16 + eta fp32 per token-head, W0 per head, W_out per
              unit), achieved from CUDA events around each launch
  cpu_baseline  the float64 oracle on a bounded sample, host cores
  e2e         the same metric through the public API with pinned host
              buffers (H2D of Q/K/V/eta, D2H of Z and the final state inside
              the timed region)
  decode      the 1024-step decode phase of the same workload (CUDA graph)
  rows        the other workloads measured the same way, the LN+residual and
              MLP decode steps, the TTT-MLP with LN+residual and the
              backward passes (informational)

--impl reference times the float64 oracle (the reference arm) on a bounded
sample of the same workload.  --b-sweep prints the mini-batch size study
(state and outputs time per b), --train one TTT-Linear training step
(forward writing the batch-start states, then the backward) and --prologue
the fused prologue (the views and the learning-rate gate from the layer
input, alone and followed by the forward) instead of the benchmark line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from test_sequence_layers_head_b200 import workloads as WL  # noqa: E402

METRIC = "TTT layer tokens/sec (prefill, per B200) and % of dual-form roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "linear_B16_H32_T32768_decode1024"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------------------
# algorithmic work (per launch)
# ---------------------------------------------------------------------------

def algorithmic_bytes(w: WL.Workload) -> int:
    """Bytes a launch must move: Q, K, V read and Z written (io dtype), eta
    read (fp32, when per-token), the initial state read once per head and the
    final state written once per unit."""
    io = 2 if w.io_dtype == WL.BF16 else 4
    th = w.units * w.T
    per_tok = 4 * w.d * io + (4 if w.eta_mode == "sigmoid" else 0)
    if w.kind == "mlp":
        state = 2 * w.d * w.hidden + w.hidden + w.d
    else:
        state = w.d * w.d + (w.d if w.kind == "ln" else 0)
    return th * per_tok + 4 * state * (w.H + w.units)


def algorithmic_flops(w: WL.Workload) -> int:
    """Dual-form flops per token-head: linear 6 d^2 + 4 b d (key residual,
    outputs, state update, causal term); LN adds the causal +1 term; MLP is
    the two-layer version with hidden m = 4d."""
    d, b, m = w.d, w.b, w.hidden
    if w.kind == "mlp":
        per = 2 * d * m * 2 + 2 * m * d * 2 + 2 * m * d + 2 * d * m + 2 * b * d + 2 * b * m + 2 * b * m + 2 * b * d
    else:
        per = 6 * d * d + 4 * b * d
    return w.units * w.T * per


def dominant_kernel(w):
    """(kernel name, source file under csrc/) of the one kernel a step of workload w launches."""
    if w.io_dtype != WL.BF16 or w.d != 64 or w.b != 16:
        return ("simt_mlp_kernel" if w.kind == "mlp" else "simt_linear_kernel"), "simt.cuh"
    if w.kind == "mlp":
        return "mlp_tc_kernel", "mlp_tc.cuh"
    upc = 1 if w.B * w.H <= 148 else 2   # the library's layout choice (one unit per CTA up to the SM count)
    return f"linear_frag_kernel<{int(w.kind == 'ln')}, {upc}>", "linear_frag.cuh"


def recorded_traffic(kernel: str, src: str):
    """DRAM bytes per launch recorded from an ncu capture in profiles/traffic.json,
    or None when the kernel source changed since the capture."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[kernel]
        sha = hashlib.sha256(open(os.path.join(ROOT, "test_sequence_layers_head_b200", "csrc", src), "rb").read())
        if sha.hexdigest()[:16] == rec["src_sha256_16"]:
            return rec["bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        pass
    return None


def tokens(w: WL.Workload) -> int:
    return w.B * w.T


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r[0] for r in rows if r[2] > 200.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def shard_units(total_sequences: int, world: int, rank: int):
    """Sequences owned by `rank` when `total_sequences` are split evenly
    (used when a fixed global batch is spread over ranks)."""
    per = (total_sequences + world - 1) // world
    lo = min(rank * per, total_sequences)
    return lo, min(lo + per, total_sequences)


def max_over_ranks(values, dist, device="cpu"):
    """Element-wise maximum of per-rank timings (the slowest rank decides)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def to_dev(raw, torch):
    if raw.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(raw)).cuda()


def call_forward(ttt, w, dev, out):
    if w.kind == "mlp":
        return ttt.mlp_forward(dev["Q"], dev["K"], dev["V"], dev.get("eta"), dev["W1"], dev["c1"], dev["W2"],
                               dev["c2"], w.b, eta_const=w.eta_const, Z=out["Z"], W1_out=out["W1"],
                               c1_out=out["c1"], W2_out=out["W2"], c2_out=out["c2"])
    ln = w.kind == "ln"
    kw = dict(c0=dev["c0"], gamma=dev["gamma"], beta=dev["beta"], eps=w.ln_eps) if ln else {}
    return ttt.linear_forward(dev["Q"], dev["K"], dev["V"], dev.get("eta"), dev["W0"], w.b, eta_const=w.eta_const,
                              use_ln=ln, Z=out["Z"], W_out=out["W"], c_out=out.get("c"), **kw)


def alloc_outputs(w, torch):
    B, H, T, d = w.B, w.H, w.T, w.d
    io = torch.bfloat16 if w.io_dtype == WL.BF16 else torch.float32
    out = {"Z": torch.empty((B, H, T, d), dtype=io, device="cuda")}
    if w.kind == "mlp":
        m = w.hidden
        out.update(W1=torch.empty((B, H, d, m), device="cuda"), c1=torch.empty((B, H, m), device="cuda"),
                   W2=torch.empty((B, H, m, d), device="cuda"), c2=torch.empty((B, H, d), device="cuda"))
    else:
        out["W"] = torch.empty((B, H, d, d), device="cuda")
        if w.kind == "ln":
            out["c"] = torch.empty((B, H, d), device="cuda")
    return out


def device_inputs(w, torch, threads):
    inp = WL.make_inputs(w, want_exact=False, threads=threads)
    dev = {k: to_dev(v, torch) for k, v in inp.raw.items()}
    if w.eta_mode == "const":
        dev.pop("eta")
    return inp, dev


def time_launches(torch, fn, steps, warmup, flush=None):
    """Per-launch CUDA-event durations (ms)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush()
        evs[i][0].record(st)
        fn()
        evs[i][1].record(st)
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in evs]
    return per


def measure_decode(ttt, w, torch, steps=3):
    """Decode phase: w.decode_steps single-token steps for all units, captured
    in one CUDA graph; returns per-step time and roofline numbers."""
    B, H, d = w.B, w.H, w.d
    g = np.random.default_rng(0)
    W = torch.tensor((g.standard_normal((B, H, d, d)) / np.sqrt(d)).astype(np.float32), device="cuda")
    n = w.decode_steps
    toks = [WL.make_decode_tokens(w, s)[0] for s in range(n)]
    q = torch.stack([to_dev(t["q"], torch) for t in toks])
    k = torch.stack([to_dev(t["k"], torch) for t in toks])
    v = torch.stack([to_dev(t["v"], torch) for t in toks])
    eta = torch.stack([to_dev(t["eta"], torch) for t in toks])
    z = torch.empty_like(q)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        for s in range(3):   # warm-up outside the graph
            ttt.linear_decode_step(W, q[s], k[s], v[s], eta[s], z=z[s], stream=st)
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cs = torch.cuda.current_stream()
        for s in range(n):
            ttt.linear_decode_step(W, q[s], k[s], v[s], eta[s], z=z[s], stream=cs)
    graph.replay()
    torch.cuda.synchronize()
    per = time_launches(torch, graph.replay, steps, 1)
    ms = statistics.median(per)
    io = 2
    bytes_step = w.units * (2 * d * d * 4 + 4 * d * io + 4)
    del graph
    return {"steps_per_graph": n, "us_per_step": 1000.0 * ms / n, "tokens_per_s": w.B * n / (ms / 1000.0),
            "bytes_per_step": bytes_step, "achieved_gbs": bytes_step * n / (ms / 1000.0) / 1e9,
            "note": "W (8.4 MB) stays L2-resident across steps; GB/s is against HBM peak for reference",
            "gpu_launches_per_graph": n}


def measure_decode_variant(ttt, torch, kind, B, H, d=64, n=1024, steps=3):
    """LN+residual or MLP decode: n single-token steps for B x H units from a
    random state, captured in one CUDA graph (informational; parity lives in
    the tests).  Returns per-step time and the state bytes each step moves."""
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    f32 = dict(device="cuda", dtype=torch.float32)
    units = B * H
    q = (torch.randn(n, B, H, d, generator=g, **f32) / 8).bfloat16()
    k = (torch.randn(n, B, H, d, generator=g, **f32) / 8).bfloat16()
    v = (torch.randn(n, B, H, d, generator=g, **f32) / 8).bfloat16()
    eta = torch.sigmoid(torch.randn(n, B, H, generator=g, **f32)) / 64
    z = torch.empty_like(q)
    if kind == "ln":
        W = torch.randn(B, H, d, d, generator=g, **f32) / 8
        c = torch.zeros(B, H, d, **f32)
        gam = 1 + torch.randn(H, d, generator=g, **f32) * 0.14
        bet = torch.randn(H, d, generator=g, **f32) * 0.14

        def step(s, st):
            ttt.linear_decode_step(W, q[s], k[s], v[s], eta[s], z=z[s], use_ln=True, c=c, gamma=gam, beta=bet,
                                   stream=st)
        state_bytes = units * (2 * d * d * 4 + 2 * d * 4)
    else:
        m = 4 * d
        W1 = torch.randn(B, H, d, m, generator=g, **f32) / 8
        c1 = torch.zeros(B, H, m, **f32)
        W2 = torch.randn(B, H, m, d, generator=g, **f32) / 16
        c2 = torch.zeros(B, H, d, **f32)

        def step(s, st):
            ttt.mlp_decode_step(W1, c1, W2, c2, q[s], k[s], v[s], eta[s], z=z[s], stream=st)
        state_bytes = units * (2 * 2 * d * m * 4 + 2 * (m + d) * 4)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        for s in range(3):
            step(s, st)
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cs = torch.cuda.current_stream()
        for s in range(n):
            step(s, cs)
    graph.replay()
    torch.cuda.synchronize()
    per = time_launches(torch, graph.replay, steps, 1)
    ms = statistics.median(per)
    del graph
    bytes_step = state_bytes + units * (4 * d * 2 + 4)
    return {"B": B, "H": H, "d": d, "steps_per_graph": n, "us_per_step": 1000.0 * ms / n,
            "tokens_per_s": B * n / (ms / 1000.0), "bytes_per_step": bytes_step,
            "achieved_gbs": bytes_step * n / (ms / 1000.0) / 1e9,
            "note": "state stays L2-resident across steps; GB/s is against HBM peak for reference"}


def measure_backward(ttt, torch, threads, name="linear_B8_H12_T2048"):
    """Outer-loop backward of TTT-Linear on a workload's shapes: the forward
    that also writes the batch-start states, then the backward with random
    upstream gradients (informational; parity lives in the tests)."""
    w = WL.WORKLOADS[name]
    _, dev = device_inputs(w, torch, threads)
    B, H, T, d = w.B, w.H, w.T, w.d
    states = torch.empty((B, H, T // w.b, d, d), device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(2)
    dZ = torch.randn(B, H, T, d, generator=g, device="cuda").to(dev["Q"].dtype)
    dW = torch.randn(B, H, d, d, generator=g, device="cuda")
    outs = [torch.empty_like(dev["Q"]) for _ in range(3)]
    deta = torch.empty((B, H, T), device="cuda")
    dW0 = torch.empty((B, H, d, d), device="cuda")
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")

    def fwd():
        ttt.linear_forward(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], w.b, W_states=states)

    def bwd():
        ttt.linear_backward(dev["Q"], dev["K"], dev["V"], dev["eta"], states, w.b, dZ=dZ, dW_out=dW,
                            dQ=outs[0], dK=outs[1], dV=outs[2], deta=deta, dW0=dW0)
    ms_f = statistics.median(time_launches(torch, fwd, 5, 2, flush=lambda: flush_buf.zero_()))
    ms_b = statistics.median(time_launches(torch, bwd, 5, 2, flush=lambda: flush_buf.zero_()))
    io = dev["Q"].element_size()
    units = B * H
    bytes_b = units * (T * d * io * 7 + T * 8 + (T // w.b) * d * d * 4 + 3 * d * d * 4)
    hbm, _, _ = measured_peaks()
    return {"workload": name, "forward_with_states_ms": ms_f, "backward_ms": ms_b,
            "tokens_per_s_backward": tokens(w) / (ms_b / 1000.0),
            "backward_bytes": bytes_b, "backward_hbm_frac": bytes_b / (ms_b / 1000.0) / 1e9 / hbm,
            "kernel": "mma_linear_backward_kernel (mma.sync, bf16 operands, fp32 accumulation)"}


def measure_ln_backward(ttt, torch, threads, T=2048):
    """Outer-loop backward of the LN+residual TTT-Linear (fp32 CUDA-core kernels:
    the forward writing W_states and c_states, then the backward) on the LN
    workload's shapes at a shorter T (informational)."""
    w = WL.scaled(WL.WORKLOADS["ln_B4_H32_T8192"], T=T)
    _, dev = device_inputs(w, torch, threads)
    B, H, d = w.B, w.H, w.d
    nb = T // w.b
    states = torch.empty((B, H, nb, d, d), device="cuda")
    cst = torch.empty((B, H, nb, d), device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(4)
    dZ = torch.randn(B, H, T, d, generator=g, device="cuda").to(dev["Q"].dtype)
    dW = torch.randn(B, H, d, d, generator=g, device="cuda")
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")
    ln = dict(use_ln=True, gamma=dev["gamma"], beta=dev["beta"], eps=w.ln_eps)

    def fwd():
        ttt.linear_forward(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], w.b, c0=dev["c0"], W_states=states,
                           c_states=cst, **ln)

    def bwd():
        ttt.linear_backward(dev["Q"], dev["K"], dev["V"], dev["eta"], states, w.b, dZ=dZ, dW_out=dW, c_states=cst,
                            **ln)
    ms_f = statistics.median(time_launches(torch, fwd, 3, 1, flush=lambda: flush_buf.zero_()))
    ms_b = statistics.median(time_launches(torch, bwd, 3, 1, flush=lambda: flush_buf.zero_()))
    return {"workload": w.name + f" (T={T})", "forward_with_states_ms": ms_f, "backward_ms": ms_b,
            "tokens_per_s_backward": tokens(w) / (ms_b / 1000.0),
            "kernel": "simt_ln_backward_kernel (fp32 CUDA cores)"}


def measure_mlp_ln(ttt, torch, threads):
    """TTT-MLP with LN+residual on the output layer (the tensor-core MLP kernel's
    LN variant) on the MLP workload's shapes (informational)."""
    w = WL.WORKLOADS["mlp_B2_H32_T8192"]
    _, dev = device_inputs(w, torch, threads)
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    gam = 1 + 0.14 * torch.randn(w.H, w.d, generator=g, device="cuda")
    bet = 0.14 * torch.randn(w.H, w.d, generator=g, device="cuda")
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")

    def fn():
        ttt.mlp_forward(dev["Q"], dev["K"], dev["V"], dev.get("eta"), dev["W1"], dev["c1"], dev["W2"], dev["c2"],
                        w.b, eta_const=w.eta_const, use_ln=True, gamma=gam, beta=bet)
    ms = statistics.median(time_launches(torch, fn, 5, 2, flush=lambda: flush_buf.zero_()))
    _, tflops, _ = measured_peaks()
    return {"ms": ms, "tokens_per_s": tokens(w) / (ms / 1000.0),
            "tensor_frac": algorithmic_flops(w) / (ms / 1000.0) / 1e12 / tflops,
            "kernel": "mlp_tc_kernel<true> (tcgen05 + mma.sync)"}


def measure_e2e_chunked(ttt, w, inp, torch, steps, chunks=8):
    """The public API on pinned host buffers, streamed along the sequence:
    the T tokens go through `chunks` calls of ttt_linear_forward, each
    resuming from the previous call's final state (per-sequence W0), so that
    the host-to-device copy of chunk k+1, the forward of chunk k and the
    device-to-host copy of chunk k-1 overlap (copy engines in both directions
    and the SMs).  Every byte of the step's inputs crosses H2D and every byte
    of Z and the final state crosses D2H inside the timed region."""
    from cuda.bindings import runtime as cudart

    B, H, T, d = w.B, w.H, w.T, w.d
    Tc = T // chunks
    units = B * H
    host = {}
    for k_, v_ in inp.raw.items():
        a = np.ascontiguousarray(v_)
        th = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        if a.dtype == np.uint16:
            th = th.view(torch.bfloat16)
        host[k_] = th.pin_memory()
    eta_on = w.eta_mode != "const"
    if not eta_on:
        host.pop("eta")
    zh = torch.empty((B, H, T, d), dtype=torch.bfloat16).pin_memory()
    wh = torch.empty((B, H, d, d), dtype=torch.float32).pin_memory()
    W0 = torch.empty_like(host["W0"], device="cuda")
    big = ["Q", "K", "V"]
    din = [{k_: torch.empty((B, H, Tc, d), dtype=torch.bfloat16, device="cuda") for k_ in big} for _ in range(2)]
    if eta_on:
        for b_ in range(2):
            din[b_]["eta"] = torch.empty((B, H, Tc), dtype=torch.float32, device="cuda")
    zd = [torch.empty((B, H, Tc, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    ws = [torch.empty((B, H, d, d), dtype=torch.float32, device="cuda") for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    H2D, D2H = cudart.cudaMemcpyKind.cudaMemcpyHostToDevice, cudart.cudaMemcpyKind.cudaMemcpyDeviceToHost

    def copy2d(dst, dpitch, src, spitch, width, height, kind, stream):
        err, = cudart.cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, height, kind, stream.cuda_stream)
        if err != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaMemcpy2DAsync: {err}")

    def step():
        main = torch.cuda.current_stream()
        for s_ in (s_in, s_cmp, s_out):
            s_.wait_stream(main)
        e_in = [torch.cuda.Event() for _ in range(chunks)]
        e_cmp = [torch.cuda.Event() for _ in range(chunks)]
        e_out = [torch.cuda.Event() for _ in range(chunks)]
        with torch.cuda.stream(s_in):
            W0.copy_(host["W0"], non_blocking=True)
        for c in range(chunks):
            bi = c & 1
            if c >= 2:
                s_in.wait_event(e_cmp[c - 2])            # the forward that read this buffer is done
            for k_, t_ in din[bi].items():
                hsrc, es = host[k_], t_.element_size()
                row = Tc * d * es if k_ != "eta" else Tc * es
                pitch = T * d * es if k_ != "eta" else T * es
                copy2d(t_.data_ptr(), row, hsrc.data_ptr() + c * row, pitch, row, units, H2D, s_in)
            e_in[c].record(s_in)
            s_cmp.wait_event(e_in[c])
            if c >= 2:
                s_cmp.wait_event(e_out[c - 2])           # Z of this buffer has left the device
            src_w = W0 if c == 0 else ws[(c - 1) & 1]
            ttt.linear_forward(din[bi]["Q"], din[bi]["K"], din[bi]["V"], din[bi].get("eta"), src_w, w.b,
                               eta_const=w.eta_const, Z=zd[bi], W_out=ws[c & 1], stream=s_cmp)
            e_cmp[c].record(s_cmp)
            s_out.wait_event(e_cmp[c])
            row = Tc * d * 2
            copy2d(zh.data_ptr() + c * row, T * d * 2, zd[bi].data_ptr(), row, row, units, D2H, s_out)
            e_out[c].record(s_out)
        with torch.cuda.stream(s_out):
            wh.copy_(ws[(chunks - 1) & 1], non_blocking=True)
        for s_ in (s_in, s_cmp, s_out):
            main.wait_stream(s_)

    per = time_launches(torch, step, steps, 1)
    ms = statistics.mean(per)
    h2d = sum(v_.numel() * v_.element_size() for v_ in host.values())
    d2h = zh.numel() * 2 + wh.numel() * 4
    del din, zd, ws, host, zh, wh
    return {"value": tokens(w) / (ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms, "chunks": chunks,
            "pipeline": "per chunk of T/8 tokens: H2D (Q, K, V, eta) | forward from the previous chunk's state | "
                        "D2H (Z); three streams, double-buffered"}


def measure_e2e(ttt, w, inp, torch, steps):
    """The public API on pinned host buffers: H2D inputs, forward, D2H of Z
    and the final state, all inside the timed region, every step."""
    if w.kind == "linear" and w.io_dtype == WL.BF16 and w.T % (8 * 2 * w.b) == 0:
        return measure_e2e_chunked(ttt, w, inp, torch, steps)
    host = {}
    for k_, v_ in inp.raw.items():
        a = np.ascontiguousarray(v_)
        th = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        if a.dtype == np.uint16:
            th = th.view(torch.bfloat16)
        host[k_] = th.pin_memory()
    if w.eta_mode == "const":
        host.pop("eta")
    dev = {k_: torch.empty_like(v_, device="cuda") for k_, v_ in host.items()}
    out = alloc_outputs(w, torch)
    out_host = {k_: torch.empty_like(v_, device="cpu").pin_memory() for k_, v_ in out.items()}
    h2d = sum(v_.numel() * v_.element_size() for v_ in host.values())
    d2h = sum(v_.numel() * v_.element_size() for v_ in out.values())

    def step():
        for k_ in host:
            dev[k_].copy_(host[k_], non_blocking=True)
        call_forward(ttt, w, dev, out)
        for k_ in out:
            out_host[k_].copy_(out[k_], non_blocking=True)

    per = time_launches(torch, step, steps, 1)
    ms = statistics.mean(per)
    del dev, out, host, out_host
    return {"value": tokens(w) / (ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms}


def cpu_baseline(w, sample_sequences=4):
    """The float64 oracle on a bounded sample: `sample_sequences` sequences
    (all heads, full length) of the workload, on every host core."""
    from oracle import oracle as O
    ws = WL.scaled(w, B=sample_sequences)
    inp = WL.make_inputs(ws, threads=O.default_threads())
    e = inp.exact
    cores = O.default_threads()
    t0 = time.perf_counter()
    if w.kind == "mlp":
        O.mlp_forward(e["Q"], e["K"], e["V"], np.full(e["eta"].shape, w.eta_const), e["W1"], e["c1"], e["W2"],
                      e["c2"], w.b, threads=cores)
    else:
        ln = w.kind == "ln"
        kw = dict(c0=e["c0"], gamma=e["gamma"], beta=e["beta"], eps=w.ln_eps) if ln else {}
        eta = e["eta"] if w.eta_mode == "sigmoid" else np.full(e["eta"].shape, w.eta_const)
        O.linear_forward(e["Q"], e["K"], e["V"], eta, e["W0"], w.b, use_ln=ln, threads=cores, **kw)
    dt = time.perf_counter() - t0
    return {"value": sample_sequences * w.T / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{sample_sequences} of {w.B} sequences x {w.H} heads x T={w.T} (float64 primal, OpenMP)",
            "seconds": dt}


def run_ours(args):
    import torch
    from test_sequence_layers_head_b200 import ttt

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    w = WL.WORKLOADS[args.workload]
    if args.T:
        w = WL.scaled(w, T=args.T)
    threads = max(1, len(os.sched_getaffinity(0)) // max(1, ws))
    inp, dev = device_inputs(w, torch, threads)
    out = alloc_outputs(w, torch)
    fn = lambda: call_forward(ttt, w, dev, out)   # noqa: E731
    fn()
    torch.cuda.synchronize()
    assert ttt.last_device_status() == ttt.TTT_OK
    hbm, tflops, peak_src = measured_peaks()

    def barrier():
        if dist is not None:
            dist.barrier()

    with ClockSampler(local) as clk:
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        st = torch.cuda.current_stream()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        t0.record(st)
        for i in range(args.steps):
            evs[i][0].record(st)
            fn()
            evs[i][1].record(st)
        t1.record(st)
        torch.cuda.synchronize()
        barrier()
    clocks = clk.summary()
    total_ms = t0.elapsed_time(t1)
    launch_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms, mean_launch = max_over_ranks([total_ms, statistics.mean(launch_ms)], dist, "cuda")
    status = ttt.last_device_status()
    ms_step = total_ms / args.steps
    value = ws * tokens(w) / (ms_step / 1000.0)

    abytes = algorithmic_bytes(w)
    aflops = algorithmic_flops(w)
    if w.kind == "mlp":
        achieved = aflops / (mean_launch / 1000.0) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tflops, "unit": "TFLOP/s",
                "frac": achieved / tflops, "peak_source": peak_src}
    else:
        achieved = abytes / (mean_launch / 1000.0) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_source": peak_src}
    kname, ksrc = dominant_kernel(w)
    roof.update({"kernel": kname,
                 "algorithmic_bytes_per_launch": abytes, "algorithmic_flops_per_launch": aflops,
                 "mean_launch_ms": mean_launch,
                 "traffic": args.traffic if args.traffic is not None else (
                     recorded_traffic(kname, ksrc) if (w.name == DEFAULT_WORKLOAD and not args.T) else None)})
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.io_dtype == WL.BF16 else "f32",
            "data": "synthetic (seeded PCG64 Gaussian inputs with the workload's distributions)",
            "config": {"workload": w.name, "kind": w.kind, "B_per_gpu": w.B, "H": w.H, "T": w.T, "d": w.d,
                       "b": w.b, "global_batch": w.B * ws, "parallelism": f"replicas x{ws} (units sharded, no collective)",
                       "l2": f"inputs larger than L2 ({abytes / 1e9:.2f} GB per step)"},
            "roofline": roof, "clocks": clocks, "gpu_launches": args.steps, "device_status": status}
    if rank == 0 and not args.no_extras:
        line["e2e"] = measure_e2e(ttt, w, inp, torch, steps=args.e2e_steps)
        if w.decode_steps:
            line["decode"] = measure_decode(ttt, w, torch)
        if not args.no_rows:
            line["rows"] = measure_rows(ttt, torch, threads)
            line["rows"]["decode_ln_B4_H32"] = measure_decode_variant(ttt, torch, "ln", 4, 32)
            line["rows"]["decode_mlp_B2_H32"] = measure_decode_variant(ttt, torch, "mlp", 2, 32)
            line["rows"]["backward_linear_B8_H12_T2048"] = measure_backward(ttt, torch, threads)
            line["rows"]["mlp_ln_B2_H32_T8192"] = measure_mlp_ln(ttt, torch, threads)
            line["rows"]["backward_ln_B4_H32_T2048"] = measure_ln_backward(ttt, torch, threads)
        line["cpu_baseline"] = cpu_baseline(w)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure_rows(ttt, torch, threads):
    """The other workloads, each timed over a few launches with an L2 flush
    between launches (informational; parity lives in the tests)."""
    res = {}
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")
    hbm, tflops, _ = measured_peaks()
    for name in ("linear_B8_H12_T2048", "ln_B4_H32_T8192", "mlp_B2_H32_T8192", "linear_d16_T256_f32"):
        w = WL.WORKLOADS[name]
        _, dev = device_inputs(w, torch, threads)
        out = alloc_outputs(w, torch)
        per = time_launches(torch, lambda: call_forward(ttt, w, dev, out), 5, 2, flush=lambda: flush_buf.zero_())
        ms = statistics.median(per)
        r = {"ms": ms, "tokens_per_s": tokens(w) / (ms / 1000.0),
             "hbm_frac": algorithmic_bytes(w) / (ms / 1000.0) / 1e9 / hbm,
             "tensor_frac": algorithmic_flops(w) / (ms / 1000.0) / 1e12 / tflops}
        res[name] = r
        del dev, out
    return res


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    w = WL.WORKLOADS[args.workload]
    if args.T:
        w = WL.scaled(w, T=args.T)
    # the sample (generated once): sequence 0, one head per host core (its first heads are the
    # workload's own), so every step keeps all cores busy and takes a fraction of a second
    from oracle import oracle as O
    cores = O.default_threads()
    heads = max(1, min(w.H, cores))
    sample = WL.scaled(w, B=1, H=heads)
    e = WL.make_inputs(sample, threads=cores).exact
    eta = e["eta"] if w.eta_mode == "sigmoid" else np.full(e["eta"].shape, w.eta_const)

    def step():
        t0 = time.perf_counter()
        if w.kind == "mlp":
            O.mlp_forward(e["Q"], e["K"], e["V"], eta, e["W1"], e["c1"], e["W2"], e["c2"], w.b, threads=cores)
        else:
            ln = w.kind == "ln"
            kw = dict(c0=e["c0"], gamma=e["gamma"], beta=e["beta"], eps=w.ln_eps) if ln else {}
            O.linear_forward(e["Q"], e["K"], e["V"], eta, e["W0"], w.b, use_ln=ln, threads=cores, **kw)
        dt = time.perf_counter() - t0
        return {"value": w.T * heads / w.H / dt, "seconds": dt, "cores": cores}
    for _ in range(args.warmup):
        step()
    vals = [step() for _ in range(args.steps)]
    value = statistics.mean(v["value"] for v in vals)
    secs = sum(v["seconds"] for v in vals)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "kind": w.kind, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "b": w.b},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": f"each step: 1 of {w.B} sequences x {heads} of {w.H} heads x T={w.T} "
                                       f"(tokens/s scaled by {w.H}/{heads} heads)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_b_sweep(args):
    """Mini-batch size study (paper digest "论文速览 | TTT", section 5.3): forward
    time split into computing the state and computing the outputs, per b, on
    the fp32 CUDA-core kernel (every b <= 64; the state-only call passes
    Z = NULL), plus the tensor-core kernel at b = 16.  Prints one JSON line."""
    import torch
    from test_sequence_layers_head_b200 import ttt
    w = WL.WORKLOADS[args.workload if args.workload != DEFAULT_WORKLOAD else "linear_B8_H12_T2048"]
    if args.T:
        w = WL.scaled(w, T=args.T)
    threads = len(os.sched_getaffinity(0))
    _, dev = device_inputs(w, torch, threads)
    B, H, T, d = w.B, w.H, w.T, w.d
    Z = torch.empty_like(dev["Q"])
    W_out = torch.empty((B, H, d, d), device="cuda")
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")
    eta = dev.get("eta")

    def fwd(b, outputs, flags):
        ttt.linear_forward(dev["Q"], dev["K"], dev["V"], eta, dev["W0"], b, eta_const=w.eta_const, Z=Z, W_out=W_out,
                           outputs=outputs, flags=flags)
    rows = []
    for b in (1, 2, 4, 8, 16, 32, 64):
        if T % b:
            continue
        full = statistics.median(time_launches(torch, lambda: fwd(b, True, ttt.FLAG_FORCE_SIMT), 3, 1,
                                               flush=lambda: flush_buf.zero_()))
        state = statistics.median(time_launches(torch, lambda: fwd(b, False, ttt.FLAG_FORCE_SIMT), 3, 1,
                                                flush=lambda: flush_buf.zero_()))
        rows.append({"b": b, "forward_ms": full, "state_only_ms": state, "outputs_ms": full - state,
                     "tokens_per_s": tokens(w) / (full / 1000.0)})
    tc = statistics.median(time_launches(torch, lambda: fwd(16, True, 0), 5, 2, flush=lambda: flush_buf.zero_()))
    assert ttt.last_device_status() == ttt.TTT_OK
    print(json.dumps({"b_sweep": rows, "workload": w.name, "dtype": "bf16" if w.io_dtype == WL.BF16 else "f32",
                      "kernel": "fp32 CUDA-core forward (state only: Z = NULL)",
                      "tensor_core_b16_ms": tc, "tensor_core_b16_tokens_per_s": tokens(w) / (tc / 1000.0)}),
          flush=True)


def run_train(args):
    """One training step per timed step: TTT-Linear (no LN), or, on the LN and
    MLP workloads, TTT-Linear with LN+residual and TTT-MLP: the forward that
    writes the batch-start states, then the outer-loop backward with random
    upstream gradients.  Prints one JSON line (not the benchmark line)."""
    import torch
    from test_sequence_layers_head_b200 import ttt
    w = WL.WORKLOADS[args.workload if args.workload != DEFAULT_WORKLOAD else "linear_B8_H12_T2048"]
    if args.T:
        w = WL.scaled(w, T=args.T)
    _, dev = device_inputs(w, torch, len(os.sched_getaffinity(0)))
    B, H, T, d = w.B, w.H, w.T, w.d
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    dZ = torch.randn(B, H, T, d, generator=g, device="cuda").to(dev["Q"].dtype)
    eta = dev.get("eta")
    if w.kind == "mlp":
        m = w.hidden
        states = torch.empty((B, H, T // w.b, 2 * d * m + m + d), device="cuda")
        ln = {}
        if args.mlp_ln:
            # LN+residual on the output layer, gamma ~ 1 + N(0, .02), beta ~ N(0, .02) as for the LN workload
            g2 = torch.Generator(device="cuda")
            g2.manual_seed(6)
            ln = dict(use_ln=True, gamma=1 + 0.02 ** 0.5 * torch.randn(H, d, generator=g2, device="cuda"),
                      beta=0.02 ** 0.5 * torch.randn(H, d, generator=g2, device="cuda"))

        def step():
            ttt.mlp_forward(dev["Q"], dev["K"], dev["V"], eta, dev["W1"], dev["c1"], dev["W2"], dev["c2"], w.b,
                            eta_const=w.eta_const, W_states=states, **ln)
            ttt.mlp_backward(dev["Q"], dev["K"], dev["V"], eta, states, w.b, eta_const=w.eta_const, dZ=dZ,
                             want_deta=eta is not None, **ln)
    elif w.kind == "ln":
        states = torch.empty((B, H, T // w.b, d, d), device="cuda")
        cst = torch.empty((B, H, T // w.b, d), device="cuda")
        dW = torch.randn(B, H, d, d, generator=g, device="cuda")
        dc = torch.randn(B, H, d, generator=g, device="cuda")
        flags = ttt.FLAG_LN_MMA_TRAINING if args.ln_mma else 0
        ln = dict(use_ln=True, gamma=dev["gamma"], beta=dev["beta"], eps=w.ln_eps, flags=flags)

        def step():
            ttt.linear_forward(dev["Q"], dev["K"], dev["V"], eta, dev["W0"], w.b, eta_const=w.eta_const, c0=dev["c0"],
                               W_states=states, c_states=cst, **ln)
            ttt.linear_backward(dev["Q"], dev["K"], dev["V"], eta, states, w.b, eta_const=w.eta_const, dZ=dZ,
                                dW_out=dW, c_states=cst, dc_out=dc, **ln)
    else:
        states = torch.empty((B, H, T // w.b, d, d), device="cuda")
        dW = torch.randn(B, H, d, d, generator=g, device="cuda")

        def step():
            ttt.linear_forward(dev["Q"], dev["K"], dev["V"], eta, dev["W0"], w.b, eta_const=w.eta_const,
                               W_states=states)
            ttt.linear_backward(dev["Q"], dev["K"], dev["V"], eta, states, w.b, eta_const=w.eta_const, dZ=dZ,
                                dW_out=dW)
    per = time_launches(torch, step, args.steps, args.warmup)
    assert ttt.last_device_status() == ttt.TTT_OK
    ms = statistics.mean(per)
    kernels = "forward with states, then the backward"
    if w.kind == "ln":
        kernels += " (mma.sync LN kernels)" if args.ln_mma else " (fp32 CUDA-core LN kernels)"
    if w.kind == "mlp":
        kernels += " (LN+residual on the output layer, fp32 CUDA cores)" if args.mlp_ln else " (mma.sync)"
    print(json.dumps({"train_step_ms": ms, "tokens_per_s": tokens(w) / (ms / 1000.0), "workload": w.name,
                      "steps": args.steps, "warmup": args.warmup, "kernels": kernels}), flush=True)


def prologue_flops(w) -> int:
    """Algorithmic flops of one prologue launch: 2 Dm per output column per
    token, over the 3 H d view columns and the H gate columns."""
    return 2 * w.tokens * w.Dm * (3 * w.H * w.d + (w.H if w.gate else 0))


def prologue_bytes(w) -> int:
    """Algorithmic HBM bytes of one launch: x and the theta matrices read once
    (bf16), Q, K, V written once (bf16), eta written once (fp32)."""
    cols = 3 * w.H * w.d + (w.H if w.gate else 0)
    return 2 * w.tokens * w.Dm + 2 * cols * w.Dm + 2 * 3 * w.tokens * w.H * w.d + (4 * w.tokens * w.H if w.gate else 0)


def run_prologue(args):
    """The fused prologue (views and learning-rate gate from the layer input,
    ttt_qkv_prologue) on the two model widths, then the prologue followed by
    the TTT-Linear forward on the 32-head width.  Tensor-bound: the roofline
    is the dense bf16 peak.  Prints one JSON line (not the benchmark line)."""
    import torch
    from test_sequence_layers_head_b200 import ttt
    hbm, tflops, src = measured_peaks()
    threads = len(os.sched_getaffinity(0))
    flush_buf = torch.empty(256 * 1024 * 1024 // 4, device="cuda")
    rows = []
    for name, w in WL.PROLOGUE_WORKLOADS.items():
        inp = WL.make_prologue_inputs(w, want_exact=False, threads=threads)
        dev = {k: to_dev(v, torch) for k, v in inp["raw"].items()}
        B, H, T, d = w.B, w.H, w.T, w.d
        Q, K, V = (torch.empty((B, H, T, d), device="cuda", dtype=torch.bfloat16) for _ in range(3))
        eta = torch.empty((B, H, T), device="cuda")

        def pro():
            ttt.qkv_prologue(dev["x"], dev["theta_q"], dev["theta_k"], dev["theta_v"], dev["theta_lr"], w.eta_base,
                             d, Q=Q, K=K, V=V, eta=eta)
        with ClockSampler(torch.cuda.current_device()) as clk:
            per = time_launches(torch, pro, args.steps, args.warmup, flush=lambda: flush_buf.zero_())
        assert ttt.last_device_status() == ttt.TTT_OK
        ms = statistics.mean(per)
        ach = prologue_flops(w) / (ms / 1000.0) / 1e12
        row = {"workload": name, "ms": ms, "tokens_per_s": w.tokens / (ms / 1000.0),
               "roofline": {"bound": "tensor", "achieved": ach, "peak": tflops, "unit": "TFLOP/s",
                            "frac": ach / tflops, "peak_source": src},
               "hbm_gbs": prologue_bytes(w) / (ms / 1000.0) / 1e9, "clocks": clk.summary()}
        if H == 32:
            # the TTT-Linear forward on the views just computed (W0 per head)
            g = torch.Generator(device="cuda")
            g.manual_seed(3)
            W0 = torch.randn(H, d, d, generator=g, device="cuda") / d ** 0.5
            Z = torch.empty_like(Q)
            W_out = torch.empty((B, H, d, d), device="cuda")

            def layer():
                pro()
                ttt.linear_forward(Q, K, V, eta, W0, 16, Z=Z, W_out=W_out)
            per2 = time_launches(torch, layer, max(3, args.steps // 4), args.warmup, flush=lambda: flush_buf.zero_())
            assert ttt.last_device_status() == ttt.TTT_OK
            ms2 = statistics.mean(per2)
            row["with_linear_forward"] = {"ms": ms2, "tokens_per_s": w.tokens / (ms2 / 1000.0)}
        rows.append(row)
        del dev, Q, K, V, eta
        torch.cuda.empty_cache()
    print(json.dumps({"prologue": rows, "dtype": "bf16", "data": "synthetic",
                      "flush": "256 MiB L2 flush before every timed launch"}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # about 0.2 s of timed work on the default workload, so that the 50 ms clock samples see the load
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WL.WORKLOAD_ORDER)
    ap.add_argument("--T", type=int, default=0, help="override T (profiling a smaller case)")
    ap.add_argument("--no-extras", action="store_true", help="only the timed prefill (profiling)")
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch from an ncu capture of the current kernel build")
    ap.add_argument("--b-sweep", action="store_true",
                    help="mini-batch size study (state vs outputs time per b) instead of the benchmark line")
    ap.add_argument("--train", action="store_true",
                    help="training step (forward with states + backward; TTT-Linear, or TTT-MLP with the MLP "
                         "workload) instead of the benchmark line")
    ap.add_argument("--ln-mma", action="store_true",
                    help="with --train on the LN workload: the mma.sync LN training kernels")
    ap.add_argument("--mlp-ln", action="store_true",
                    help="with --train on the MLP workload: TTT-MLP with LN+residual on the output layer")
    ap.add_argument("--prologue", action="store_true",
                    help="the fused prologue (views and learning-rate gate from the layer input) instead of the "
                         "benchmark line")
    args = ap.parse_args()
    if args.prologue:
        run_prologue(args)
    elif args.train:
        run_train(args)
    elif args.b_sweep:
        run_b_sweep(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
