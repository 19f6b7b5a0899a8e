"""Failure detection on the GPU without a fault: every device-side wait in the
tensor-core kernels is bounded.  The test hook TTT_FLAG_TEST_STALL makes the
MMA issuer wait on an mbarrier that nothing arrives on; the wait runs out
after wait_timeout_ms, the kernel records the timeout, stops issuing work,
drains what it issued and returns.  The host reads TTT_ERR_TIMEOUT from
ttt_last_device_status(), and the context stays usable: the next call
succeeds and matches the oracle."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from test_sequence_layers_head_b200 import workloads as WL
from tests.gpu_util import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["linear", "ln", "mlp", "mlp_ln"])
def test_stalled_wait_reports_timeout_and_context_survives(ttt_lib, kind):
    mlp = kind.startswith("mlp")
    inp = WL.random_case("mlp" if mlp else kind, 1, 3, 128, 64, 16, eta_mode="const" if mlp else "sigmoid",
                         eta_const=1 / 64, seed=71)
    d = {k: to_dev(v) for k, v in inp.raw.items()}
    rng = np.random.default_rng(72)
    gr, ge = WL.store(1 + rng.standard_normal((3, 64)) * 0.14, WL.F32)
    br, be = WL.store(rng.standard_normal((3, 64)) * 0.14, WL.F32)
    mln = dict(use_ln=True, gamma=to_dev(gr), beta=to_dev(br)) if kind == "mlp_ln" else {}
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK

    def run(flags):
        if mlp:
            return ttt_lib.mlp_forward(d["Q"], d["K"], d["V"], d["eta"], d["W1"], d["c1"], d["W2"], d["c2"], 16,
                                       flags=flags, wait_timeout_ms=300, **mln)
        ln = kind == "ln"
        kw = dict(c0=d["c0"], gamma=d["gamma"], beta=d["beta"]) if ln else {}
        return ttt_lib.linear_forward(d["Q"], d["K"], d["V"], d["eta"], d["W0"], 16, use_ln=ln, flags=flags,
                                      wait_timeout_ms=300, **kw)

    run(ttt_lib.FLAG_TEST_STALL)
    assert ttt_lib.last_device_status() == ttt_lib.TTT_ERR_TIMEOUT
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK        # the status word was cleared
    out = run(0)
    torch.cuda.synchronize()
    assert ttt_lib.last_device_status() == ttt_lib.TTT_OK
    e = inp.exact
    if mlp:
        kw = dict(use_ln=True, gamma=ge, beta=be) if kind == "mlp_ln" else {}
        ref = O.mlp_forward(e["Q"], e["K"], e["V"], e["eta"], e["W1"], e["c1"], e["W2"], e["c2"], 16, **kw)
    else:
        ln = kind == "ln"
        kw = dict(c0=e["c0"], gamma=e["gamma"], beta=e["beta"]) if ln else {}
        ref = O.linear_forward(e["Q"], e["K"], e["V"], e["eta"], e["W0"], 16, use_ln=ln, **kw)
    assert_close("Z after recovery", to_host(out[0]), ref[0], WL.BF16)
