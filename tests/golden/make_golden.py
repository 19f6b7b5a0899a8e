"""Write tests/golden/oracle_small.json: a regression fixture of the oracle.

The paper prints formulas but no worked numbers, so no fixture here comes
from the pages.  This fixture records the float64 oracle's outputs on three
tiny seeded cases (linear, LN+residual, MLP) so that an unintended change to
the oracle's arithmetic shows up as a test failure.  It calls only the oracle
and the seeded input generators.  Re-run it only together with a commit that
names the passage justifying the change.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import oracle as O  # noqa: E402
from test_sequence_layers_head_b200 import workloads as WL  # noqa: E402

CASES = {
    "linear": dict(kind="linear", B=1, H=2, T=40, d=8, b=16, io_dtype=WL.BF16, eta_mode="sigmoid"),
    "ln": dict(kind="ln", B=1, H=2, T=40, d=8, b=16, io_dtype=WL.BF16, eta_mode="sigmoid"),
    "mlp": dict(kind="mlp", B=1, H=1, T=40, d=4, b=16, io_dtype=WL.BF16, eta_mode="const", eta_const=0.05),
}


def run_case(name):
    c = CASES[name]
    inp = WL.random_case(seed=99, **c)
    e = inp.exact
    if c["kind"] == "mlp":
        Z, W1, c1, W2, c2 = O.mlp_forward(e["Q"], e["K"], e["V"], e["eta"], e["W1"], e["c1"], e["W2"], e["c2"],
                                          c["b"])
        return {"Z": Z.ravel().tolist(), "W1": W1.ravel().tolist(), "W2": W2.ravel().tolist(),
                "c1": c1.ravel().tolist(), "c2": c2.ravel().tolist()}
    ln = c["kind"] == "ln"
    kw = dict(c0=e["c0"], gamma=e["gamma"], beta=e["beta"]) if ln else {}
    Z, W, cc = O.linear_forward(e["Q"], e["K"], e["V"], e["eta"], e["W0"], c["b"], use_ln=ln, **kw)
    out = {"Z": Z.ravel().tolist(), "W": W.ravel().tolist()}
    if ln:
        out["c"] = cc.ravel().tolist()
    return out


if __name__ == "__main__":
    data = {"note": "regression fixture of the float64 oracle; see make_golden.py",
            "cases": CASES, "outputs": {k: run_case(k) for k in CASES}}
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(data, f)
    print("written")
