"""Plant mistakes in a copy of the oracle (on the CPU) and check that the pins
catch every one of them.

Each mutation is a one-line change of ``oracle/ttt_oracle.c`` compiled into a
temporary library; the pin suite (``test_oracle_pins.py``) is then run against
it in a subprocess and must fail.  This is evidence that the pins are strong
enough to detect the plausible mistakes a primal TTT implementation can make.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ttt_oracle.c")

MUTATIONS = {
    "update_sign": ("Wi[j] -= a * delta[j];", "Wi[j] += a * delta[j];"),
    "output_from_batch_start": ("linear_model_forward(d, q, Wc, cc,", "linear_model_forward(d, q, Ws, cs,"),
    "gradient_at_running_state": ("linear_model_delta(d, k, v, Ws, cs,", "linear_model_delta(d, k, v, Wc, cc,"),
    "ln_unbiased_variance": ("    var /= n;\n", "    var /= (n - 1);\n"),
    "ln_dropped_backward_term": ("r * (delta[j] - mean_g - xh[j] * mean_gx)", "r * (delta[j] - mean_g)"),
    "gelu_grad_missing_term": ("return Phi + x * phi;", "return Phi;"),
    "eta_ignored": ("const double et = eta[t];", "const double et = 0.1;"),
    "transposed_state": ("y[j] += xi * Wi[j];", "y[j] += xi * W[(size_t)j * n_out + i];"),
    "mlp_bias2_not_updated": ("c2c[j] -= et * e[j];", "(void)0;"),
    "mlp_w2_update_uses_prev_h": ("const double ah = et * hh[p];", "const double ah = et * a[p];"),
    "decode_output_before_update": (
        "        vec_mat(d, d, qu, Wu, z + (size_t)u * d);\n        free(e);",
        "        free(e);"),
}

# mistakes in the outer-loop backward, caught by its own pins
BACKWARD_MUTATIONS = {
    "bwd_eta_grad_sign": ("deta[t] = -ge;", "deta[t] = ge;"),
    "bwd_dq_from_batch_start": ("acc += dz[j] * Wt[(size_t)a * d + j];", "acc += dz[j] * Ws[(size_t)a * d + j];"),
    "bwd_missing_residual_path": ("dK[(size_t)t * d + a] = -eta[t] * acc1 + acc2;",
                                  "dK[(size_t)t * d + a] = -eta[t] * acc1;"),
    "bwd_state_grad_drops_residual": ("for (size_t x = 0; x < dd; ++x) D[x] += dWs[x];", "(void)dWs;"),
    "bwd_ln_explicit_r_term_dropped": ("for (int j = 0; j < d; ++j) dy[j] += dr * (-rr[li] * rr[li] * xt[j] / d);",
                                       "(void)dr;"),
    "bwd_ln_xhat_path_through_u_dropped": ("dxh[j] = -t1[j] * mgx[li] - gt[j] * mdux;", "dxh[j] = 0.0;"),
    "bwd_mlp_gelu_second_derivative_dropped": ("da[p] = dd1[p] * mm[p] * gelu_grad2(a[p]);", "da[p] = 0.0;"),
    "bwd_mlp_path_through_e_w2t_dropped": ("for (int p = 0; p < m; ++p) acc += dmv[p] * W2P(S)[(size_t)p * d + j];",
                                           "(void)dmv;"),
    "bwd_output_grad_dropped_from_state": (
        "            if (dz)\n                for (int a = 0; a < d; ++a)\n                    for (int j = 0; j < d; ++j) D[(size_t)a * d + j] += q[a] * dz[j];\n",
        ""),
}


def _build_mutant(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) >= 1, name
    mut = src.replace(old, new, 1)
    if name == "decode_output_before_update":
        mut = mut.replace("        vec_mat(d, d, ku, Wu, e);\n",
                          "        vec_mat(d, d, qu, Wu, z + (size_t)u * d);\n        vec_mat(d, d, ku, Wu, e);\n", 1)
    c = os.path.join(tmp, f"{name}.c")
    so = os.path.join(tmp, f"{name}.so")
    open(c, "w").write(mut)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-D_GNU_SOURCE", "-o", so, c,
                    "-lm"], check=True)
    return so


# mistakes in the MLP with LN+residual, caught by its own pins
MLP_LN_MUTATIONS = {
    "mlp_ln_residual_from_wrong_input": ("ln_residual_delta(d, k, v, y, gamma, beta, eps, e, xh);",
                                         "ln_residual_delta(d, v, v, y, gamma, beta, eps, e, xh);"),
    "mlp_ln_output_without_residual": ("z[j] = q[j] + gamma[j] * xh[j] + beta[j];",
                                       "z[j] = gamma[j] * xh[j] + beta[j];"),
}

# mistakes in the backward of TTT-MLP with LN+residual, caught by the backward pins
MLP_LN_BACKWARD_MUTATIONS = {
    "bwd_mlp_ln_delta2_path_through_w2_dropped": ("dd2[j] += acc;", "(void)acc;"),
    "bwd_mlp_ln_xhat_path_through_e_dropped": (
        "dxh[j] = -du[j] * MGX[li] - gamma[j] * e[j] * mdux + gamma[j] * de;",
        "dxh[j] = -du[j] * MGX[li] - gamma[j] * e[j] * mdux;"),
    "bwd_mlp_ln_explicit_r_term_dropped": (
        "for (int j = 0; j < d; ++j) dy[j] += dr * (-RR[li] * RR[li] * xh[j] / d);", "(void)dr;"),
}

# mistakes in the prologue (views and learning-rate gate), caught by its own pins
PROLOGUE_MUTATIONS = {
    "prologue_transposed_view": ("acc += row[k] * x[k];", "acc += theta[(size_t)k * H * d + h * d + j] * x[k];"),
    "prologue_head_stride": ("const size_t hs = (size_t)T * d;", "const size_t hs = (size_t)d;"),
    "prologue_k_from_q_view": ("project_view(H, d, Dm, theta_k, xt, K + o, hs);",
                               "project_view(H, d, Dm, theta_q, xt, K + o, hs);"),
    "prologue_gate_sign": ("eta_base * sigmoid(u);", "eta_base * sigmoid(-u);"),
    "prologue_gate_base_dropped": ("eta_base * sigmoid(u);", "sigmoid(u);"),
    "prologue_gate_head_row": ("const double *g = theta_lr + (size_t)h * Dm;", "const double *g = theta_lr;"),
}

PIN_FILES = {**{n: "test_oracle_pins.py" for n in MUTATIONS},
             **{n: "test_oracle_backward.py" for n in BACKWARD_MUTATIONS},
             **{n: "test_oracle_mlp_ln.py" for n in MLP_LN_MUTATIONS},
             **{n: "test_oracle_prologue.py" for n in PROLOGUE_MUTATIONS},
             **{n: "test_oracle_backward.py" for n in MLP_LN_BACKWARD_MUTATIONS}}
ALL_MUTATIONS = {**MUTATIONS, **BACKWARD_MUTATIONS, **MLP_LN_MUTATIONS, **PROLOGUE_MUTATIONS,
                 **MLP_LN_BACKWARD_MUTATIONS}


@pytest.mark.parametrize("name", sorted(ALL_MUTATIONS))
def test_pins_catch_planted_mistake(name):
    old, new = ALL_MUTATIONS[name]
    pins = PIN_FILES[name]
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(name, old, new, tmp)
        env = dict(os.environ, TTT_ORACLE_LIB_OVERRIDE=so)
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            os.path.join(ROOT, "tests", pins)],
                           env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"mutation {name} survived the pins:\n{r.stdout[-2000:]}"
