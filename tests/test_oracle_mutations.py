"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle's C source — a dropped term, a wrong
sign, a swapped operand, a shifted index — builds it, points the oracle package at the
mutated library and runs the pins of tests/test_oracle.py.  At least one pin must fail for
every planted mistake; the unmutated source must pass them all.  Nothing here touches a GPU
or the CUDA library.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle as pins

# (name, text in kda_oracle.c, replacement)
MUTATIONS = [
    ("read before the write", """        /* S = S' + k u^T */
        for (int c = 0; c < dk; ++c) {
            double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] += kt[c] * u[j];
        }
        /* o = S^T q */
        if (oh) {
            double *ot = oh + (size_t)t * sv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int c = 0; c < dk; ++c) {
                const double *row = S + (size_t)c * dv;
                for (int j = 0; j < dv; ++j) ot[j] += qt[c] * row[j];
            }
        }""", """        if (oh) {
            double *ot = oh + (size_t)t * sv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int c = 0; c < dk; ++c) {
                const double *row = S + (size_t)c * dv;
                for (int j = 0; j < dv; ++j) ot[j] += qt[c] * row[j];
            }
        }
        for (int c = 0; c < dk; ++c) {
            double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] += kt[c] * u[j];
        }"""),
    ("write not scaled by beta", "u[j] = beta * (vt[j] - kS[j]);", "u[j] = (vt[j] - kS[j]);"),
    ("sign of the correction", "u[j] = beta * (vt[j] - kS[j]);", "u[j] = beta * (vt[j] + kS[j]);"),
    ("log-decay scale", """        for (int c = 0; c < dk; ++c) {
            const double a = exp(gt[c]);""", """        for (int c = 0; c < dk; ++c) {
            const double a = exp(0.5 * gt[c]);"""),
    ("read with k instead of q", "for (int j = 0; j < dv; ++j) ot[j] += qt[c] * row[j];",
     "for (int j = 0; j < dv; ++j) ot[j] += kt[c] * row[j];"),
    ("conv tap order", "acc += w[(size_t)c * 4 + i] * x[", "acc += w[(size_t)c * 4 + (3 - i)] * x["),
    ("softplus", "return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x));", "return exp(x);"),
    ("L2-norm epsilon outside the root", "const double inv = 1.0 / sqrt(ss + eps);",
     "const double inv = 1.0 / (sqrt(ss) + eps);"),
    ("gate bias sign", "softplus(x[r * dk + c] + bias)", "softplus(x[r * dk + c] - bias)"),
    ("gate bound direction", "g[r * dk + c] = v < lb ? lb : v;", "g[r * dk + c] = v > lb ? lb : v;"),
    ("RMS over dv - 1", "ms /= (double)dv;", "ms /= (double)(dv - 1);"),
    ("gradient: sign of dg", "acc_g += dsp * sp;", "acc_g -= dsp * sp;"),
    ("gradient: dbeta without the readout", "dbt += du[j] * (v[tv + j] - R[(size_t)t * dv + j]);",
     "dbt += du[j] * v[tv + j];"),
    ("gradient: dk without the readout term", "acc_k += dS[(size_t)c * dv + j] * U[(size_t)t * dv + j] + sp * da[j];",
     "acc_k += dS[(size_t)c * dv + j] * U[(size_t)t * dv + j];"),
    ("gradient: dS' without k da^T", "const double dsp = dS[(size_t)c * dv + j] + k[tk + c] * da[j];",
     "const double dsp = dS[(size_t)c * dv + j];"),
]

PINS = [
    lambda: pins.test_chunked_rewrite_equals_recurrence(4, 16),
    lambda: pins.test_unrolled_product_of_transition_matrices(5),
    pins.test_zero_decay_zero_beta_is_readout_of_initial_state,
    pins.test_small_beta_limit_is_causal_linear_attention,
    pins.test_delta_rule_retrieval,
    pins.test_pure_decay_closed_form,
    pins.test_short_conv_matches_torch_depthwise_conv1d,
    pins.test_short_conv_one_hot_taps_shift,
    pins.test_l2norm_closed_form,
    pins.test_gate_special_values_and_library_softplus,
    pins.test_gate_lower_bound,
    pins.test_out_norm_gate_closed_forms,
    lambda: pins.test_layer_wiring_with_identity_conv(None),
    pins.test_backward_equals_central_differences,
    pins.test_backward_equals_torch_autograd,
]


def _build(src_text, path):
    c = str(path) + ".c"
    with open(c, "w") as f:
        f.write(src_text)
    so = str(path) + ".so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", so, c, "-lm"])
    return oracle.declare(ctypes.CDLL(so))


def _failing_pins(lib, monkeypatch):
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed += 1
    return failed


def test_unmutated_source_passes_every_pin(tmp_path, monkeypatch):
    lib = _build(open(oracle._SRC).read(), tmp_path / "clean")
    assert _failing_pins(lib, monkeypatch) == 0


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(name, old, new, tmp_path, monkeypatch):
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor for '{name}' not found exactly once"
    lib = _build(src.replace(old, new), tmp_path / "mutant")
    assert _failing_pins(lib, monkeypatch) >= 1, f"no pin catches: {name}"
