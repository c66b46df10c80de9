"""The pins catch plausible mistakes: each test plants one mistake in a copy
of the C oracle (on the CPU), loads it in place of the real one, runs the
pin suite and requires at least one pin to fail.  Mistakes in the numpy
parts are planted by swapping one function for the duration of a run."""
import inspect
import json
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import msr as omsr
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "retention_oracle.c")

MUTANTS = {
    "no_decay_in_recurrence": ("S[(size_t)i * dv + j] = gamma * S[(size_t)i * dv + j] + kn[i] * vn[j];",
                               "S[(size_t)i * dv + j] = S[(size_t)i * dv + j] + kn[i] * vn[j];"),
    "transposed_outer_product": ("+ kn[i] * vn[j];", "+ kn[j % dk] * vn[i % dv];"),
    "readout_wrong_index": ("for (int j = 0; j < dv; j++) on[j] += qn[i] * S[(size_t)i * dv + j];",
                            "for (int j = 0; j < dv; j++) on[j] += qn[j % dk] * S[(size_t)(i % dv) * dv + (j + i) % dv];"),
    "rotation_sign": ("row[2 * p] = x0 * c - x1 * s;", "row[2 * p] = x0 * c + x1 * s;"),
    "rotation_frequency": ("-2.0 * p / (double)d", "-1.0 * p / (double)d"),
    "parallel_decay_off_by_one": ("orc_gamma_pow(gamma, n - m)", "orc_gamma_pow(gamma, n - m + 1)"),
    "parallel_not_inclusive": ("for (int m = 0; m <= n; m++)", "for (int m = 0; m < n; m++)"),
    "chunk_xi_off_by_one": ("orc_gamma_pow(gamma, r + 1)", "orc_gamma_pow(gamma, r)"),
    "chunk_zeta_off_by_one": ("orc_gamma_pow(gamma, L - 1 - r)", "orc_gamma_pow(gamma, L - r)"),
    "chunk_state_decay": ("double gL = orc_gamma_pow(gamma, L);", "double gL = orc_gamma_pow(gamma, L - 1);"),
    "decode_no_decay": ("S[(size_t)i * dv + j] = gamma * S[(size_t)i * dv + j] + kb[i] * vb[j];",
                        "S[(size_t)i * dv + j] = S[(size_t)i * dv + j] + kb[i] * vb[j];"),
    "gamma_pow_zero_exponent": ("if (e == 0) return 1.0;", "if (e == 0) return gamma;"),
    "backward_dk_on_the_query_row": ("dkk[IDX4(b, m, h, i, N, H, dk)] += w * g * qn[i];",
                                     "dkk[IDX4(b, n, h, i, N, H, dk)] += w * g * qn[i];"),
    "backward_dv_with_the_wrong_score": ("+= w * a * gn[j];", "+= w * g * gn[j];"),
    "backward_dq_with_the_wrong_score": ("dq[IDX4(b, n, h, i, N, H, dk)] += w * g * km[i];",
                                         "dq[IDX4(b, n, h, i, N, H, dk)] += w * a * km[i];"),
    "decay_norm_without_sqrt": ("double dscale = (flags & 1) ? 1.0 / sqrt(dsum) : 1.0;",
                                "double dscale = (flags & 1) ? 1.0 / dsum : 1.0;"),
    "score_norm_sum_of_abs": ("rsum += row[m];", "rsum += fabs(row[m]);"),
    "score_norm_before_decay_norm": ("rsum += row[m];", "rsum += row[m] / dscale;"),
    "score_norm_without_clamp": ("den = fabs(rsum) > 1.0 ? fabs(rsum) : 1.0;", "den = fabs(rsum);"),
}


def _pin_functions():
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if name.startswith("test_"):
            yield name, fn


def _run_pins(golden):
    failed = []
    for name, fn in _pin_functions():
        params = inspect.signature(fn).parameters
        marks = getattr(fn, "pytestmark", [])
        param_sets = [{}]
        for m in marks:
            if m.name == "parametrize":
                argname, values = m.args[0], m.args[1]
                param_sets = [{argname: v} for v in values]
        for ps in param_sets:
            kw = dict(ps)
            if "golden" in params:
                kw["golden"] = golden
            try:
                fn(**kw)
            except Exception:
                failed.append(name)
                break
    return failed


@pytest.fixture(scope="module")
def golden_data():
    with open(os.path.join(os.path.dirname(__file__), "golden", "running_example.json")) as f:
        return json.load(f)


def test_unmutated_oracle_passes_every_pin(golden_data):
    assert _run_pins(golden_data) == []


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_mutant(mutant, tmp_path, golden_data):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {old!r}"
    mutated = src.replace(old, new)
    c = tmp_path / f"{mutant}.c"
    so = tmp_path / f"{mutant}.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-std=c11", str(c), "-o", str(so), "-lm"])
    prev = oracle.swap_library(str(so))
    try:
        failed = _run_pins(golden_data)
    finally:
        oracle.swap_library(prev)
    assert failed, f"no pin caught mutant {mutant}"


# Plausible mistakes in the numpy parts of the oracle (the RetNet block),
# planted by replacing one function of oracle.msr for the duration of a run.
def _ln_unbiased(x, gain=None, bias=None, eps=1e-5):
    x = np.asarray(x, np.float64)
    y = (x - x.mean(-1, keepdims=True)) / np.sqrt(x.var(-1, ddof=1, keepdims=True) + eps)
    return y * (1.0 if gain is None else gain) + (0.0 if bias is None else bias)


def _gelu_tanh(x):
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def _block_post_norm(x, wq, wk, wv, wg, wo, w1, w2, gammas, H, k_scale, gn_eps=1e-5, ln_eps=1e-5,
                     ln1=(None, None), ln2=(None, None), theta_base=10000.0, return_y=False):
    y = omsr.layer_norm(omsr.msr_forward(x, wq, wk, wv, wg, wo, gammas, H, k_scale, gn_eps, theta_base) + x,
                        ln1[0], ln1[1], ln_eps)
    out = omsr.layer_norm(omsr.ffn(y, w1, w2) + y, ln2[0], ln2[1], ln_eps)
    return (out, y) if return_y else out


def _block_residual_of_the_normed_input(x, wq, wk, wv, wg, wo, w1, w2, gammas, H, k_scale, gn_eps=1e-5,
                                        ln_eps=1e-5, ln1=(None, None), ln2=(None, None), theta_base=10000.0,
                                        return_y=False):
    xn = omsr.layer_norm(x, ln1[0], ln1[1], ln_eps)
    y = omsr.msr_forward(xn, wq, wk, wv, wg, wo, gammas, H, k_scale, gn_eps, theta_base) + xn
    yn = omsr.layer_norm(y, ln2[0], ln2[1], ln_eps)
    out = omsr.ffn(yn, w1, w2) + yn
    return (out, y) if return_y else out


def _msr_without_rotation(x, wq, wk, wv, wg, wo, gammas, H, k_scale, eps, theta_base=10000.0, heads=None,
                          return_parts=False):
    """msr_forward with the xPos rotation of Q and K left out."""
    x = np.asarray(x, np.float64)
    B, N, _ = x.shape
    dk, dv = wq.shape[1] // H, wv.shape[1] // H
    q = omsr.project(x, wq).reshape(B, N, H, dk)
    k = omsr.project(x, wk).reshape(B, N, H, dk) * k_scale
    v = omsr.project(x, wv).reshape(B, N, H, dv)
    ret, _ = oracle.retention_recurrent(q, k, v, np.asarray(gammas, np.float64))
    z = omsr.swish(omsr.project(x, wg).reshape(B, N, H, dv)) * omsr.group_norm_heads(ret, eps)
    return omsr.project(z.reshape(B, N, H * dv), wo)


def _msr_gate_before_group_norm(x, wq, wk, wv, wg, wo, gammas, H, k_scale, eps, theta_base=10000.0, heads=None,
                                return_parts=False):
    """msr_forward with the swish gate applied before the GroupNorm."""
    x = np.asarray(x, np.float64)
    B, N, _ = x.shape
    dk, dv = wq.shape[1] // H, wv.shape[1] // H
    q = oracle.xpos_rotate(omsr.project(x, wq).reshape(B, N, H, dk), 0, theta_base)
    k = oracle.xpos_rotate(omsr.project(x, wk).reshape(B, N, H, dk) * k_scale, 0, theta_base)
    v = omsr.project(x, wv).reshape(B, N, H, dv)
    ret, _ = oracle.retention_recurrent(q, k, v, np.asarray(gammas, np.float64))
    z = omsr.group_norm_heads(omsr.swish(omsr.project(x, wg).reshape(B, N, H, dv)) * ret, eps)
    return omsr.project(z.reshape(B, N, H * dv), wo)


PY_MUTANTS = {
    "msr_rotation_dropped": ("msr_forward", _msr_without_rotation),
    "msr_gate_before_group_norm": ("msr_forward", _msr_gate_before_group_norm),
    "layer_norm_unbiased_variance": ("layer_norm", _ln_unbiased),
    "gelu_tanh_approximation": ("gelu", _gelu_tanh),
    "block_post_norm": ("retnet_block", _block_post_norm),
    "block_residual_of_the_normed_input": ("retnet_block", _block_residual_of_the_normed_input),
}


@pytest.mark.parametrize("mutant", sorted(PY_MUTANTS))
def test_pins_catch_numpy_mutant(mutant, golden_data, monkeypatch):
    name, fn = PY_MUTANTS[mutant]
    monkeypatch.setattr(omsr, name, fn)
    assert _run_pins(golden_data), f"no pin caught mutant {mutant}"
