"""The pins catch plausible mistakes: each test plants one mistake in a copy
of the C oracle (on the CPU), loads it in place of the real one, runs the
pin suite and requires at least one pin to fail."""
import inspect
import json
import os
import subprocess

import pytest

import oracle
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
