"""The pins catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of sas_oracle.c (on the CPU, in a
temporary directory), loads the mutant in place of the oracle and checks that
at least one pin of test_oracle_pins fails against it.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "sas_oracle.c")

MUTANTS = {
    "gate dropped": ("bias[m] = logg[j]; ++m;", "bias[m] = 0.0; ++m;"),
    "current block excludes the query": ("x <= p; ++x) { tok[m] = x;", "x < p; ++x) { tok[m] = x;"),
    "tie to the higher index": ("return (x->i < y->i) ? -1 : (x->i > y->i);",
                                "return (x->i > y->i) ? -1 : (x->i < y->i);"),
    "score gradient sign": ("dsr[c] = -exp((double)s[c] - lse) * tot;",
                            "dsr[c] = exp((double)s[c] - lse) * tot;"),
    "scale missing on dk": ("dk[kv + tok[j] * d + x] += scale * dS[j]", "dk[kv + tok[j] * d + x] += dS[j]"),
    "gate normaliser off by one": ("for (int64_t i = 0; i < C; ++i) l += exp",
                                   "for (int64_t i = 1; i < C; ++i) l += exp"),
    "dv uses dS": ("dv[kv + tok[j] * d + x] += P[j] * (double)dOh[x];",
                   "dv[kv + tok[j] * d + x] += dS[j] * (double)dOh[x];"),
    "sigmoid gate derivative uses g instead of 1 - g": (
        "dsr[idx[jj]] = gs[jj] * (1.0 - exp(log_sigmoid((double)s[idx[jj]])));",
        "dsr[idx[jj]] = gs[jj] * exp(log_sigmoid((double)s[idx[jj]]));"),
    "kept-block softmax normalised over all candidates": (
        "for (int32_t j = 0; j < n; ++j) logg[j] = (double)s[idx[j]] - lk;",
        "for (int32_t j = 0; j < n; ++j) logg[j] = (double)s[idx[j]] - *lse;"),
    "hard gate gradient without the gate factor": (
        "for (int32_t jj = 0; jj < n; ++jj) dsr[idx[jj]] += gs[jj] * exp((double)s[idx[jj]] - lse);",
        "for (int32_t jj = 0; jj < n; ++jj) dsr[idx[jj]] += gs[jj];"),
}

PIN_CALLS = [
    lambda m: pins.test_bias_matrix_forward(m, 0, 2, 0),
    lambda m: pins.test_autograd_backward(m, 0, 2, 0),
    lambda m: pins.test_golden_worked_example(m),
    lambda m: pins.test_golden_topk_ties(m),
    lambda m: pins.test_topk_bruteforce_lexsort(m),
    lambda m: pins.test_gate_modes_forward_and_autograd(m, 2),
    lambda m: pins.test_gate_modes_forward_and_autograd(m, 4),
    lambda m: pins.test_gate_modes_forward_and_autograd(m, 5),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, monkeypatch, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor must be unique"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                           str(mut), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle._setup(ctypes.CDLL(str(so))))
    failures = 0
    for call in PIN_CALLS:
        try:
            call(oracle)
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught the mutant '{name}'"


def test_per_head_composition_mistake_is_caught(monkeypatch):
    """The per-query-head composition pins catch K/V heads matched to the wrong
    query heads (tiled instead of repeated: head h paired with KV head h mod Hkv)."""
    monkeypatch.setattr(oracle, "_repeat_heads", lambda x, G: __import__("numpy").tile(oracle._f32(x), (1, G, 1, 1)))
    with pytest.raises(AssertionError):
        pins.test_per_head_selection_pins(oracle, 11, 2, 0)
