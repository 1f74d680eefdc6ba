"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a private copy of oracle/oracle.c (on the
CPU), builds it, points the oracle module at the broken build and runs the pin
tests of tests/test_oracle_router.py and tests/test_oracle_forward.py against it.
A mistake that every pin lets through would mean the pins do not tie that part
of the oracle to the pages; the test requires at least one pin to fail.
"""

import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_forward as tf
import test_oracle_router as tr

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    # router
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-r));", "return 1.0 / (1.0 + exp(r));"),
    "bias_ignored_in_selection": ("sp[e] = s[e] + (double)b[e];", "sp[e] = s[e];"),
    "bias_in_weights": ("double sv = s[chosen[t]];", "double sv = sp[chosen[t]];"),
    "weights_without_alpha": ("? alpha * sv / (sum + 1e-20) : alpha * sv",
                              "? sv / (sum + 1e-20) : alpha * sv"),
    "weights_not_renormalised": ("? alpha * sv / (sum + 1e-20) : alpha * sv",
                                 "? alpha * sv : alpha * sv"),
    "group_score_top1_only": ("gs[g] = sp[i1] + sp[i2];", "gs[g] = sp[i1];"),
    "ties_to_higher_index": ("if (best < 0 || v[i] > v[best])", "if (best < 0 || v[i] >= v[best])"),
    "group_restriction_dropped": ("cand[e] = kept[e / m];", "cand[e] = 1;"),
    "logit_dot_drops_last_term": ("for (int i = 0; i < len; ++i)\n        acc += a[i] * b[i];",
                                  "for (int i = 0; i + 1 < len; ++i)\n        acc += a[i] * b[i];"),
    # forward
    "gate_up_swapped": ("swiglu_accumulate(gate_up, gu, gate_up, gu + (size_t)d * D, down,",
                        "swiglu_accumulate(gate_up, gu + (size_t)d * D, gate_up, gu, down,"),
    "silu_missing_factor": ("static double silu(double a) { return a * sigmoid(a); }",
                            "static double silu(double a) { return sigmoid(a); }"),
    "shared_expert_dropped": ("swiglu_accumulate(sh_gate, 0, sh_up, 0, sh_down, 0, dt, D, d_sh, xn, 1.0, yn, row,",
                              "if (0) swiglu_accumulate(sh_gate, 0, sh_up, 0, sh_down, 0, dt, D, d_sh, xn, 1.0, yn, row,"),
    "shared_expert_scaled": ("swiglu_accumulate(sh_gate, 0, sh_up, 0, sh_down, 0, dt, D, d_sh, xn, 1.0, yn, row,",
                             "swiglu_accumulate(sh_gate, 0, sh_up, 0, sh_down, 0, dt, D, d_sh, xn, 2.5, yn, row,"),
    "shared_width_capped_at_d_moe": ("swiglu_accumulate(sh_gate, 0, sh_up, 0, sh_down, 0, dt, D, d_sh, xn, 1.0,",
                                     "swiglu_accumulate(sh_gate, 0, sh_up, 0, sh_down, 0, dt, D, d_sh < d ? d_sh : d, xn, 1.0,"),
    "routed_weight_ignored": ("w[(size_t)n * k + j], yn, row, h, gate_max, up_max);",
                              "1.0, yn, row, h, gate_max, up_max);"),
    "sentinel_not_skipped": ("const int i = idx[(size_t)n * k + j];\n                if (i == E)",
                             "const int i = idx[(size_t)n * k + j] == E ? E - 1 : idx[(size_t)n * k + j];\n                if (i == E)"),
    "gate_clamped_both_sides": ("if (a > gate_max)\n            a = gate_max;",
                                "if (a > gate_max)\n            a = gate_max;\n        if (a < -gate_max)\n            a = -gate_max;"),
    "up_clamped_above_only": ("if (u < -up_max)\n            u = -up_max;", ""),
    "bf16_widened_wrong": ("uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;",
                           "uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 15;"),
}

PINS = [getattr(m, n) for m in (tr, tf) for n in sorted(dir(m))
        if n.startswith("test_") and callable(getattr(m, n))]


def _run_pin(fn):
    """Run one pin test function (parametrised pins over their parameter sets)."""
    marks = getattr(fn, "pytestmark", [])
    params = [m for m in marks if m.name == "parametrize"]
    if not params:
        fn()
        return
    names, values = params[0].args[0], params[0].args[1]
    names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
    for v in values:
        v = v if isinstance(v, (tuple, list)) and len(names) > 1 else (v,)
        fn(**dict(zip(names, v)))


@pytest.fixture
def mutant_oracle(tmp_path, monkeypatch):
    def build(name):
        old, new = MUTANTS[name]
        src = open(SRC).read()
        assert old in src, "mutation anchor not found: %s" % name
        path = tmp_path / ("oracle_%s.c" % name)
        path.write_text(src.replace(old, new, 1))
        lib = tmp_path / ("liboracle_%s.so" % name)
        subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(path),
                        "-lm"], check=True)
        monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(str(lib))))
    return build


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, mutant_oracle):
    mutant_oracle(name)
    caught = []
    for fn in PINS:
        try:
            _run_pin(fn)
        except (AssertionError, ValueError) as exc:  # a pin failed on the broken oracle
            caught.append(fn.__name__)
    assert caught, "no pin fails when the oracle has mistake '%s'" % name
