"""The scan oracle's pins catch plausible mistakes in its C code.

Each case copies oracle/ssm_oracle.c, plants one mistake by text substitution
(a dropped factor, a swapped operand, a wrong sign, a misplaced bias, a term
left out of the adjoint), builds it into a temporary library, points the
oracle at that library, and checks that at least one of the pins of
test_oracle.py fails.  The oracle's own source and library are untouched."""
import os
import shutil
import subprocess

import pytest

import oracle
import test_oracle as T

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")

FWD_PINS = [
    T.test_golden_lti_impulse_kernel,
    T.test_hand_unrolled_n1_l3,
    T.test_hand_unrolled_two_states_two_channels,
    T.test_lti_equals_bruteforce_convolution,
    T.test_A_zero_is_running_sum,
    T.test_gate_identity,
    T.test_softplus_identities,
    T.test_zoh_matches_ode_solution,
]
BWD_PINS = [
    lambda: T.test_adjoint_matches_central_differences(True, True, True),
    lambda: T.test_adjoint_matches_central_differences(False, False, False),
    lambda: T.test_zoh_adjoint_matches_central_differences(1.0),
]

MUTANTS = {
    # forward
    "input dropped from the update": ("h[n] = abar * h[n] + bbar * x;", "h[n] = abar * h[n] + bbar;"),
    "step size missing in the decay": ("double abar = exp(dt * a);", "double abar = exp(a);"),
    "skip term with the wrong sign": (
        "if (D) y += D[d] * x;\n                if (zb) y *= zb[t] * sigmoid(zb[t]);",
        "if (D) y -= D[d] * x;\n                if (zb) y *= zb[t] * sigmoid(zb[t]);"),
    "B read in place of C": ("y += Cb[(size_t)n * seqlen + t] * h[n];",
                             "y += Bb[(size_t)n * seqlen + t] * h[n];"),
    "gate without z": ("if (zb) y *= zb[t] * sigmoid(zb[t]);", "if (zb) y *= sigmoid(zb[t]);"),
    "bias added after the softplus": (
        "double r = db[t] + (delta_bias ? delta_bias[d] : 0.0);\n"
        "                double dt = delta_softplus ? softplus(r) : r;",
        "double r = db[t];\n"
        "                double dt = (delta_softplus ? softplus(r) : r) + (delta_bias ? delta_bias[d] : 0.0);"),
    "zoh factor without 1/A": ("bbar = expm1(dt * a) / a * Bb[(size_t)n * seqlen + t];",
                               "bbar = expm1(dt * a) * Bb[(size_t)n * seqlen + t];"),
    # backward
    "adjoint: decay term missing from dDelta": (
        "ddt += l * (Ad[n] * abar * hprev[n] + Bt * x * dk_ddt);", "ddt += l * (Bt * x * dk_ddt);"),
    "adjoint: lambda not propagated": ("lam[n] = abar * l;", "lam[n] = l;"),
    "adjoint: dC from the previous state": ("bC[(size_t)n * seqlen + t] += gy * hcur[n];",
                                            "bC[(size_t)n * seqlen + t] += gy * hprev[n];"),
    "adjoint: softplus derivative dropped": ("double dr = delta_softplus ? ddt * sigmoid(r) : ddt;",
                                             "double dr = ddt;"),
}


def _fails(pins):
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    return failed


@pytest.fixture(scope="module")
def built_mutants():
    import pathlib
    src = open(SRC).read()
    out = {}
    # a scratch folder inside the repository's (git-ignored) build area
    d = pathlib.Path(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))) / "_build" / "oracle_mutants"
    shutil.rmtree(d, ignore_errors=True)
    d.mkdir(parents=True)
    for i, (name, (old, new)) in enumerate(MUTANTS.items()):
        assert src.count(old) == 1, name
        msrc = d / f"m{i}.c"
        msrc.write_text(src.replace(old, new))
        lib = d / f"libm{i}.so"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
                               str(msrc), "-o", str(lib), "-lm"])
        out[name] = (str(msrc), str(lib))
    yield out
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", list(MUTANTS))
def test_c_mutant_is_caught(monkeypatch, built_mutants, name):
    msrc, lib = built_mutants[name]
    monkeypatch.setattr(oracle, "_SRC", msrc)
    monkeypatch.setattr(oracle, "_LIB", lib)
    monkeypatch.setattr(oracle, "_lib", None)
    pins = BWD_PINS if name.startswith("adjoint") else FWD_PINS
    assert _fails(pins) >= 1, name


def test_pins_pass_on_the_oracle():
    assert _fails(FWD_PINS) == 0 and _fails(BWD_PINS) == 0
