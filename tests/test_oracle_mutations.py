"""Planted mistakes in a COPY of the oracle must be caught by the pins.

Each mutation is a plausible slip (wrong sign, wrong head mapping, off-by-one
mask, dropped term, transposed pairing).  The copy is compiled into a
temporary library on the CPU; the real oracle is never modified.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _adversarial_case, _brute_scores_and_out

SRC = os.path.join(os.path.dirname(oracle.lib_path()), "..", "lazy_oracle.c")

MUTATIONS = {
    "sin_sign": ("y[i] = a * c - b * s;", "y[i] = a * c + b * s;"),
    "gqa_modulo": ("int kvh = h / G;", "int kvh = h % Hkv;"),
    "mask_strict": ("if (P[u] <= p) {", "if (P[u] < p) {"),
    "dropped_local_index": ("P[t] = (int64_t)seg_off[g] + j;", "P[t] = (int64_t)seg_off[g];"),
    "interleaved_pairs": ("double a = x[i], b = x[i + half];", "double a = x[2 * i], b = x[2 * i + 1];"),
    "dropped_scale": ("s[u] = acc * scale;", "s[u] = acc;"),
    "theta_exponent": ("pow(base, -2.0 * (double)i / (double)d)", "pow(base, -1.0 * (double)i / (double)d)"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.check_call(["gcc", "-O1", "-std=gnu99", "-fPIC", "-shared", "-o", str(so), str(mut), "-lm"])
    lib = oracle.load_library(str(so))
    case = _adversarial_case(hq=4, hkv=2)
    _, ref = _brute_scores_and_out(case)
    out = oracle.attend(**case.oracle_kwargs(), lib=lib)
    assert not np.allclose(out, ref, rtol=1e-9, atol=1e-10), f"mutation {name} was not detected"
    # and the unmutated oracle passes the same check
    assert np.allclose(oracle.attend(**case.oracle_kwargs()), ref, rtol=1e-12, atol=1e-13)
