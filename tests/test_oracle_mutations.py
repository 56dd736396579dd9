"""Planted mistakes in a COPY of the oracle must be caught by the pins.

Each mutation is a plausible slip (wrong sign, wrong head mapping, off-by-one
mask, dropped term, transposed pairing).  The copy is compiled into a
temporary library on the CPU; the real oracle is never modified.
"""
import importlib.util
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import ALIBI_PINS, _adversarial_case, _brute_scores_and_out

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


ALIBI_MUTATIONS = {
    "alibi_sign": ("s[u] -= g_alibi[h] * (double)(p - P[u]);", "s[u] += g_alibi[h] * (double)(p - P[u]);"),
    "alibi_kv_head_slope": ("s[u] -= g_alibi[h] * (double)(p - P[u]);", "s[u] -= g_alibi[kvh] * (double)(p - P[u]);"),
    "alibi_no_key_position": ("s[u] -= g_alibi[h] * (double)(p - P[u]);", "s[u] -= g_alibi[h] * (double)(p);"),
    "alibi_query_still_rotated": ("if (alibi)\n                memcpy(qr, xq", "if (0)\n                memcpy(qr, xq"),
    "alibi_slopes_odd_terms": ("alibi_geometric(2 * m, 2 * (k - m))", "alibi_geometric(2 * m, 2 * (k - m) + 1)"),
    "alibi_slopes_exponent": ("-8.0 * (double)(k + 1)", "-8.0 * (double)k"),
}


def _alibi_pins_fail(lib) -> list[str]:
    failed = []
    for pin in ALIBI_PINS:
        try:
            pin(lib=lib)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(ALIBI_MUTATIONS))
def test_planted_alibi_mistake_is_caught(name, tmp_path):
    old, new = ALIBI_MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.check_call(["gcc", "-O1", "-std=gnu99", "-fPIC", "-shared", "-o", str(so), str(mut), "-lm"])
    assert _alibi_pins_fail(oracle.load_library(str(so))), f"mutation {name} was not detected"
    assert not _alibi_pins_fail(None)


# ----------------------------------------------------------------------------- reference block cache
CACHE_SRC = os.path.join(os.path.dirname(oracle.__file__), "cache_ref.py")

CACHE_MUTATIONS = {
    "evict_most_recent": ("self.entries.popitem(last=False)", "self.entries.popitem(last=True)"),
    "no_refresh_on_hit": ("self.entries.move_to_end(key)", "pass"),
    "prefix_reuse_past_a_miss": ('hit = cache.access(("seq",) + seq, n) and chain_intact',
                                 'hit = cache.access(("seq",) + seq, n)'),
    "aware_writes_no_copy": ("cache.access(here, n)                            # the re-encoded copy", "pass"),
    "exact_offset_ignored": ('hit = cache.access(("doc@", d, offset), n)', 'hit = cache.access(("doc@", d, 0), n)'),
    "offset_not_advanced": ("offset += int(doc_tokens[d])", "offset += 0"),
    "blocks_rounded_down": ("n = -(-int(doc_tokens[d]) // block_tokens)", "n = int(doc_tokens[d]) // block_tokens"),
}


def _cache_pins_fail(mod, monkeypatch) -> list[str]:
    from tests import test_cache as T
    monkeypatch.setattr(T, "RefLRU", mod.RefLRU)
    monkeypatch.setattr(T, "ref_simulate", mod.ref_simulate)
    checks = [("lru", T.test_ref_lru_hand_worked), ("trace", T.test_ref_policies_hand_worked_trace),
              ("prefix", T.test_ref_prefix_reuse_stops_at_the_first_miss),
              ("unlimited", T.test_ref_unlimited_capacity_closed_forms)]
    checks += [(f"pin{args}", (lambda a=args: T.test_ref_policies_hand_worked(*a))) for args in T.POLICY_PINS]
    failed = []
    for name, fn in checks:
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


@pytest.mark.parametrize("name", sorted(CACHE_MUTATIONS))
def test_planted_cache_mistake_is_caught(name, tmp_path, monkeypatch):
    old, new = CACHE_MUTATIONS[name]
    src = open(CACHE_SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"cache_ref_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"cache_ref_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert _cache_pins_fail(mod, monkeypatch), f"mutation {name} was not detected"
    import oracle.cache_ref as real
    assert not _cache_pins_fail(real, monkeypatch)
