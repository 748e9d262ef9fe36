"""The oracle's pins catch plausible mistakes (CPU only).  Each mutant is the oracle's C source
with one deliberate error planted, compiled into a temporary directory; the named pins of
``test_oracle.py`` are then run against it and must fail.  The real oracle passes the same pins
in ``test_oracle.py``.  Every mutant keeps all memory accesses in bounds."""
import os

import pytest

import test_oracle as P
from oracle import oracle as O

# name: (text of the oracle, planted replacement, pins that must fail)
MUTANTS = {
    "summary divides by span - 1": (
        "out[(bh * nspan + j) * D + d] = rnd(acc / (double)span, prec);",
        "out[(bh * nspan + j) * D + d] = rnd(acc / (double)(span - 1), prec);",
        [("test_summaries_one_hot_position", {}),
         ("test_summaries_closed_form_offset_plus_zero_mean_pattern", {"prec": 64})]),
    "block query over strided query heads": (
        "const int64_t h = kh * G + hh;\n                        for (int64_t t = n * qblock;",
        "const int64_t h = hh * Hkv + kh;\n                        for (int64_t t = n * qblock;",
        [("test_block_query_one_hot_gqa_mapping", {})]),
    "ties go to the higher index": (
        "return (a->i < b->i) ? -1 : (a->i > b->i);",
        "return (a->i > b->i) ? -1 : (a->i < b->i);",
        [("test_topk_ties_go_to_lower_index", {}), ("test_worked_example_golden", {})]),
    "group candidates of a chunk indexed with the wrong stride": (
        "const int64_t j = csel[c] * gpc + r;",
        "const int64_t j = csel[c] + r * nch;",
        [("test_route_brute_force_tiny", {"prec": 64}), ("test_route_planted_chunks_are_selected", {})]),
    "query head h reads KV head h % Hkv": (
        "const int64_t G = L->Hq / L->Hkv, kh = h / G, n = t / L->qblock;",
        "const int64_t G = L->Hq / L->Hkv, kh = h % L->Hkv, n = t / L->qblock;",
        [("test_dense_equivalence_with_full_budget", {})]),
    "causal local part drops the diagonal": (
        "for (int64_t u = 0; u <= t; ++u) {",
        "for (int64_t u = 0; u < t; ++u) {",
        [("test_routed_attention_equals_masked_dense_attention", {}), ("test_worked_example_golden", {})]),
    "dK with the wrong sign": (
        "dk[i * D + d] += scale * ds * qv[d];",
        "dk[i * D + d] -= scale * ds * qv[d];",
        [("test_gradients_match_finite_differences", {}), ("test_dense_equivalence_with_full_budget", {})]),
    "dV weighted by dS instead of P": (
        "dv[i * D + d] += pu * dov[d];",
        "dv[i * D + d] += ds * dov[d];",
        [("test_gradients_match_finite_differences", {})]),
}


@pytest.fixture
def mutant_oracle(tmp_path, monkeypatch):
    """Returns a function that builds the oracle with one text replaced and points the oracle module
    at it for the rest of the test (the module's library handle is restored afterwards)."""
    src = open(O._SRC).read()

    def make(old, new):
        assert src.count(old) == 1, old
        path = os.path.join(tmp_path, "hga_oracle.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        monkeypatch.setattr(O, "_SRC", path)
        monkeypatch.setattr(O, "_LIB_PATH", os.path.join(tmp_path, "libhga_oracle.so"))
        monkeypatch.setattr(O, "_lib", None)
        return O

    return make


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_fail_on_planted_mistake(mutant_oracle, name):
    old, new, pins = MUTANTS[name]
    mo = mutant_oracle(old, new)
    for pin, kw in pins:
        with pytest.raises(AssertionError):
            getattr(P, pin)(mo, **kw)
