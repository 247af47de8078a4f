"""Plant plausible mistakes in the oracle (a mutated copy of its C source, or
a patched Python function) and check that the pins catch every one: at least
one pin must fail against each mutant.  CPU only; the real oracle is untouched.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import test_oracle_pins as P

_GROUP_ROWS = oracle.group_rows   # the real one, for the unstable-grouping mutant

# (name, exact text of oracle.c, mutated text)
C_MUTANTS = [
    ("level offset 2^b/2 instead of (2^b-1)/2",
     "return (double)c - ((double)((1 << bits) - 1)) / 2.0;", "return (double)c - ((double)(1 << bits)) / 2.0;"),
    ("SiLU with e^+z", "return z / (1.0 + exp(-z)); }", "return z / (1.0 + exp(z)); }"),
    ("shared expert dropped", "if (!rc && shared) {", "if (!rc && shared && 0) {"),
    ("router ties to the higher index", "if (best < 0 || l[e] > l[best]) best = e;",
     "if (best < 0 || l[e] >= l[best]) best = e;"),
    ("gate and up swapped", "h[i] = oracle_silu(g[i]) * u[i];", "h[i] = oracle_silu(u[i]) * g[i];"),
    ("block scale index reversed along k", "scale_value(M->bits, M->scales, n * (cols / 32) + k / 32)",
     "scale_value(M->bits, M->scales, n * (cols / 32) + (cols / 32 - 1 - k / 32))"),
    ("E8M0 bias 128", "return ldexp(1.0, (int)e - 127);", "return ldexp(1.0, (int)e - 128);"),
    ("softmax normaliser misses the top logit", "for (int j = 0; j < k; ++j) z += exp(",
     "for (int j = 1; j < k; ++j) z += exp("),
    ("RMS over H - 1", "double r = sqrt(ss / (double)H);", "double r = sqrt(ss / (double)(H - 1));"),
    ("bf16 truncation instead of round-to-nearest-even", "r = ldexp(nearbyint(ldexp(m, 8)), e - 8);",
     "r = ldexp(floor(ldexp(m, 8)), e - 8);"),
    ("binary16 subnormal exponent -25", "if (e == 0) v = ldexp((double)m, -24);",
     "if (e == 0) v = ldexp((double)m, -25);"),
]

PINS = ([(P.test_levels_match_fixed_table, (b,)) for b in (2, 3, 4)] +
        [(P.test_dequant_matches_table_and_numpy_f16, (b,)) for b in (2, 3, 4)] +
        [(P.test_scale_special_values, ())] +
        [(P.test_gemv_matches_numpy_dense, a) for a in ((2, 48, 160, 1), (3, 33, 96, 3), (4, 17, 224, 5))] +
        [(P.test_unit_vector_probe_returns_column, (b,)) for b in (2, 3, 4)] +
        [(P.test_gemv_closed_forms, (b,)) for b in (2, 3, 4)] +
        [(P.test_q_columns_equal_independent_columns, ()), (P.test_router_matches_stable_sort_and_softmax, ()),
         (P.test_router_k_equals_E_is_full_softmax, ()), (P.test_silu_matches_scipy, ()),
         (P.test_expert_closed_form_distinguishes_gate_up_down, ()), (P.test_moe_token_matches_dense_numpy, ()),
         (P.test_bf16_round_matches_torch, ()), (P.test_prefill_operand_rounding_matches_torch_bf16, ()),
         (P.test_gemv_bf16_weights_matches_torch_rounding, ()), (P.test_rms_bf16_closed_form_and_torch, ()),
         (P.test_group_rows_brute_force, ()), (P.test_router_logits_unit_vector_probe, ()),
         (P.test_router_logits_closed_form_and_bias_only, ()), (P.test_router_logits_brute_force, ())])


def first_failing_pin():
    for fn, args in PINS:
        try:
            fn(*args)
        except Exception:   # an assertion, or the mutant breaking a call outright
            return fn.__name__
    return None


def test_pins_pass_on_the_real_oracle():
    assert first_failing_pin() is None


@pytest.mark.parametrize("name,old,new", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_pins_catch_planted_c_mistake(name, old, new, tmp_path, monkeypatch):
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old}"
    path = tmp_path / "oracle_mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-fopenmp",
                           "-o", str(so), str(path), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle.load(str(so)))
    assert first_failing_pin() is not None, f"no pin catches: {name}"


def _logits_bias_sign(w_router, bias, x):
    W = oracle._bf16_bits_to_f64(np.asarray(w_router, dtype=np.uint16))
    X = oracle._bf16_bits_to_f64(np.atleast_2d(np.asarray(x, dtype=np.uint16)))
    lg, mag = X @ W.T, np.abs(X) @ np.abs(W).T
    if bias is not None:
        b = np.asarray(bias, dtype=np.float32).astype(np.float64)
        lg, mag = lg - b[None, :], mag + np.abs(b)[None, :]
    return lg, mag


def _logits_mag_without_bias(w_router, bias, x):
    W = oracle._bf16_bits_to_f64(np.asarray(w_router, dtype=np.uint16))
    X = oracle._bf16_bits_to_f64(np.atleast_2d(np.asarray(x, dtype=np.uint16)))
    lg, mag = X @ W.T, np.abs(X) @ np.abs(W).T
    if bias is not None:
        lg = lg + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    return lg, mag


def _group_rows_unstable(idx, w, E):
    counts, tok, wt, order = _GROUP_ROWS(idx, w, E)
    # swap the first two rows of the first expert with more than one row
    first = np.concatenate([[0], np.cumsum(counts)[:-1]])
    for e in range(E):
        if counts[e] > 1:
            a = first[e]
            tok, wt, order = tok.copy(), wt.copy(), order.copy()
            tok[[a, a + 1]] = tok[[a + 1, a]]
            wt[[a, a + 1]] = wt[[a + 1, a]]
            order[[a, a + 1]] = order[[a + 1, a]]
            break
    return counts, tok, wt, order


@pytest.mark.parametrize("attr,fake", [("router_logits", _logits_bias_sign),
                                       ("router_logits", _logits_mag_without_bias),
                                       ("group_rows", _group_rows_unstable)],
                         ids=["projection bias subtracted", "projection magnitude without the bias",
                              "grouping not stable"])
def test_pins_catch_planted_python_mistake(attr, fake, monkeypatch):
    monkeypatch.setattr(oracle, attr, fake)
    assert first_failing_pin() is not None
