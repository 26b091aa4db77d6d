"""The pins must catch plausible mistakes.  Each case compiles a copy of the
oracle with one planted error (on the CPU, in a temporary directory) and
checks that at least one pin fails against it; the real oracle is restored
afterwards."""
import os
import subprocess

import numpy as np
import pytest

import enum_harness as eh
from oracle import oracle

# (name, exact source fragment, planted replacement)
MUTANTS = [
    ("residual_sign", "double d = et[v] / Zt - ed[v] / Zd;", "double d = ed[v] / Zd - et[v] / Zt;"),
    ("ratio_inverted", "double ratio = pt / pd;", "double ratio = pd / pt;"),
    ("verify_conditions_on_current_token",
     "draft_bias(U, Arec, W, V, r, x0[b], x + (size_t)b * G, k, hs, hs + r, delta);",
     "draft_bias(U, Arec, W, V, r, x0[b], x + (size_t)b * G, k + 1, hs, hs + r, delta);"),
    ("draft_ignores_previous_token", "draft_bias(U, A, W, V, r, x0[b], x_out + (size_t)b * G, i + 1, h, h + r, delta);",
     "draft_bias(U, A, W, V, r, x0[b], x_out + (size_t)b * G, 1, h, h + r, delta);"),
    ("bonus_from_last_admitted_row", "int ks = A + 1;", "int ks = (A == lb && A > 0) ? A : A + 1;"),
    ("residual_without_clamp", "q[v] = d > 0.0 ? d : 0.0;", "q[v] = d > 0.0 ? d : -d;"),
    ("target_row_shifted", "const float *Trow = Tlog + ((size_t)b * (G + 1) + (k - 1)) * (size_t)V;",
     "const float *Trow = Tlog + ((size_t)b * (G + 1) + k) * (size_t)V;"),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(oracle.source_path()).read()
    assert src.count(old) == 1, name
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o",
                    str(so), str(path), "-lm"], check=True)
    return str(so)


def _preservation_probe():
    """Worst preservation error over a few exact-enumeration scenarios."""
    worst = 0.0
    for seed, (V, G, r, T) in enumerate([(3, 3, 2, 1.0), (4, 2, 2, float(np.float32(0.7)))]):
        rng = np.random.default_rng(100 + seed)
        Lrows = rng.normal(0, 1.5, (G, V)).astype(np.float32)
        U = rng.normal(0, 1.0, (V, r)).astype(np.float32)
        W = rng.normal(0, 1.0, (r, V)).astype(np.float32)
        target = eh.random_target(rng, V, G)
        for ell in range(G + 1):
            sc = eh.Scenario(Lrows, U, W, int(rng.integers(0, V)), T, target, ell_fixed=ell)
            try:
                law = sc.output_law()
            except Exception:
                return np.inf
            worst = max(worst, eh.preservation_error(law, target, T, V))
    return worst


def test_real_oracle_passes_probe():
    oracle.use_library(oracle.build())
    assert _preservation_probe() < 1e-12


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    so = _build_mutant(tmp_path, name, old, new)
    try:
        oracle.use_library(so)
        assert _preservation_probe() > 1e-6
    finally:
        oracle.use_library(oracle.build())


# Planted mistakes in the scheduler variants, caught by the scheduler pins.
SCHED_MUTANTS = [
    ("topk_counts_from_one", "int n = capacity < 0 ? 0 : (capacity > N ? N : capacity);",
     "int n = capacity < 1 ? 0 : (capacity > N ? N : capacity - 1);"),
    ("topk_ignores_budget", "    if (budget >= 0 && budget < n) n = budget;\n    for (int b = 0; b < B; ++b) ell_out[b] = 0;\n"
     "    for (int k = 0; k < n; ++k) ell_out[c[k].idx % B] += 1;\n    *n_adm_out = n;\n    free(c);\n"
     "    return ORACLE_OK;\n}\n\n/* ----",
     "    for (int b = 0; b < B; ++b) ell_out[b] = 0;\n"
     "    for (int k = 0; k < n; ++k) ell_out[c[k].idx % B] += 1;\n    *n_adm_out = n;\n    free(c);\n"
     "    return ORACLE_OK;\n}\n\n/* ----"),
    ("topk_request_index", "for (int k = 0; k < n; ++k) ell_out[c[k].idx % B] += 1;\n    *n_adm_out = n;\n    free(c);\n"
     "    return ORACLE_OK;\n}\n\n/* ----",
     "for (int k = 0; k < n; ++k) ell_out[c[k].idx / G % B] += 1;\n    *n_adm_out = n;\n    free(c);\n"
     "    return ORACLE_OK;\n}\n\n/* ----"),
]


@pytest.mark.parametrize("name,old,new", SCHED_MUTANTS, ids=[m[0] for m in SCHED_MUTANTS])
def test_scheduler_mutant_is_caught(tmp_path, name, old, new):
    import test_oracle_pins as pins
    so = _build_mutant(tmp_path, name, old, new)
    caught = False
    try:
        oracle.use_library(so)
        for pin in (pins.test_scheduler_topk_is_the_first_k_of_the_stable_order,
                    pins.test_scheduler_topk_with_the_greedy_count_is_the_greedy_schedule):
            try:
                pin()
            except AssertionError:
                caught = True
    finally:
        oracle.use_library(oracle.build())
    assert caught, f"no scheduler pin catches {name}"



# Planted mistakes in the RNN head, caught by the RNN pins.
RNN_MUTANTS = [
    ("rnn_state_not_carried", "        for (int c = 0; c < r; ++c) h[c] = hn[c];\n", "\n"),
    ("rnn_without_tanh", "            hn[c] = tanh(a);\n        }\n        for (int c = 0; c < r; ++c) h[c] = hn[c];",
     "            hn[c] = a;\n        }\n        for (int c = 0; c < r; ++c) h[c] = hn[c];"),
    ("rnn_state_from_current_token", "int tok = (j == 1) ? x0 : xs[j - 2];", "int tok = (j == 1) ? x0 : xs[j - 1];"),
]


@pytest.mark.parametrize("name,old,new", RNN_MUTANTS, ids=[m[0] for m in RNN_MUTANTS])
def test_rnn_mutant_is_caught(tmp_path, name, old, new):
    import test_oracle_rnn as pins
    so = _build_mutant(tmp_path, name, old, new)
    caught = []
    try:
        oracle.use_library(so)
        for pin, args in ((pins.test_zero_recurrence_is_the_markov_head_with_tanh_factor, (1.0,)),
                          (pins.test_bias_depends_on_the_whole_prefix, ()),
                          (pins.test_rnn_head_keeps_the_target_law, (0, 3, 3, 2, 1.0)),
                          (pins.test_rnn_and_markov_drafts_differ_when_the_state_carries, ())):
            try:
                pin(*args)
            except (AssertionError, ValueError):
                caught.append(pin.__name__)
    finally:
        oracle.use_library(oracle.build())
    assert caught, f"no RNN pin catches {name}"


# Planted mistakes in the decision margins, caught by the margin pins.
MARGIN_MUTANTS = [
    ("draft_margin_unnormalised", "double m0 = u - prev, m1 = c - u;",
     "double m0 = (u - prev) * tot, m1 = (c - u) * tot;"),
    ("draft_margin_without_lower_edge", "*margin = m0 < m1 ? m0 : m1;", "*margin = m1;"),
    ("draft_margin_constant", "*margin = m0 < m1 ? m0 : m1;", "*margin = 1.0;"),
    ("greedy_margin_not_a_gap", "*gap = (V > 1) ? z[best] - second : INFINITY;",
     "*gap = (V > 1) ? z[best] : INFINITY;"),
    ("accept_margin_against_p_t", "margin_acc_out[o] = fabs(u_accept[o] - ratio);",
     "margin_acc_out[o] = fabs(u_accept[o] - pt);"),
    ("greedy_accept_margin_against_argmax", "margin_acc_out[o] = fabs(yt[xk] - best_other);",
     "margin_acc_out[o] = gap;"),
    ("admission_margin_absolute", "double rel = fabs(th1 - theta) / theta;", "double rel = fabs(th1 - theta);"),
    ("admission_margin_smallest_seen",
     "            if (margins_out) margins_out[n] = rel;\n"
     "            if (Vn1 * t0 < Vn * t1) { /* Theta_{n+1} < Theta_n: stop */\n"
     "                mtheta = rel;\n",
     "            if (margins_out) margins_out[n] = rel;\n"
     "            if (rel < mtheta) mtheta = rel;\n"
     "            if (Vn1 * t0 < Vn * t1) { /* Theta_{n+1} < Theta_n: stop */\n"),
]


@pytest.mark.parametrize("name,old,new", MARGIN_MUTANTS, ids=[m[0] for m in MARGIN_MUTANTS])
def test_margin_mutant_is_caught(tmp_path, name, old, new):
    import test_oracle_margins as pins
    so = _build_mutant(tmp_path, name, old, new)
    caught = []
    try:
        oracle.use_library(so)
        for pin, args in ((pins.test_draft_margin_is_the_distance_to_the_nearer_cdf_edge, (1.0,)),
                          (pins.test_draft_margin_near_each_edge, ()),
                          (pins.test_greedy_draft_margin_is_the_top_two_gap, ()),
                          (pins.test_accept_and_final_margins_follow_their_definitions, ()),
                          (pins.test_greedy_accept_margin_is_the_gap_to_the_best_other_logit, ()),
                          (pins.test_admission_margin_is_taken_at_the_stop_point, ()),
                          (pins.test_admission_margins_match_brute_force, (0,))):
            try:
                pin(*args)
            except AssertionError:
                caught.append(pin.__name__)
    finally:
        oracle.use_library(oracle.build())
    assert caught, f"no margin pin catches {name}"
