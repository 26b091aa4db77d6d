"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's formulas: they check it against library
routines (torch / scipy in fp64), exact enumeration of tiny rounds, brute
force, closed forms, invariants and the worked counterexample printed in the
paperlayer.ai summary (Appendix A).
"""
import itertools
import os

import numpy as np
import pytest
import scipy.special as sps
import torch

import enum_harness as eh
from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(s):
    return np.random.default_rng(s)


def _f32(a):
    return np.asarray(a, np.float32)


# --------------------------------------------------------------------------
# Drafting: Markov bias, temperature softmax, inverse CDF (library routines)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1.0, 0.7, 1.3])
def test_draft_matches_torch_softmax_and_cdf(T):
    rng = _rng(1)
    B, G, V, r = 6, 4, 97, 8
    L = _f32(rng.normal(0, 2, (B, G, V)))
    U = _f32(rng.normal(0, 0.5, (V, r)))
    W = _f32(rng.normal(0, 0.5, (r, V)))
    x0 = rng.integers(0, V, B).astype(np.int32)
    u = rng.random((B, G))
    res = oracle.draft(L, U, W, x0, np.full(B, T, np.float32), u)
    Ut, Wt, Lt = (torch.from_numpy(a.astype(np.float64)) for a in (U, W, L))
    T = float(np.float32(T))  # the oracle receives the temperature as fp32
    for b in range(B):
        prev = int(x0[b])
        for i in range(G):
            z = (Lt[b, i] + Ut[prev] @ Wt) / T          # library matmul
            p = torch.softmax(z, 0)                      # library softmax
            C = torch.cumsum(p, 0).numpy()
            x = int(res.x[b, i])
            lo = C[x - 1] if x > 0 else 0.0
            assert lo <= u[b, i] < C[x] + 1e-15
            assert res.pd[b, i] == pytest.approx(float(p[x]), rel=1e-12, abs=1e-300)
            assert res.rowmax[b, i] == pytest.approx(float(z.max()) * T, rel=1e-13)
            assert np.log(res.rowsum[b, i]) + res.rowmax[b, i] / T == pytest.approx(
                float(torch.logsumexp(z, 0)), rel=1e-12)
            prev = x


def test_draft_conditions_on_previous_sampled_token():
    """Position i's bias uses the token sampled at i-1 (x0 at i = 1): forcing
    a different x_1 must change row 2's distribution exactly as U[x_1] W says."""
    rng = _rng(2)
    V, r = 11, 3
    L = _f32(rng.normal(0, 1, (1, 2, V)))
    U = _f32(rng.normal(0, 1, (V, r)))
    W = _f32(rng.normal(0, 1, (r, V)))
    for forced in range(V):
        res = oracle.draft(L, U, W, np.array([4], np.int32), np.ones(1, np.float32),
                           np.array([[0.3, 0.6]]), force_x=np.array([[forced, -1]], np.int32))
        z = L[0, 1].astype(np.float64) + U[forced].astype(np.float64) @ W.astype(np.float64)
        p = sps.softmax(z)
        assert res.x[0, 0] == forced
        assert res.pd[0, 1] == pytest.approx(p[res.x[0, 1]], rel=1e-12)


def test_draft_zero_factor_is_plain_inverse_cdf_on_a_grid():
    """U = 0: the draft is plain inverse-CDF sampling of softmax(L/T).  Driving
    it with N evenly spaced uniforms gives every token N p_v draws, +-1."""
    rng = _rng(3)
    V, N, T = 9, 4000, float(np.float32(0.8))
    Lrow = _f32(rng.normal(0, 1.5, V))
    L = np.broadcast_to(Lrow, (N, 1, V))
    u = ((np.arange(N) + 0.5) / N)[:, None]
    res = oracle.draft(L, np.zeros((V, 2), np.float32), np.zeros((2, V), np.float32),
                       np.zeros(N, np.int32), np.full(N, T, np.float32), u)
    counts = np.bincount(res.x[:, 0], minlength=V)
    p = sps.softmax(Lrow.astype(np.float64) / T)
    assert np.all(np.abs(counts - N * p) <= 1.0)


def test_draft_greedy_is_argmax():
    rng = _rng(4)
    B, G, V, r = 5, 3, 50, 4
    L = _f32(rng.normal(0, 2, (B, G, V)))
    U = _f32(rng.normal(0, 1, (V, r)))
    W = _f32(rng.normal(0, 1, (r, V)))
    x0 = rng.integers(0, V, B).astype(np.int32)
    res = oracle.draft(L, U, W, x0, np.zeros(B, np.float32), rng.random((B, G)))
    for b in range(B):
        prev = x0[b]
        for i in range(G):
            z = L[b, i].astype(np.float64) + U[prev].astype(np.float64) @ W.astype(np.float64)
            assert res.x[b, i] == int(np.argmax(z))
            assert res.pd[b, i] == 1.0
            prev = res.x[b, i]


def test_draft_greedy_ties_take_lowest_index():
    L = np.zeros((1, 1, 6), np.float32)
    L[0, 0, [2, 4]] = 3.0
    res = oracle.draft(L, np.zeros((6, 1), np.float32), np.zeros((1, 6), np.float32),
                       np.zeros(1, np.int32), np.zeros(1, np.float32), np.zeros((1, 1)))
    assert res.x[0, 0] == 2 and res.margin[0, 0] == 0.0


# --------------------------------------------------------------------------
# Confidence head and prefix survival
# --------------------------------------------------------------------------

def test_confidence_matches_expit_and_cumprod():
    rng = _rng(5)
    B, G, d = 7, 6, 33
    h = _f32(rng.normal(0, 1, (B, G, d)))
    w = _f32(rng.normal(0, 0.3, d))
    tau = rng.uniform(0.5, 2.0, G)
    for t in (None, tau):
        c, S = oracle.confidence(h, w, 0.25, t)
        a = h.astype(np.float64) @ w.astype(np.float64) + 0.25
        if t is not None:
            a = a / t[None, :]
        np.testing.assert_allclose(c, sps.expit(a), rtol=1e-13)
        np.testing.assert_allclose(S, np.cumprod(sps.expit(a), axis=1), rtol=1e-13)
        assert np.all(np.diff(S, axis=1) <= 0)          # survival never increases
        assert np.all((S > 0) & (S < 1))


# --------------------------------------------------------------------------
# Scheduler (Algorithm 1)
# --------------------------------------------------------------------------

def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split("=", 1)
                vals[k.strip()] = [float(t) for t in v.split()]
    return vals


def _appendix_a():
    g = _read_golden("appendix_a_counterexample.txt")
    return g


@pytest.mark.parametrize("case", ["high", "low"])
def test_appendix_a_scheduler_values(case):
    """The worked counterexample: with early stop, l = 0 for both draws of x_1;
    offline search without it picks l = 2 when c_2 = 0.9 and l = 0 when c_2 = 0."""
    g = _appendix_a()
    a1 = g["a1"][0]
    c2 = g["c2_high"][0] if case == "high" else g["c2_low"][0]
    S = np.array([[a1, a1 * c2]])
    kn = np.array([0, 1, 2], np.int32)
    kt = np.array(g["t"], np.float64)
    es = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP)
    gs = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GLOBAL_ARGMAX)
    assert es.n_adm == int(g["ell_early_stop"][0]) and es.ell[0] == 0
    assert es.theta == pytest.approx(g["theta0"][0], abs=1e-15)
    assert gs.ell[0] == int(g[f"ell_global_{case}"][0])
    th2 = g[f"theta2_{case}"][0]
    all_ = oracle.schedule(S, kn, kt, -1, oracle.SCHED_ALL)
    assert all_.theta == pytest.approx(th2, rel=1e-6)
    one = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP, force_n=1)
    assert one.theta == pytest.approx(g["theta1"][0], rel=1e-12)


def _prefix_sets(B, G):
    """All admission sets that are a prefix of every request's block."""
    for ells in itertools.product(range(G + 1), repeat=B):
        yield ells


def _monotone_S(rng, B, G):
    return np.cumprod(rng.uniform(0.05, 1.0, (B, G)), axis=1)


def test_scheduler_topn_is_best_prefix_closed_set():
    """For every admitted size n, the globally sorted top-n reaches the largest
    total survival among all prefix-closed sets of that size (brute force)."""
    rng = _rng(6)
    for trial in range(40):
        B, G = rng.integers(1, 4), rng.integers(1, 4)
        S = _monotone_S(rng, B, G)
        best = {}
        for ells in _prefix_sets(B, G):
            n = sum(ells)
            tot = sum(S[b, :ells[b]].sum() for b in range(B))
            best[n] = max(best.get(n, -1), tot)
        kn = np.array([0], np.int32); kt = np.array([1.0])
        for n in range(B * G + 1):
            res = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP, force_n=n)
            got = sum(S[b, :res.ell[b]].sum() for b in range(B))
            assert got == pytest.approx(best[n], rel=1e-12)
            assert res.ell.sum() == n


def _convex_profile(rng):
    slopes = np.sort(rng.uniform(0.01, 2.0, 3))
    kn = np.array([0, 2, 4, 7], np.int32)
    kt = np.concatenate([[rng.uniform(1, 20)], np.zeros(3)])
    for j in range(1, 4):
        kt[j] = kt[j - 1] + slopes[j - 1] * (kn[j] - kn[j - 1])
    return kn, kt


def _t_of(kn, kt, n):
    """Library interpolation of the profile (numpy), continued with the last slope."""
    if n <= kn[-1]:
        return float(np.interp(n, kn, kt))
    s = (kt[-1] - kt[-2]) / (kn[-1] - kn[-2])
    return float(kt[-1] + (n - kn[-1]) * s)


def test_scheduler_early_stop_is_global_optimum_for_convex_profiles():
    """Theta(n) = (B + best survival mass of size n) / t(n) is quasi-concave when
    t is convex, so the first decrease is the global maximum (brute force)."""
    rng = _rng(7)
    for trial in range(60):
        B, G = int(rng.integers(1, 4)), int(rng.integers(1, 4))
        S = _monotone_S(rng, B, G)
        kn, kt = _convex_profile(rng)
        best = {}
        for ells in _prefix_sets(B, G):
            n = sum(ells)
            best[n] = max(best.get(n, -1), sum(S[b, :ells[b]].sum() for b in range(B)))
        theta = [(B + best[n]) / _t_of(kn, kt, n) for n in range(B * G + 1)]
        res = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP)
        assert res.n_adm == int(np.argmax(theta))
        assert res.theta == pytest.approx(max(theta), rel=1e-12)


def test_scheduler_profile_and_budget():
    rng = _rng(8)
    B, G = 5, 4
    S = _monotone_S(rng, B, G)
    kn = np.array([0, 3, 6], np.int32); kt = np.array([2.0, 2.3, 3.5])
    for n in range(B * G + 1):
        res = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP, force_n=n)
        mass = B + sum(S[b, :res.ell[b]].sum() for b in range(B))
        assert res.theta == pytest.approx(mass / _t_of(kn, kt, n), rel=1e-12)
    flat = np.array([0], np.int32), np.array([1.0])
    for budget in range(0, B * G + 1):
        res = oracle.schedule(S, *flat, budget, oracle.SCHED_GREEDY_EARLY_STOP)
        assert res.n_adm == min(budget, B * G)   # a flat profile admits all it may
    res = oracle.schedule(S, *flat, -1, oracle.SCHED_ALL)
    assert np.all(res.ell == G)


def test_scheduler_prefix_property_with_ties():
    """Equal survivals (c = 1 somewhere) still give prefix-closed admissions."""
    rng = _rng(9)
    for trial in range(50):
        B, G = int(rng.integers(1, 6)), int(rng.integers(1, 6))
        c = rng.choice([1.0, 0.5, 0.25], size=(B, G))
        S = np.cumprod(c, axis=1)
        for n in range(B * G + 1):
            res = oracle.schedule(S, np.array([0], np.int32), np.array([1.0]), -1,
                                  oracle.SCHED_GREEDY_EARLY_STOP, force_n=n)
            adm = set(int(i) for i in res.order[:n])
            for b in range(B):
                pos = sorted(i // B for i in adm if i % B == b)
                assert pos == list(range(len(pos)))
                assert len(pos) == res.ell[b]


def test_scheduler_non_anticipation():
    """Whether (b, k) is admitted never depends on survivals of later positions
    of the same request (perturbed keeping S monotone)."""
    rng = _rng(10)
    for trial in range(60):
        B, G = int(rng.integers(1, 5)), int(rng.integers(2, 5))
        S = _monotone_S(rng, B, G)
        kn, kt = _convex_profile(rng)
        res = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP)
        b = int(rng.integers(0, B)); k = int(rng.integers(0, G - 1))
        S2 = S.copy()
        S2[b, k + 1:] = S[b, k] * np.cumprod(rng.uniform(0.0, 1.0, G - k - 1))
        res2 = oracle.schedule(S2, kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP)
        assert (res.ell[b] > k) == (res2.ell[b] > k)


def test_scheduler_global_search_maximises_theta():
    """The offline-search variant admits the count that maximises Theta over
    every n (the lowest such n), whatever the profile's shape (brute force over
    prefix-closed sets; non-convex step profiles included)."""
    rng = _rng(11)
    for trial in range(60):
        B, G = int(rng.integers(1, 4)), int(rng.integers(1, 4))
        S = _monotone_S(rng, B, G)
        if trial % 2:
            kn, kt = _convex_profile(rng)
        else:   # a step-shaped, non-convex profile
            kn = np.array([0, 1, 2, 3], np.int32)
            kt = np.array([1.0, 1.0 + rng.uniform(0, 2), 3.2, 3.3])
        best = {}
        for ells in _prefix_sets(B, G):
            n = sum(ells)
            best[n] = max(best.get(n, -1), sum(S[b, :ells[b]].sum() for b in range(B)))
        theta = [(B + best[n]) / _t_of(kn, kt, n) for n in range(B * G + 1)]
        res = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GLOBAL_ARGMAX)
        assert res.n_adm == int(np.argmax(theta))
        assert res.theta == pytest.approx(max(theta), rel=1e-12)


def test_scheduler_threshold_is_the_survival_cut():
    """Static-threshold pruning admits exactly the candidates with S >= the
    threshold (all of them, or the first `budget` in the stable order), which
    for monotone survivals are prefixes of every request."""
    rng = _rng(12)
    for trial in range(80):
        B, G = int(rng.integers(1, 6)), int(rng.integers(1, 6))
        c = rng.choice([1.0, 0.9, 0.5, 0.25], size=(B, G))
        S = np.cumprod(c, axis=1)
        th = float(rng.choice(S.ravel())) if trial % 3 else float(rng.uniform(0, 1))
        budget = -1 if trial % 4 else int(rng.integers(0, B * G + 1))
        ell, n_adm, order = oracle.schedule_threshold(S, th, budget)
        # The stable order by S descending over the position-major list.
        ids = sorted(range(B * G), key=lambda i: (-S[i % B, i // B], i))
        assert list(order) == ids
        above = [i for i in ids if S[i % B, i // B] >= th]
        take = above if budget < 0 else above[:budget]
        assert n_adm == len(take)
        for b in range(B):
            assert ell[b] == sum(1 for i in take if i % B == b)
            assert all(S[b, k] >= th for k in range(ell[b]))   # a prefix of the request
            if budget < 0:
                assert all(S[b, k] < th for k in range(ell[b], G))


def test_scheduler_topk_is_the_first_k_of_the_stable_order():
    """Dynamic top-K admits the first K candidates of the stable order by S
    descending (Python's sort as the reference), clamped to [0, B*G] and to the
    budget; with monotone survivals every request's admitted set is a prefix."""
    rng = _rng(13)
    for trial in range(80):
        B, G = int(rng.integers(1, 6)), int(rng.integers(1, 6))
        c = rng.choice([1.0, 0.9, 0.5, 0.25], size=(B, G))
        S = np.cumprod(c, axis=1)
        cap = int(rng.integers(-2, B * G + 3))
        budget = -1 if trial % 4 else int(rng.integers(0, B * G + 1))
        ell, n_adm, order = oracle.schedule_topk(S, cap, budget)
        ids = sorted(range(B * G), key=lambda i: (-S[i % B, i // B], i))
        assert list(order) == ids
        k = min(max(cap, 0), B * G)
        if budget >= 0:
            k = min(k, budget)
        take = ids[:k]
        assert n_adm == k
        for b in range(B):
            assert ell[b] == sum(1 for i in take if i % B == b)
            admitted = {i // B for i in take if i % B == b}
            assert admitted == set(range(ell[b]))              # a prefix of the request


def test_scheduler_topk_with_the_greedy_count_is_the_greedy_schedule():
    """With K equal to Algorithm 1's admitted count on the same survivals, the
    top-K selection admits exactly Algorithm 1's set (both are prefixes of the
    same stable order), and with the global search's count, that search's set."""
    rng = _rng(14)
    for trial in range(40):
        B, G = int(rng.integers(1, 9)), int(rng.integers(1, 6))
        S = _monotone_S(rng, B, G)
        kn, kt = _convex_profile(rng)
        for mode in (oracle.SCHED_GREEDY_EARLY_STOP, oracle.SCHED_GLOBAL_ARGMAX):
            res = oracle.schedule(S, kn, kt, -1, mode)
            ell, n_adm, order = oracle.schedule_topk(S, res.n_adm)
            assert n_adm == res.n_adm and np.array_equal(ell, res.ell) and np.array_equal(order, res.order)


def test_production_schedule_takes_its_capacity_from_the_previous_round():
    """The production form's admitted count depends on the previous round
    only: changing the current round's survivals changes which candidates are
    admitted, never how many."""
    rng = _rng(15)
    kn, kt = np.array([0, 4, 8], np.int32), np.array([10.0, 10.5, 30.0])   # a step in capacity
    for trial in range(30):
        B, G = int(rng.integers(2, 7)), int(rng.integers(1, 5))
        S_prev = _monotone_S(rng, B, G)
        cap, _, n1, _ = oracle.production_schedule(S_prev, _monotone_S(rng, B, G), kn, kt)
        _, _, n2, _ = oracle.production_schedule(S_prev, _monotone_S(rng, B, G), kn, kt)
        assert n1 == n2 == min(cap, B * G)
        assert cap == oracle.schedule(S_prev, kn, kt, -1, oracle.SCHED_GLOBAL_ARGMAX).n_adm


# --------------------------------------------------------------------------
# Verification
# --------------------------------------------------------------------------

def test_verify_identical_draft_and_target_accepts_all():
    """p_d = p_t: every admitted token is accepted and the bonus row is drawn."""
    rng = _rng(11)
    B, G, V = 8, 4, 30
    base = _f32(rng.normal(0, 2, (B, G + 1, V)))
    L = base[:, :G].copy()
    zU = np.zeros((V, 2), np.float32); zW = np.zeros((2, V), np.float32)
    x0 = np.zeros(B, np.int32); temp = np.full(B, 0.9, np.float32)
    dr = oracle.draft(L, zU, zW, x0, temp, rng.random((B, G)))
    ell = rng.integers(0, G + 1, B).astype(np.int32)
    vr = oracle.verify(base, L, zU, zW, x0, dr.x, temp, rng.random((B, G)) * 0.999999,
                       rng.random(B), ell)
    assert np.all(vr.acc == ell) and np.all(vr.final_kind == 1)
    for b in range(B):
        assert list(vr.tokens[b, :ell[b]]) == list(dr.x[b, :ell[b]])
        p = sps.softmax(base[b, ell[b]].astype(np.float64) / 0.9)
        np.testing.assert_allclose(vr.pt_x[b, :ell[b]], vr.pd_x[b, :ell[b]], rtol=1e-13)


def test_verify_greedy_exact_match():
    rng = _rng(12)
    B, G, V = 10, 5, 20
    base = _f32(rng.normal(0, 2, (B, G + 1, V)))
    Tl = base.copy()
    L = base[:, :G].copy()
    L[:, 2] += _f32(rng.normal(0, 3, (B, V)))          # position 3 often disagrees
    zU = np.zeros((V, 1), np.float32); zW = np.zeros((1, V), np.float32)
    dr = oracle.draft(L, zU, zW, np.zeros(B, np.int32), np.zeros(B, np.float32), np.zeros((B, G)))
    ell = np.full(B, G, np.int32)
    vr = oracle.verify(Tl, L, zU, zW, np.zeros(B, np.int32), dr.x, np.zeros(B, np.float32),
                       np.zeros((B, G)), np.zeros(B), ell)
    for b in range(B):
        am = np.argmax(Tl[b], axis=1)
        A = 0
        while A < G and am[A] == dr.x[b, A]:
            A += 1
        assert vr.acc[b] == A and vr.tokens[b, A] == am[A] and vr.final_kind[b] == 2
        assert list(vr.tokens[b, :A]) == list(dr.x[b, :A])
        assert np.all(vr.tokens[b, A + 1:] == -1)


def test_verify_acceptance_closed_form():
    """With no Markov bias and prefix-free target rows, the chance that x_k is
    accepted is sum_v min(p_t, p_d) = 1 - TV, and E[A] = sum_k prod_{i<=k} alpha_i
    (exact enumeration)."""
    rng = _rng(13)
    V, G, T = 5, 3, 1.0
    Lrows = _f32(rng.normal(0, 1.5, (G, V)))
    rows = [_f32(Lrows[k] + rng.normal(0, 0.6 * (k + 1), V)).astype(np.float64) for k in range(G)]
    rows.append(_f32(rng.normal(0, 1, V)).astype(np.float64))
    target = {p: rows[len(p)] for n in range(G + 1) for p in itertools.product(range(V), repeat=n)}
    sc = eh.Scenario(Lrows, np.zeros((V, 1)), np.zeros((1, V)), 0, T, target, ell_fixed=G)
    law = sc.output_law()
    alpha = [np.minimum(sps.softmax(rows[k] / T), sps.softmax(Lrows[k].astype(np.float64) / T)).sum()
             for k in range(G)]
    EA = sum(p * (len(o) - 1) for o, p in law.items())
    assert EA == pytest.approx(sum(np.prod(alpha[:k + 1]) for k in range(G)), abs=1e-12)
    P1 = sum(p for o, p in law.items() if len(o) > 1)
    assert P1 == pytest.approx(alpha[0], abs=1e-12)
    assert sum(law.values()) == pytest.approx(1.0, abs=1e-12)


@pytest.mark.parametrize("V,G,r,T,seed", [(2, 3, 1, 1.0, 20), (3, 3, 2, 1.0, 21), (4, 2, 3, 0.7, 22),
                                          (6, 2, 2, 1.4, 23), (5, 3, 2, 1.0, 24)])
def test_distribution_preservation_exhaustive(V, G, r, T, seed):
    """Exact law of the emitted tokens over every draft path and every accept /
    reject / residual / bonus outcome: each emitted token, given the emitted
    prefix, follows the target's distribution (the lossless claim)."""
    rng = _rng(seed)
    T = float(np.float32(T))  # the oracle receives the temperature as fp32
    Lrows = _f32(rng.normal(0, 1.5, (G, V)))
    U = _f32(rng.normal(0, 1.0, (V, r)))
    W = _f32(rng.normal(0, 1.0, (r, V)))
    target = eh.random_target(rng, V, G)
    for ell in range(G + 1):
        sc = eh.Scenario(Lrows, U, W, int(rng.integers(0, V)), T, target, ell_fixed=ell)
        law = sc.output_law()
        assert sum(law.values()) == pytest.approx(1.0, abs=1e-12)
        assert eh.preservation_error(law, target, T, V) < 1e-12


def test_distribution_preservation_greedy():
    """T = 0: the output is the target's greedy continuation of the accepted prefix."""
    rng = _rng(25)
    V, G = 4, 3
    target = eh.random_target(rng, V, G)
    for trial in range(10):
        Lrows = _f32(rng.normal(0, 1.5, (G, V)))
        U = _f32(rng.normal(0, 1, (V, 2))); W = _f32(rng.normal(0, 1, (2, V)))
        x0 = int(rng.integers(0, V))
        dr = oracle.draft(Lrows[None], U, W, np.array([x0], np.int32), np.zeros(1, np.float32),
                          np.zeros((1, G)))
        x = tuple(int(t) for t in dr.x[0])
        Tl = np.stack([target[x[:k]] for k in range(G + 1)])[None]
        vr = oracle.verify(Tl, Lrows[None], U, W, np.array([x0], np.int32), dr.x,
                           np.zeros(1, np.float32), np.zeros((1, G)), np.zeros(1),
                           np.array([G], np.int32))
        out = tuple(int(t) for t in vr.tokens[0, :vr.nout[0]])
        for j, z in enumerate(out):
            assert z == int(np.argmax(target[out[:j]]))


def _appendix_a_scenario(mode):
    """The counterexample as a two-token round (A = 0, B = 1): p_t = (0.5, 0.5),
    p_d = (0.7, 0.3), so a_1 = sum min = 0.8 = S_1; c_2 = 0.9 after x_1 = A and
    ~0 after x_1 = B (a Markov confidence head); profile t(0), t(1), t(2) from
    the golden file."""
    g = _appendix_a()
    pd = np.array(g["p_d"]); pt = np.array(g["p_t"])
    Lrows = np.stack([np.log(pd), np.log(pd)]).astype(np.float32)
    target = {p: np.log(pt).astype(np.float32).astype(np.float64)
              for n in range(3) for p in itertools.product(range(2), repeat=n)}
    a1, c2h = g["a1"][0], g["c2_high"][0]
    logit = lambda p: float(np.log(p / (1 - p)))
    Htab = np.array([[[logit(a1)], [logit(a1)]],        # position 1: c_1 = a_1 whatever x_0
                     [[logit(c2h)], [-60.0]]],          # position 2: c_2 depends on x_1
                    np.float32)
    U = np.zeros((2, 1), np.float32); W = np.zeros((1, 2), np.float32)
    sc = eh.Scenario(Lrows, U, W, 0, 1.0, target, hconf=(Htab, np.ones(1, np.float32), 0.0),
                     knots_n=np.array([0, 1, 2], np.int32), knots_t=np.array(g["t"]), mode=mode)
    return sc, target, g


def _first_token_law(law):
    first = np.zeros(2)
    for o, p in law.items():
        first[o[0]] += p
    return first


def test_appendix_a_early_stop_is_lossless():
    sc, target, g = _appendix_a_scenario(oracle.SCHED_GREEDY_EARLY_STOP)
    assert {sc.ell_for(p) for p in sc.draft_paths()} == {int(g["ell_early_stop"][0])}
    law = sc.output_law()
    np.testing.assert_allclose(_first_token_law(law), g["first_token_early_stop"], atol=1e-7)
    assert eh.preservation_error(law, target, 1.0, 2) < 1e-12


def test_appendix_a_global_search_is_biased():
    """Negative control: the offline search without early stop lets x_1 leak
    into its own admission, and the first emitted token is no longer p_t."""
    sc, target, g = _appendix_a_scenario(oracle.SCHED_GLOBAL_ARGMAX)
    assert sc.ell_for((0, 0)) == int(g["ell_global_high"][0])
    assert sc.ell_for((1, 0)) == int(g["ell_global_low"][0])
    law = sc.output_law()
    np.testing.assert_allclose(_first_token_law(law), g["first_token_global"], atol=1e-7)
    assert eh.preservation_error(law, target, 1.0, 2) > 0.1


@pytest.mark.parametrize("seed", [30, 31, 32])
def test_distribution_preservation_with_scheduler_in_the_loop(seed):
    """Markov confidence (hidden state a function of x_{k-1}) feeding the
    early-stop scheduler, with other requests competing for the budget: the
    round stays lossless for whatever prefix length it picks."""
    rng = _rng(seed)
    V, G, d = 3, 3, 2
    Lrows = _f32(rng.normal(0, 1.5, (G, V)))
    U = _f32(rng.normal(0, 1, (V, 2))); W = _f32(rng.normal(0, 1, (2, V)))
    target = eh.random_target(rng, V, G)
    Htab = _f32(rng.normal(0, 2, (G, V, d)))
    w = _f32(rng.normal(0, 1, d))
    others = np.cumprod(rng.uniform(0.3, 1.0, (3, G)), axis=1)
    kn = np.array([0, 2, 5], np.int32); kt = np.array([3.0, 3.4, 5.0])
    sc = eh.Scenario(Lrows, U, W, int(rng.integers(0, V)), 1.0, target, hconf=(Htab, w, 0.1),
                     knots_n=kn, knots_t=kt, mode=oracle.SCHED_GREEDY_EARLY_STOP, others_S=others)
    ells = {sc.ell_for(p) for p in sc.draft_paths()}
    law = sc.output_law()
    assert eh.preservation_error(law, target, 1.0, V) < 1e-12
    assert len(ells) >= 1
