"""Pins of the oracle's decision margins.

Every GPU/oracle disagreement the parity tests excuse rests on a margin the
oracle reports: how far the decision's uniform (or logit) lies from the
threshold that would flip it.  These tests recompute each margin from its
definition with library routines in fp64 (torch softmax and cumsum, top-k)
and with brute force for the scheduler, so that a margin in the wrong units,
one that ignores an edge of the interval, or one taken at the wrong
comparison fails here:

  draws (inverse CDF): min(u - C_{x-1}, C_x - u) on the normalised CDF of the
      distribution drawn from (C_{-1} = 0);
  argmax (T = 0): the gap between the largest and the second-largest logit;
  accept test: |u - p_t(x) / p_d(x)|; greedy accept: the gap between the
      drafted token's target logit and the best other one;
  admission: the relative objective change |Theta_{n+1} - Theta_n| / Theta_n
      at the comparison that stopped the early-stop scan, and at every
      comparison it made.

(paperlayer.ai summary of DSpark, §3.1 for the draws and Appendix A for the
early stop; menfem.com KB entry, "Methodology", for the accept test.)
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from speculative_decoding_draft_rank_b200 import synth


def _cdf_margin(p, u):
    """Inverse-CDF draw from probabilities p (fp64 torch) at u: the token and
    its margin, from torch.cumsum."""
    C = torch.cumsum(p / p.sum(), 0).numpy()
    x = int(np.searchsorted(C, u, side="right"))
    x = min(x, len(C) - 1)
    lo = C[x - 1] if x > 0 else 0.0
    return x, min(u - lo, C[x] - u)


def _draft_case(seed, T):
    rng = np.random.default_rng(seed)
    B, G, V, r = 5, 3, 61, 8
    L = rng.normal(0, 2, (B, G, V)).astype(np.float32)
    U = rng.normal(0, 0.5, (V, r)).astype(np.float32)
    W = rng.normal(0, 0.5, (r, V)).astype(np.float32)
    x0 = rng.integers(0, V, B).astype(np.int32)
    return L, U, W, x0, np.full(B, T, np.float32), rng.random((B, G))


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_draft_margin_is_the_distance_to_the_nearer_cdf_edge(T):
    L, U, W, x0, temp, u = _draft_case(3, T)
    B, G, V = L.shape
    res = oracle.draft(L, U, W, x0, temp, u)
    Lt, Ut, Wt = (torch.from_numpy(a.astype(np.float64)) for a in (L, U, W))
    Tf = float(np.float32(T))
    for b in range(B):
        prev = int(x0[b])
        for i in range(G):
            p = torch.softmax((Lt[b, i] + Ut[prev] @ Wt) / Tf, 0)
            x, m = _cdf_margin(p, u[b, i])
            assert x == res.x[b, i]
            assert res.margin[b, i] == pytest.approx(m, rel=1e-9, abs=1e-15)
            prev = x


def test_draft_margin_near_each_edge():
    """Uniforms placed just inside the lower and just below the upper edge of
    a token's CDF interval give margins of that size (in CDF units)."""
    L, U, W, x0, temp, _ = _draft_case(4, 1.0)
    L, x0, temp = L[:1, :1], x0[:1], temp[:1]
    Lt, Ut, Wt = (torch.from_numpy(a.astype(np.float64)) for a in (L, U, W))
    p = torch.softmax(Lt[0, 0] + Ut[int(x0[0])] @ Wt, 0)
    C = torch.cumsum(p, 0).numpy()
    k = int(np.argmax(p.numpy()))          # a wide interval [C_{k-1}, C_k)
    lo = C[k - 1] if k > 0 else 0.0
    for u, want in ((lo + 3e-7, 3e-7), (C[k] - 5e-7, 5e-7), ((lo + C[k]) / 2, (C[k] - lo) / 2)):
        res = oracle.draft(L, U, W, x0, temp, np.array([[u]]))
        assert res.x[0, 0] == k
        assert res.margin[0, 0] == pytest.approx(want, rel=1e-6)


def test_greedy_draft_margin_is_the_top_two_gap():
    L, U, W, x0, temp, u = _draft_case(5, 0.0)
    res = oracle.draft(L, U, W, x0, temp, u)
    Lt, Ut, Wt = (torch.from_numpy(a.astype(np.float64)) for a in (L, U, W))
    B, G, _ = L.shape
    for b in range(B):
        prev = int(x0[b])
        for i in range(G):
            y = Lt[b, i] + Ut[prev] @ Wt
            top = torch.topk(y, 2).values
            assert res.margin[b, i] == pytest.approx(float(top[0] - top[1]), rel=1e-12)
            prev = int(res.x[b, i])


def _verify_case(seed, temps):
    B = len(temps)
    inp = synth.generate(B, 3, 48, 8, 8, "f32", seed=seed, hot=2, sigma_t=0.8, temps=np.float32(temps))
    d = oracle.draft(inp.L, inp.U, inp.W, inp.x0, inp.temp, inp.u_draft.astype(np.float64))
    ell = np.full(B, 3, np.int32)
    v = oracle.verify(inp.Tlog, inp.L, inp.U, inp.W, inp.x0, d.x, inp.temp, inp.u_accept.astype(np.float64),
                      inp.u_final.astype(np.float64), ell)
    return inp, d, ell, v


def test_accept_and_final_margins_follow_their_definitions():
    temps = [1.0, 0.8, 1.2] * 4
    inp, d, ell, v = _verify_case(21, temps)
    B, G = d.x.shape
    ua, uf = inp.u_accept.astype(np.float64), inp.u_final.astype(np.float64)
    Lt, Ut, Wt, Tt = (torch.from_numpy(a.astype(np.float64)) for a in (inp.L, inp.U, inp.W, inp.Tlog))
    kinds = set()
    for b in range(B):
        T = float(inp.temp[b])
        prevs = [int(inp.x0[b])] + [int(t) for t in d.x[b]]
        pd_rows, pt_rows = [], []
        for k in range(G + 1):
            pt_rows.append(torch.softmax(Tt[b, k] / T, 0))
            if k < G:
                pd_rows.append(torch.softmax((Lt[b, k] + Ut[prevs[k]] @ Wt) / T, 0))
        for k in range(int(ell[b])):
            x = int(d.x[b, k])
            ratio = float(pt_rows[k][x] / pd_rows[k][x])
            assert v.margin_acc[b, k] == pytest.approx(abs(ua[b, k] - ratio), rel=1e-9, abs=1e-15)
        A = int(v.acc[b])
        if A < ell[b]:
            q = torch.clamp(pt_rows[A] - pd_rows[A], min=0.0)
            y, m = _cdf_margin(q, uf[b])
            kinds.add(0)
        else:
            y, m = _cdf_margin(pt_rows[A], uf[b])
            kinds.add(1)
        assert v.tokens[b, A] == y
        assert v.margin_fin[b] == pytest.approx(m, rel=1e-9, abs=1e-15)
    assert kinds == {0, 1}, "the case must hold both residual and bonus draws"


def test_greedy_accept_margin_is_the_gap_to_the_best_other_logit():
    inp, d, ell, v = _verify_case(22, [0.0] * 8)
    B, G = d.x.shape
    for b in range(B):
        for k in range(G):
            y = inp.Tlog[b, k].astype(np.float64)
            x = int(d.x[b, k])
            other = np.delete(y, x).max()
            assert v.margin_acc[b, k] == pytest.approx(abs(y[x] - other), rel=1e-12)


def _theta_scan(S, kn, kt, budget):
    """Brute force of the early stop: sorted survivals, Theta at every count,
    the stop point and the relative change of every comparison."""
    B, G = S.shape
    cand = sorted(((-S[b, i], i * B + b) for i in range(G) for b in range(B)))
    s = np.array([-c[0] for c in cand])
    t = np.interp(np.arange(len(s) + 1), kn, kt, right=None)
    n_last = len(s) if budget < 0 else min(budget, len(s))
    # Extrapolate past the last knot with the last slope.
    if len(kn) > 1:
        slope = (kt[-1] - kt[-2]) / (kn[-1] - kn[-2])
        beyond = np.arange(len(s) + 1) > kn[-1]
        t[beyond] = kt[-1] + (np.arange(len(s) + 1)[beyond] - kn[-1]) * slope
    V = B + np.concatenate([[0.0], np.cumsum(s)])
    theta = V / t
    rel, stop = [], None
    for n in range(n_last):
        rel.append(abs(theta[n + 1] - theta[n]) / theta[n])
        if theta[n + 1] < theta[n]:
            stop = n
            break
    return stop, np.array(rel)


def test_admission_margin_is_taken_at_the_stop_point():
    """A profile whose first comparison is nearly flat (Theta_1 just above
    Theta_0) and whose stop is a clear drop: the margin is the drop's, not the
    smallest change seen on the way."""
    S = np.array([[0.5, 0.49, 0.05]])
    kn = np.array([0, 1, 2, 3], np.int32)
    kt = np.array([1.0, 1.5 - 1e-7, 1.9, 3.0])
    stop, rel = _theta_scan(S, kn, kt, -1)
    assert stop == 2 and rel[0] < 1e-6 < rel[2]
    o = oracle.schedule(S, kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP)
    assert o.n_adm == 2
    assert o.margin_theta == pytest.approx(rel[2], rel=1e-12)
    assert np.allclose(o.margins[:3], rel, rtol=1e-12, atol=0)
    assert np.all(np.isnan(o.margins[3:]))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_admission_margins_match_brute_force(seed):
    rng = np.random.default_rng(seed)
    B, G = 7, 4
    S = np.cumprod(rng.uniform(0.4, 1.0, (B, G)), axis=1)
    kn = np.array([0, 6, 12, 20], np.int32)
    kt = np.array([5.0, 6.0, 8.5, 14.0])
    for budget in (-1, 9):
        stop, rel = _theta_scan(S, kn, kt, budget)
        o = oracle.schedule(S, kn, kt, budget, oracle.SCHED_GREEDY_EARLY_STOP)
        made = len(rel)
        assert np.allclose(o.margins[:made], rel, rtol=1e-12, atol=0)
        assert np.all(np.isnan(o.margins[made:]))
        if stop is None:
            assert o.margin_theta == np.inf
        else:
            assert o.n_adm == stop
            assert o.margin_theta == pytest.approx(rel[stop], rel=1e-12)
