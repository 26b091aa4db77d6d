"""Exhaustive enumeration of one round on a tiny vocabulary.

Every random decision of a round is a monotone step function of one supplied
uniform: inverse-CDF draws are non-decreasing in u, and the accept test is
"accept iff u < threshold".  The harness finds each step's breakpoints by
bisection, calling the oracle as a black box, and so obtains the exact
probability (to ~1e-16) of every interval of every uniform.  Weighting each
outcome by its interval lengths gives the exact law of the emitted tokens,
without re-deriving any of the oracle's arithmetic.

The scenario: a draft block of G positions over a V-token vocabulary, a
target model given as a table of logit rows indexed by the token prefix
(so row k depends only on x_1..x_{k-1}, as a causal target does), and
optionally a confidence head whose hidden state at position k is a table row
indexed by (k, x_{k-1}) (the Markov confidence of the counterexample in the
paperlayer.ai summary, Appendix A) feeding the scheduler.
"""
from __future__ import annotations

import itertools

import numpy as np

from oracle import oracle

ITERS = 64


def _bisect(evaluate, ntracks_q, nvals, iters=ITERS):
    """Breakpoints of ntracks_q monotone step functions with values in
    0..nvals-1.  evaluate(q_index[], v_index[], u[]) -> outputs[].
    Returns (probs [q, nvals], mids [q, nvals])."""
    q = np.repeat(np.arange(ntracks_q), nvals - 1)
    v = np.tile(np.arange(nvals - 1), ntracks_q)
    lo = np.zeros(q.size)
    hi = np.ones(q.size)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        out = evaluate(q, v, mid)
        gt = out > v
        hi = np.where(gt, mid, hi)
        lo = np.where(gt, lo, mid)
    b = hi.reshape(ntracks_q, nvals - 1)
    edges = np.concatenate([np.zeros((ntracks_q, 1)), b, np.ones((ntracks_q, 1))], axis=1)
    return np.diff(edges, axis=1), 0.5 * (edges[:, :-1] + edges[:, 1:])


class Scenario:
    """Tables of one tiny round.  Lrows [G, V] backbone logits, U [V, r],
    W [r, V], x0, T, target: dict prefix-tuple -> logits [V] (every prefix of
    length 0..G), hconf: None or (Htab [G, V, d], w [d], bias) with the hidden
    state at position k equal to Htab[k-1, x_{k-1}], and the scheduler setup."""

    def __init__(self, Lrows, U, W, x0, T, target, hconf=None, knots_n=None, knots_t=None,
                 budget=-1, mode=oracle.SCHED_ALL, others_S=None, ell_fixed=None, A=None):
        self.Lrows = np.asarray(Lrows, np.float32)
        self.G, self.V = self.Lrows.shape
        self.U = np.asarray(U, np.float32)
        self.W = np.asarray(W, np.float32)
        self.x0 = int(x0)
        self.T = float(T)
        self.target = target
        self.hconf = hconf
        self.knots_n = knots_n
        self.knots_t = knots_t
        self.budget = budget
        self.mode = mode
        self.others_S = others_S  # [B_other, G] fixed survivals of other requests
        self.ell_fixed = ell_fixed
        self.A = None if A is None else np.asarray(A, np.float32)   # RNN head (None: Markov head)

    # -- drafting -------------------------------------------------------
    def _draft(self, u_rows, force=None):
        n = u_rows.shape[0]
        L = np.broadcast_to(self.Lrows, (n, self.G, self.V))
        return oracle.draft(L, self.U, self.W, np.full(n, self.x0, np.int32),
                            np.full(n, self.T, np.float32), u_rows, force_x=force, A=self.A)

    def draft_paths(self):
        """All draft paths with probabilities and uniforms realising them."""
        G, V = self.G, self.V
        paths = {(): (1.0, [])}
        for i in range(G):
            keys = list(paths.keys())
            base_u = np.full((len(keys), G), 0.5)
            for j, k in enumerate(keys):
                base_u[j, :i] = paths[k][1]

            def ev(q, v, u):
                rows = base_u[q].copy()
                rows[:, i] = u
                return self._draft(rows).x[:, i]

            probs, mids = _bisect(ev, len(keys), V)
            new = {}
            for j, k in enumerate(keys):
                p0, us = paths[k]
                for x in range(V):
                    if probs[j, x] > 0:
                        new[k + (x,)] = (p0 * probs[j, x], us + [mids[j, x]])
            paths = new
        return paths

    # -- confidence + scheduler -----------------------------------------
    def ell_for(self, path):
        if self.ell_fixed is not None:
            return int(self.ell_fixed)
        Htab, w, bias = self.hconf
        prev = (self.x0,) + tuple(path[:-1])
        h = np.stack([Htab[k, p] for k, p in enumerate(prev)])[None]
        _, S = oracle.confidence(h, w, bias)
        if self.others_S is not None:
            S = np.concatenate([S, np.asarray(self.others_S, np.float64)], axis=0)
        res = oracle.schedule(S, self.knots_n, self.knots_t, self.budget, self.mode)
        return int(res.ell[0])

    # -- verification ---------------------------------------------------
    def _tlog(self, path):
        return np.stack([self.target[tuple(path[:k])] for k in range(self.G + 1)])

    def output_law(self):
        """dict emitted-token tuple -> probability."""
        G, V = self.G, self.V
        paths = self.draft_paths()
        keys = list(paths.keys())
        n = len(keys)
        X = np.asarray(keys, np.int32).reshape(n, G)
        Tl = np.stack([self._tlog(k) for k in keys]).astype(np.float32)
        L = np.broadcast_to(self.Lrows, (n, G, V))
        ell = np.asarray([self.ell_for(k) for k in keys], np.int32)
        x0 = np.full(n, self.x0, np.int32)
        temp = np.full(n, self.T, np.float32)

        def run(idx, ua, uf):
            return oracle.verify(Tl[idx], L[idx], self.U, self.W, x0[idx], X[idx], temp[idx],
                                 ua, uf, ell[idx], A=self.A)

        # Accept thresholds per (path, k): probability that x_k is accepted
        # given x_1..x_{k-1} were.
        racc = np.ones((n, G))
        for k in range(G):
            live = np.nonzero(ell > k)[0]
            if live.size == 0:
                continue

            def ev(q, v, u):
                ua = np.full((q.size, G), 0.5)
                ua[:, :k] = 0.0
                ua[:, k] = u
                res = run(live[q], ua, np.full(q.size, 0.5))
                return (res.acc <= k).astype(np.int64)  # 0 accept, 1 reject

            probs, _ = _bisect(ev, live.size, 2)
            racc[live, k] = probs[:, 0]

        law = {}
        tracks = []  # (path index, A, probability of (path, A), uniforms realising A)
        for pi in range(n):
            pa = paths[keys[pi]][0]
            run_p = 1.0
            for A in range(ell[pi] + 1):
                if A < ell[pi]:
                    pA = run_p * (1.0 - racc[pi, A])
                    ua = np.zeros(G)
                    ua[A] = 0.5 * (racc[pi, A] + 1.0)
                    ua[A + 1:] = 0.5
                else:
                    pA = run_p
                    ua = np.zeros(G)
                if pA > 0:
                    tracks.append((pi, A, pa * pA, ua))
                if A < ell[pi]:
                    run_p *= racc[pi, A]
        tidx = np.asarray([t[0] for t in tracks])
        tua = np.stack([t[3] for t in tracks])

        def evf(q, v, u):
            res = run(tidx[q], tua[q], u)
            return res.tokens[np.arange(q.size), np.asarray([tracks[j][1] for j in q])]

        probs, _ = _bisect(evf, len(tracks), V)
        for j, (pi, A, p, _) in enumerate(tracks):
            for y in range(V):
                if probs[j, y] > 0:
                    out = tuple(int(t) for t in X[pi, :A]) + (y,)
                    law[out] = law.get(out, 0.0) + p * probs[j, y]
        return law


def softmax(z, T):
    z = np.asarray(z, np.float64) / T
    e = np.exp(z - z.max())
    return e / e.sum()


def preservation_error(law, target, T, V):
    """Largest |M(q, z) - M(q) p_t(z | q)| over emitted prefixes q and tokens
    z, where M(q, z) is the probability that the output continues prefix q
    with z.  Zero for a lossless round."""
    M = {}
    for out, p in law.items():
        for j in range(len(out)):
            M.setdefault(out[:j], np.zeros(V))[out[j]] += p
    worst = 0.0
    for q, m in M.items():
        pt = softmax(target[q], T)
        worst = max(worst, float(np.abs(m - m.sum() * pt).max()))
    return worst


def random_target(rng, V, G, scale=1.5):
    """Prefix-indexed target logits, rounded to fp32 (the oracle's input type)."""
    return {p: rng.normal(0, scale, V).astype(np.float32).astype(np.float64) for n in range(G + 1)
            for p in itertools.product(range(V), repeat=n)}
