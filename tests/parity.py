"""Stage-by-stage comparison of the CUDA round with the fp64 oracle.

Decisions (draft tokens, accept tests, admitted counts, emitted tokens) must
agree exactly, except where the oracle reports a margin below ``TIE`` (the
uniform lies within 1e-5 of a threshold, or two logits within 1e-5 decide an
argmax).  Such near-ties are counted; the oracle is then rerun with the GPU's
decision forced so the rest of the round is still compared.  Besides the
disagreements, the report counts the near-tie window (the checked decisions
with an oracle margin below ``TIE``) and keeps the disagreements' margins.  Probabilities
(p_d(x), p_t(x), c, S), the row max and log Z agree within ``ATOL``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from oracle import oracle
from speculative_decoding_draft_rank_b200 import synth

TIE = 1e-5
ATOL = 1e-5


@dataclass
class Report:
    """near_ties: decisions where the GPU and the oracle differ (each one
    within TIE of its threshold, as the oracle measures it); window: the
    checked decisions whose oracle margin is below TIE at all (the near-tie
    window: at V ~ 1e5 most tokens' CDF intervals are narrower than 1e-5, so
    most draws fall inside it); tie_margins: the oracle margins of the
    disagreements."""
    near_ties: dict = field(default_factory=lambda: {"draft": 0, "accept": 0, "final": 0, "schedule": 0})
    window: dict = field(default_factory=lambda: {"draft": 0, "accept": 0, "final": 0})
    decisions: dict = field(default_factory=lambda: {"draft": 0, "accept": 0, "final": 0})
    tie_margins: list = field(default_factory=list)
    checked_rows: int = 0

    def total_ties(self):
        return sum(self.near_ties.values())

    def summary(self):
        return (f"disagreements {self.near_ties}, near-tie window {self.window} of decisions {self.decisions}, "
                f"largest disagreement margin {max(self.tie_margins) if self.tie_margins else 0.0:.3g}")


# The GPU's fp32 CDFs, ratios and logits are accurate to about 1e-7 (the
# largest disagreement measured over every full-size workload: 1.1e-7), far
# inside the 1e-5 near-tie window; a disagreement further than this from its
# threshold is treated as an error.
FP32_TIE = 1e-6


def assert_few_ties(rep: Report):
    """Every disagreement lies inside the near-tie window (checked one by one
    by the stage checks) and within FP32_TIE of its threshold; and only a
    small part of the window may disagree: at most a tenth of it (at least
    one).  A systematic error of the size of the window would flip most of
    it (at V ~ 1e5 about half of all draws fall inside the window)."""
    win = sum(rep.window.values())
    assert rep.total_ties() <= max(1, win // 10), rep.summary()
    assert not rep.tie_margins or max(rep.tie_margins) < FP32_TIE, rep.summary()


def _close(name, got, want, atol=ATOL):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    bad = ~(np.abs(got - want) <= atol)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{name}: {bad.sum()} entries off by > {atol}; first at {tuple(i)}: "
                             f"gpu {got[tuple(i)]!r} oracle {want[tuple(i)]!r}")


def check_draft(inp: synth.RoundInputs, idx, gx, gpd, grmax, grsum, rep: Report, A=None):
    """Draft stage of requests idx against the oracle run on the same inputs
    (A: the RNN head's recurrent matrix, None for the Markov head)."""
    sub = synth.select_requests(inp, idx)
    gx, gpd, grmax, grsum = gx[idx], gpd[idx], grmax[idx], grsum[idx]
    B, G = gx.shape
    force = np.full((B, G), -1, np.int32)
    for _ in range(G + 1):
        o = oracle.draft(sub.L, sub.U, sub.W, sub.x0, sub.temp, sub.u_draft.astype(np.float64), force_x=force,
                         A=A)
        mism = (o.x != gx) & (force < 0)
        if not mism.any():
            break
        for b in np.nonzero(mism.any(axis=1))[0]:
            i = int(np.argmax(mism[b]))
            assert o.margin[b, i] < TIE, (
                f"draft token mismatch at request {idx[b]} position {i}: gpu {gx[b, i]} oracle {o.x[b, i]} "
                f"(margin {o.margin[b, i]:.3g})")
            force[b, i] = gx[b, i]
            rep.near_ties["draft"] += 1
            rep.tie_margins.append(float(o.margin[b, i]))
    else:
        raise AssertionError("draft near-tie resolution did not converge")
    assert np.array_equal(o.x, gx)
    rep.window["draft"] += int(np.sum(o.margin < TIE))
    rep.decisions["draft"] += int(o.margin.size)
    _close("p_d(x)", gpd, o.pd)
    _close("row max", grmax, o.rowmax)
    _close("log Z", np.log(grsum), np.log(o.rowsum))
    rep.checked_rows += B
    return o


def check_confidence(inp, gc, gS, tau=None):
    c, S = oracle.confidence(inp.h, inp.w, inp.bias, tau)
    _close("c", gc, c)
    _close("S", gS, S)
    assert np.all(np.diff(gS, axis=1) <= 0), "GPU survival increased along the block"
    return c, S


def check_schedule(gS, gell, gnadm, gtheta, gorder, knots_n, knots_t, budget, mode, G, rep: Report):
    """Scheduler fed the GPU's own survivals: admitted count and sets exact."""
    o = oracle.schedule(gS.astype(np.float64), knots_n, knots_t, budget, mode)
    if o.n_adm != gnadm:
        if mode == oracle.SCHED_GLOBAL_ARGMAX:
            # The global search has no single comparison to take a margin
            # from: the GPU's count must reach the oracle's best Theta to
            # within fp64 summation-order noise.
            alt = oracle.schedule(gS.astype(np.float64), knots_n, knots_t, budget, mode, force_n=int(gnadm))
            assert abs(alt.theta - o.theta) <= 1e-12 * abs(o.theta), (
                f"admitted count gpu {gnadm} oracle {o.n_adm}: Theta {alt.theta!r} vs best {o.theta!r}")
        else:
            # The count differs only if the comparison at the earlier of the
            # two stop points is a near-tie (the oracle's stop, or the
            # comparison where the GPU stopped and the oracle admitted).
            k = min(int(gnadm), int(o.n_adm))
            mk = o.margins[k] if k < len(o.margins) else np.inf
            assert mk < TIE, f"admitted count gpu {gnadm} oracle {o.n_adm} (margin at {k}: {mk:.3g})"
        rep.near_ties["schedule"] += 1
        o = oracle.schedule(gS.astype(np.float64), knots_n, knots_t, budget, mode, force_n=int(gnadm))
    assert np.array_equal(o.ell, gell), "admitted prefix lengths differ"
    if mode != oracle.SCHED_ALL:
        assert np.array_equal(o.order, gorder), "sorted candidate order differs"
    assert abs(o.theta - gtheta) <= 1e-9 * max(1.0, abs(o.theta))
    # Prefix property and budget, on the GPU's own output.
    B = gS.shape[0]
    adm = gorder[:gnadm]
    for b in range(B):
        pos = np.sort(adm[adm % B == b] // B)
        assert np.array_equal(pos, np.arange(len(pos))) and len(pos) == gell[b]
    if budget >= 0:
        assert gell.sum() <= budget
    assert np.all((gell >= 0) & (gell <= G))
    return o


def check_verify(inp: synth.RoundInputs, idx, gx, gell, gacc, gtok, gnout, gptx, rep: Report, A=None):
    """Verification of requests idx with the GPU's draft tokens and admitted
    lengths; the oracle rebuilds p_d itself in fp64 (A as for check_draft)."""
    sub = synth.select_requests(inp, idx)
    x, ell = gx[idx], gell[idx]
    gacc, gtok, gnout, gptx = gacc[idx], gtok[idx], gnout[idx], gptx[idx]
    B, G = x.shape
    force = np.full((B, G), -1, np.int32)
    for _ in range(G + 1):
        o = oracle.verify(sub.Tlog, sub.L, sub.U, sub.W, sub.x0, x, sub.temp,
                          sub.u_accept.astype(np.float64), sub.u_final.astype(np.float64), ell,
                          force_accept=force, A=A)
        mism = o.acc != gacc
        if not mism.any():
            break
        for b in np.nonzero(mism)[0]:
            k = int(min(o.acc[b], gacc[b]))
            assert force[b, k] < 0 and o.margin_acc[b, k] < TIE, (
                f"accepted count at request {idx[b]}: gpu {gacc[b]} oracle {o.acc[b]} "
                f"(margin {o.margin_acc[b, k]:.3g})")
            force[b, k] = 1 if gacc[b] > k else 0
            rep.near_ties["accept"] += 1
            rep.tie_margins.append(float(o.margin_acc[b, k]))
    else:
        raise AssertionError("accept near-tie resolution did not converge")
    assert np.array_equal(o.nout, gnout)
    deciding = (np.arange(G)[None, :] <= o.acc[:, None]) & (np.arange(G)[None, :] < ell[:, None])
    rep.window["accept"] += int(np.sum(deciding & (o.margin_acc < TIE)))
    rep.decisions["accept"] += int(np.sum(deciding))
    rep.window["final"] += int(np.sum(o.margin_fin < TIE))
    rep.decisions["final"] += B
    for b in range(B):
        A = o.acc[b]
        assert np.array_equal(o.tokens[b, :A], gtok[b, :A])
        assert np.all(gtok[b, A + 1:] == -1)
        if o.tokens[b, A] != gtok[b, A]:
            assert o.margin_fin[b] < TIE, (f"final token at request {idx[b]}: gpu {gtok[b, A]} oracle "
                                           f"{o.tokens[b, A]} (kind {o.final_kind[b]}, margin {o.margin_fin[b]:.3g})")
            rep.near_ties["final"] += 1
            rep.tie_margins.append(float(o.margin_fin[b]))
    m = np.arange(G)[None, :] < ell[:, None]
    _close("p_t(x)", np.where(m, gptx, 0.0), np.where(m, o.pt_x, 0.0))
    assert np.all(gptx[~m] == -1.0)
    return o
