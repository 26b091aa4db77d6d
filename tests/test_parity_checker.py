"""The GPU parity checkers must be able to fail.  Fed the oracle's own outputs
they pass; fed copies with one planted error each (a wrong token, a
probability off by more than the tolerance, a wrong admitted length or order,
a wrong accepted count or final token, missing padding) they raise.  CPU only:
the "device" outputs here are the oracle's."""
import numpy as np
import pytest

import parity
from oracle import oracle
from speculative_decoding_draft_rank_b200 import synth

KN, KT = np.array([0, 8], np.int32), np.array([10.0, 12.0])


@pytest.fixture(scope="module")
def round_outputs():
    inp = synth.generate(6, 3, 64, 16, 8, "f32", seed=21, hot=4, temps=np.float32([1.0, 0.7, 0.0, 1.2, 1.0, 0.9]))
    d = oracle.draft(inp.L, inp.U, inp.W, inp.x0, inp.temp, inp.u_draft.astype(np.float64))
    c, S = oracle.confidence(inp.h, inp.w, inp.bias)
    S32 = S.astype(np.float32)
    s = oracle.schedule(S32.astype(np.float64), KN, KT, -1, oracle.SCHED_GREEDY_EARLY_STOP)
    v = oracle.verify(inp.Tlog, inp.L, inp.U, inp.W, inp.x0, d.x, inp.temp, inp.u_accept.astype(np.float64),
                      inp.u_final.astype(np.float64), s.ell)
    m = np.arange(3)[None, :] < s.ell[:, None]
    out = {"x": d.x.copy(), "pd": d.pd.copy(), "rowmax": d.rowmax.copy(), "rowsum": d.rowsum.copy(),
           "c": c.copy(), "S": S32, "ell": s.ell.copy(), "n_adm": s.n_adm, "theta": s.theta,
           "order": s.order.copy(), "acc": v.acc.copy(), "tokens": v.tokens.copy(), "nout": v.nout.copy(),
           "pt_x": np.where(m, v.pt_x, -1.0), "margin_draft": d.margin, "margin_acc": v.margin_acc,
           "margin_fin": v.margin_fin}
    return inp, out


def _run_all(inp, o):
    rep = parity.Report()
    idx = np.arange(inp.B)
    parity.check_draft(inp, idx, o["x"], o["pd"], o["rowmax"], o["rowsum"], rep)
    parity.check_confidence(inp, o["c"], o["S"])
    parity.check_schedule(o["S"], o["ell"], o["n_adm"], o["theta"], o["order"], KN, KT, -1,
                          oracle.SCHED_GREEDY_EARLY_STOP, inp.G, rep)
    parity.check_verify(inp, idx, o["x"], o["ell"], o["acc"], o["tokens"], o["nout"], o["pt_x"], rep)
    return rep


def test_oracle_outputs_pass(round_outputs):
    inp, o = round_outputs
    rep = _run_all(inp, o)
    assert rep.total_ties() == 0 and rep.checked_rows == inp.B


def _sure(margins):
    """Index of an entry whose decision margin is far from a tie."""
    i = np.argwhere(margins > 1e-2)
    assert len(i), "no decision with a comfortable margin"
    return tuple(i[0])


def _plant(o, what):
    o = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in o.items()}
    if what == "draft_token":
        b, i = _sure(o["margin_draft"])
        o["x"][b, i] = (o["x"][b, i] + 1) % 64
    elif what == "p_d":
        o["pd"][0, 0] += 1e-4
    elif what == "row_max":
        o["rowmax"][1, 2] += 1e-4
    elif what == "log_Z":
        o["rowsum"][2, 1] *= 1.001
    elif what == "confidence":
        o["c"][3, 1] += 1e-4
    elif what == "survival_rises":
        o["S"][0, 2] = o["S"][0, 1] + 1e-3
    elif what == "admitted_length":
        b = int(np.argmax(o["ell"] < 3))
        o["ell"][b] += 1
    elif what == "order":
        o["order"][[0, 1]] = o["order"][[1, 0]]
    elif what == "accepted_count":
        b = int(np.argmax(o["ell"] > 0))
        o["acc"][b] = (o["acc"][b] + 1) % (o["ell"][b] + 1)
        o["nout"][b] = o["acc"][b] + 1
    elif what == "final_token":
        b = int(np.argmax(o["margin_fin"] > 1e-2))
        A = o["acc"][b]
        o["tokens"][b, A] = (o["tokens"][b, A] + 1) % 64
    elif what == "padding":
        b = int(np.argmax(o["nout"] <= 3))
        o["tokens"][b, 3] = 0
    elif what == "p_t":
        b = int(np.argmax(o["ell"] > 0))
        o["pt_x"][b, 0] += 1e-4
    return o


PLANTS = ["draft_token", "p_d", "row_max", "log_Z", "confidence", "survival_rises", "admitted_length", "order",
          "accepted_count", "final_token", "padding", "p_t"]


@pytest.mark.parametrize("what", PLANTS)
def test_planted_error_is_caught(round_outputs, what):
    inp, o = round_outputs
    with pytest.raises(AssertionError):
        _run_all(inp, _plant(o, what))
