"""Failure detection on the GPU without a fault: the bounded device waits run
out and the kernels return.

DSPARK_WAIT_BUDGET_CYCLES sets the clock budget of the library's bounded
waits (mbarrier waits, grid barriers, stage rings) when a launch is enqueued.
A budget of a few hundred cycles is shorter than any real copy or MMA, so the
first wait gives up: the kernel raises DSPARK_DEV_TIMEOUT in the status word,
drains its own copies and MMAs, frees its tensor memory and returns.  The
test checks that the status arrives, that the calls return, and that the
next round on the same workspace, with the normal budget, is oracle-identical.
"""
import numpy as np
import pytest
import torch

import parity
from speculative_decoding_draft_rank_b200 import _lib, synth

pytestmark = pytest.mark.gpu

SHORT = "200"


def _round(B, G, V, r, seed):
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    temps = np.tile(np.float32([1.0, 0.0, 0.7, 1.3]), B)[:B]
    inp = synth.generate(B, G, V, r, 16, "bf16", seed=seed, hot=8, temps=temps)
    kn, kt = np.array([0, 20, 60], np.int32), np.array([10.0, 11.0, 14.0])
    return inp, DeviceRound(inp, kn, kt, -1, 0), (kn, kt)


@pytest.mark.parametrize("B,G,V,r", [(130, 3, 4104, 64), (256, 2, 20000, 256)])
def test_wait_budget_runs_out_and_the_next_round_is_exact(monkeypatch, B, G, V, r):
    inp, dr, (kn, kt) = _round(B, G, V, r, seed=B + V)
    t, o = dr.t, dr.o
    monkeypatch.setenv("DSPARK_WAIT_BUDGET_CYCLES", SHORT)
    _lib.dspark_clear_device_status(dr.ws)
    _lib.dspark_draft_markov(t["L"], t["U"], t["Wt"], t["x0"], t["temp"], t["u_draft"], dr.ws, o["x"],
                             o["pd_x"], o["rowmax"], o["rowsum"])
    st = dr.device_status()
    assert st & _lib.DEV_TIMEOUT, f"drafting: status {st:#x}"
    # Verification with every position admitted: the staged row pass and the
    # residual tile pass give up too.
    o["ell"].fill_(G)
    o["x"].clamp_(0, V - 1)
    o["pd_x"].fill_(0.5)
    o["rowmax"].fill_(0.0)
    o["rowsum"].fill_(1.0)
    _lib.dspark_clear_device_status(dr.ws)
    _lib.dspark_verify(t["Tlog"], t["L"], t["U"], t["Wt"], t["x0"], o["x"], o["pd_x"], o["rowmax"], o["rowsum"],
                       t["temp"], t["u_accept"], t["u_final"], o["ell"], dr.ws, o["acc"], o["tokens"], o["nout"],
                       o["pt_x"])
    st = dr.device_status()
    assert st & _lib.DEV_TIMEOUT, f"verification: status {st:#x}"
    # The normal budget again: the same workspace gives the oracle's round.
    monkeypatch.delenv("DSPARK_WAIT_BUDGET_CYCLES")
    _lib.dspark_clear_device_status(dr.ws)
    dr.run()
    torch.cuda.synchronize()
    out = dr.outputs()
    rep = parity.Report()
    idx = np.arange(0, B, max(1, B // 12))
    parity.check_draft(inp, idx, out["x"], out["pd_x"], out["rowmax"], out["rowsum"], rep)
    parity.check_verify(inp, idx, out["x"], out["ell"], out["acc"], out["tokens"], out["nout"], out["pt_x"], rep)
    assert dr.device_status() == 0
    parity.assert_few_ties(rep)
