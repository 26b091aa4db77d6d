"""The device's near-tie counts (dspark_get_near_ties) on rounds with planted
ties.

Uniforms are placed on the edge of a token's CDF interval at the first draft
position of some requests, and on the accept threshold p_t(x)/p_d(x) at the
first verified position of others (computed in fp64 from the round's own
inputs, then rounded to fp32, so the margin is ~1e-7 on any arithmetic).  The
counts must include every planted tie and otherwise agree with the oracle's
margins below 1e-5, up to the decisions whose oracle margin lies so close to
1e-5 that fp32 arithmetic may put them on either side.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from speculative_decoding_draft_rank_b200 import _lib, synth

pytestmark = pytest.mark.gpu

TIE = 1e-5


def _band(m):
    """Oracle margins that fp32 evaluation may count either way."""
    return int(np.sum((m > 0.2 * TIE) & (m < 5 * TIE)))


def test_planted_near_ties_are_counted():
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    B, G, V, r = 24, 3, 3000, 32
    inp = synth.generate(B, G, V, r, 16, "bf16", seed=31, hot=4, sigma_t=0.6)
    Lt, Ut, Wt = (torch.from_numpy(a.astype(np.float64)) for a in (inp.L, inp.U, inp.W))
    planted_draft = list(range(0, 6))
    for b in planted_draft:   # u on the upper edge of the most likely token's interval
        p = torch.softmax(Lt[b, 0] + Ut[int(inp.x0[b])] @ Wt, 0)
        C = torch.cumsum(p, 0).numpy()
        inp.u_draft[b, 0] = np.float32(C[int(torch.argmax(p))])
    d0 = oracle.draft(inp.L, inp.U, inp.W, inp.x0, inp.temp, inp.u_draft.astype(np.float64))
    planted_accept = []
    Tt = torch.from_numpy(inp.Tlog.astype(np.float64))
    for b in range(8, B):    # u on the accept threshold at the first position
        x = int(d0.x[b, 0])
        pd = torch.softmax(Lt[b, 0] + Ut[int(inp.x0[b])] @ Wt, 0)[x]
        pt = torch.softmax(Tt[b, 0], 0)[x]
        ratio = float(pt / pd)
        if ratio < 0.95 and len(planted_accept) < 6:
            inp.u_accept[b, 0] = np.float32(ratio)
            planted_accept.append(b)
    assert len(planted_accept) >= 3
    kn, kt = np.array([0], np.int32), np.array([1.0])
    dr = DeviceRound(inp, kn, kt, -1, 0)   # every position verified
    _lib.dspark_clear_device_status(dr.ws)
    dr.run()
    torch.cuda.synchronize()
    out = dr.outputs()
    nd, nv = _lib.dspark_get_near_ties(dr.ws)
    # The oracle's account of the same round (along the GPU's drafted tokens).
    od = oracle.draft(inp.L, inp.U, inp.W, inp.x0, inp.temp, inp.u_draft.astype(np.float64))
    assert np.all(od.margin[planted_draft, 0] < 1e-6)
    want_d = int(np.sum(od.margin < TIE))
    assert nd >= len(planted_draft)
    assert abs(nd - want_d) <= _band(od.margin), (nd, want_d)
    ov = oracle.verify(inp.Tlog, inp.L, inp.U, inp.W, inp.x0, out["x"], inp.temp,
                       inp.u_accept.astype(np.float64), inp.u_final.astype(np.float64), out["ell"])
    deciding = np.arange(G)[None, :] <= ov.acc[:, None]
    m_acc = np.where(deciding, ov.margin_acc, np.inf)
    assert np.all(m_acc[planted_accept, 0] < 1e-6)
    want_v = int(np.sum(m_acc < TIE)) + int(np.sum(ov.margin_fin < TIE))
    assert nv >= len(planted_accept)
    assert abs(nv - want_v) <= _band(m_acc) + _band(ov.margin_fin), (nv, want_v)
    # Cleared with the status word.
    _lib.dspark_clear_device_status(dr.ws)
    assert _lib.dspark_get_near_ties(dr.ws) == (0, 0)
