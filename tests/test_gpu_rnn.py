"""Parity of the RNN sequential head's CUDA path with the fp64 oracle.

The paperlayer.ai summary (§3.1) and the menfem.com KB entry ("Key
Contributions") name an RNN head beside the Markov head: a recurrent state
that summarises the whole in-block prefix.  The reading built here is
h_1 = tanh(U[x_0]), h_k = tanh(h_{k-1} A + U[x_{k-1}]), bias h_k W.  The GPU's
drafted tokens, p_d(x), row statistics and states, and its verification
(accepted counts, emitted tokens, p_t(x)) must equal the oracle's under the
same bars as the Markov head (decisions exact except counted near-ties,
probabilities within 1e-5).  U is scaled up by 4 (a power of two, exact in
bf16) so that the state (~0.25) and its bias (~0.25 logits, four times the
Markov head's on the unscaled factors) matter.
"""
import numpy as np
import pytest
import torch

import parity
from oracle import oracle
from speculative_decoding_draft_rank_b200 import synth

pytestmark = pytest.mark.gpu

PROFILE = (np.array([0, 20, 60], np.int32), np.array([10.0, 11.0, 14.0]))


def _rnn_inputs(B, G, V, r, seed, temps, u_scale=4.0, w_scale=1.0):
    inp = synth.generate(B, G, V, r, 16, "bf16", seed=seed, hot=8, temps=temps)
    U = (inp.U * np.float32(u_scale)).astype(np.float32)      # exact: powers of two
    W = (inp.W * np.float32(w_scale)).astype(np.float32)
    inp.U, inp.W = U, W
    inp.bits["U"], inp.bits["W"] = synth.bf16_bits(U), synth.bf16_bits(W)
    A = synth.bf16_to_f32(synth.bf16_bits(synth.rnn_matrix(r, seed=seed))).reshape(r, r)
    return inp, A


def _run(inp, A, mode=1, budget=-1):
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    dr = DeviceRound(inp, *PROFILE, budget, mode, Arec=A)
    dr.run()
    torch.cuda.synchronize()
    return dr, dr.outputs()


@pytest.mark.parametrize("B,G,V,r", [(37, 3, 5000, 64), (130, 4, 3072, 256), (200, 5, 4104, 128),
                                     (64, 8, 2056, 32)])
def test_rnn_round_parity(B, G, V, r):
    temps = np.tile(np.float32([1.0, 0.0, 0.6, 1.2]), B)[:B]
    inp, A = _rnn_inputs(B, G, V, r, seed=B + V, temps=temps)
    dr, out = _run(inp, A)
    assert dr.device_status() == 0
    rep = parity.Report()
    idx = np.arange(B)
    parity.check_draft(inp, idx, out["x"], out["pd_x"], out["rowmax"], out["rowsum"], rep, A=A)
    # The states the drafting kernel used (fp32) against the oracle's along
    # the same tokens.
    h = oracle.rnn_states(inp.U, A, inp.x0, out["x"])
    assert np.abs(out["H"] - h).max() <= 1e-5
    parity.check_confidence(inp, out["c"], out["S"])
    parity.check_schedule(out["S"], out["ell"], int(out["n_adm"][0]), float(out["theta"][0]), out["order"],
                          *PROFILE, -1, 1, G, rep)
    parity.check_verify(inp, idx, out["x"], out["ell"], out["acc"], out["tokens"], out["nout"], out["pt_x"], rep,
                        A=A)
    parity.assert_few_ties(rep)


def test_rnn_verify_everything():
    """Every drafted position verified (many residual draws at rejected
    positions deep in the block, rebuilt from the stored states)."""
    B, G, V, r = 96, 6, 3000, 64
    inp, A = _rnn_inputs(B, G, V, r, seed=9, temps=np.float32(1.0))
    dr, out = _run(inp, A, mode=0)
    assert np.all(out["ell"] == G)
    rep = parity.Report()
    idx = np.arange(B)
    parity.check_draft(inp, idx, out["x"], out["pd_x"], out["rowmax"], out["rowsum"], rep, A=A)
    o = parity.check_verify(inp, idx, out["x"], out["ell"], out["acc"], out["tokens"], out["nout"], out["pt_x"],
                            rep, A=A)
    assert int(np.sum(o.final_kind == 0)) >= 20
    parity.assert_few_ties(rep)


def test_rnn_head_differs_from_markov_head():
    """The RNN head's state carries the prefix: its drafts differ from the
    Markov head's on the same inputs."""
    B, G, V, r = 64, 4, 2056, 64
    inp, A = _rnn_inputs(B, G, V, r, seed=5, temps=np.float32(1.0))
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    dm = DeviceRound(inp, *PROFILE, -1, 1)
    dm.run()
    torch.cuda.synchronize()
    _, out = _run(inp, A)
    assert (dm.outputs()["x"] != out["x"]).any()
