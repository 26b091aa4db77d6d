"""Parity of the CUDA round (through the C ABI) with the fp64 oracle.

Small rounds that the oracle finishes in seconds but that span several
column tiles with a ragged tail, in fp32 and bf16, with mixed temperatures
(greedy rows included) and the scheduler's edge cases.
"""
import numpy as np
import pytest
import torch

import parity
from oracle import oracle
from speculative_decoding_draft_rank_b200 import synth, workloads as wl

pytestmark = pytest.mark.gpu


def _round(B, G, V, r, d, dtype, seed, knots_n, knots_t, budget=-1, mode=1, temps=None, sigma_t=0.3,
           hot=8):
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    inp = synth.generate(B, G, V, r, d, dtype, seed=seed, hot=hot, sigma_t=sigma_t, temps=temps)
    dr = DeviceRound(inp, knots_n, knots_t, budget, mode)
    dr.run()
    torch.cuda.synchronize()
    return inp, dr


def _check_round(inp, dr, knots_n, knots_t, budget, mode, idx=None):
    out = dr.outputs()
    rep = parity.Report()
    idx = np.arange(inp.B) if idx is None else np.asarray(idx)
    parity.check_draft(inp, idx, out["x"], out["pd_x"], out["rowmax"], out["rowsum"], rep)
    parity.check_confidence(inp, out["c"], out["S"])
    parity.check_schedule(out["S"], out["ell"], int(out["n_adm"][0]), float(out["theta"][0]), out["order"],
                          knots_n, knots_t, budget, mode, inp.G, rep)
    parity.check_verify(inp, idx, out["x"], out["ell"], out["acc"], out["tokens"], out["nout"], out["pt_x"],
                        rep)
    assert dr.device_status() == 0
    return out, rep


PROFILE = (np.array([0, 20, 60], np.int32), np.array([10.0, 11.0, 14.0]))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,G,V,r,d", [(37, 5, 5000, 32, 96), (9, 3, 1288, 16, 40), (64, 8, 3072, 64, 256),
                                       (130, 4, 9000, 256, 128), (200, 2, 2056, 80, 64),
                                       (150, 3, 4104, 320, 64), (70, 3, 3000, 512, 64)])
def test_round_parity_small(dtype, B, G, V, r, d):
    temps = np.tile(np.float32([1.0, 0.0, 0.6, 1.2]), B)[:B]
    inp, dr = _round(B, G, V, r, d, dtype, seed=B + V, knots_n=PROFILE[0], knots_t=PROFILE[1], temps=temps)
    out, rep = _check_round(inp, dr, *PROFILE, -1, 1)
    # At a 1e-5 margin a counted near-tie is a rare event (about 2e-5 per
    # decision, and a disagreement needs a far smaller margin still).
    parity.assert_few_ties(rep)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_verify_everything_and_nothing(dtype):
    """ALL mode (every position verified) and a zero budget (fresh target token only)."""
    B, G, V, r, d = 16, 4, 2048, 16, 32
    inp, dr = _round(B, G, V, r, d, dtype, seed=5, knots_n=PROFILE[0], knots_t=PROFILE[1], mode=0)
    out, _ = _check_round(inp, dr, *PROFILE, -1, 0)
    assert np.all(out["ell"] == G)
    inp, dr = _round(B, G, V, r, d, dtype, seed=6, knots_n=PROFILE[0], knots_t=PROFILE[1], budget=0)
    out, _ = _check_round(inp, dr, *PROFILE, 0, 1)
    assert np.all(out["ell"] == 0) and np.all(out["nout"] == 1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tiny_vocab_and_single_request(dtype):
    shapes = [(1, 1, 2), (3, 2, 7), (1, 16, 300)] if dtype == "f32" else [(1, 1, 8), (3, 2, 16), (1, 16, 304)]
    for (B, G, V) in shapes:
        inp, dr = _round(B, G, V, 16, 8, dtype, seed=V, knots_n=np.array([0], np.int32),
                         knots_t=np.array([1.0]), hot=1)
        _check_round(inp, dr, np.array([0], np.int32), np.array([1.0]), -1, 1)


def test_workload_tiny_full():
    """The tiny fp32 workload (B=4, G=5, V=1024, r=16, d=64), every stage."""
    w = wl.tiny()
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    inp = w.inputs()
    dr = DeviceRound(inp, w.knots_n, w.knots_t, w.budget, w.mode)
    dr.run()
    torch.cuda.synchronize()
    out, rep = _check_round(inp, dr, w.knots_n, w.knots_t, w.budget, w.mode)
    assert out["ell"].sum() <= 12
