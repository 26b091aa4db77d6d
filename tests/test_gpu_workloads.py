"""The full-size workloads on the GPU, in the launch configuration the
benchmark times (graph-free, one stream), checked against the oracle:
scheduler on the whole batch (the GPU's survivals), confidence on the whole
batch, drafting and verification on a seeded sample of requests (the oracle
recomputes them one by one), and invariants on every request."""
import numpy as np
import pytest
import torch

import parity
from speculative_decoding_draft_rank_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CASES = [("qwen_vocab", wl.qwen_vocab, 12), ("headline", wl.headline, 16), ("saturated", wl.saturated, 16)] + \
        [(f"long_block_g{g}", (lambda g=g: wl.long_block(g)), 6) for g in (4, 8, 12, 16)]


@pytest.mark.parametrize("name,make,nsample", CASES, ids=[c[0] for c in CASES])
def test_workload_parity(name, make, nsample, capsys):
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    w = make()
    inp = w.inputs()
    dr = DeviceRound(inp, w.knots_n, w.knots_t, w.budget, w.mode)
    dr.run()
    torch.cuda.synchronize()
    out = dr.outputs()
    assert dr.device_status() == 0
    rep = parity.Report()
    parity.check_confidence(inp, out["c"], out["S"])
    parity.check_schedule(out["S"], out["ell"], int(out["n_adm"][0]), float(out["theta"][0]), out["order"],
                          w.knots_n, w.knots_t, w.budget, w.mode, w.G, rep)
    rng = np.random.default_rng(1234)
    idx = np.sort(rng.choice(w.B, size=min(nsample, w.B), replace=False))
    if w.temps is not None:  # make sure every temperature group is sampled
        groups = np.unique(np.asarray(w.temps))
        for g in groups:
            members = np.nonzero(np.asarray(w.temps) == g)[0]
            if not np.isin(members, idx).any():
                idx = np.sort(np.append(idx, members[0]))
    parity.check_draft(inp, idx, out["x"], out["pd_x"], out["rowmax"], out["rowsum"], rep)
    parity.check_verify(inp, idx, out["x"], out["ell"], out["acc"], out["tokens"], out["nout"], out["pt_x"], rep)
    # Invariants on every request.
    assert np.all((out["x"] >= 0) & (out["x"] < w.V))
    assert np.all((out["acc"] >= 0) & (out["acc"] <= out["ell"]))
    assert np.array_equal(out["nout"], out["acc"] + 1)
    for b in range(w.B):
        A = out["acc"][b]
        assert np.array_equal(out["tokens"][b, :A], out["x"][b, :A])
        assert 0 <= out["tokens"][b, A] < w.V and np.all(out["tokens"][b, A + 1:] == -1)
    if w.mode == wl.MODE_ALL:
        assert np.all(out["ell"] == w.G)
    with capsys.disabled():
        print(f"\n{name}: {rep.summary()}")
    parity.assert_few_ties(rep)
