"""Full-size drafting and verification parity on wide samples of requests.

The headline workload (B=256, G=5, V=129280) and the saturated one (B=1024,
G=8, mixed temperatures) run once through the C ABI in the launch
configuration the benchmark times; the oracle then recomputes 128 headline
and 96 saturated requests one by one: both 128-row M-blocks of the headline batch, every
temperature quarter of the saturated batch, and among them at least twenty
rejections whose replacement token comes from the residual max(0, p_t - p_d)
at full vocabulary width (menfem.com KB entry, "Methodology": rejection
sampling keeps the target distribution).  The number of counted near-ties is
printed and bounded.
"""
import numpy as np
import pytest
import torch

import parity
from speculative_decoding_draft_rank_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _sample(w, n):
    """n requests spread evenly over the M-blocks (and temperature groups)."""
    groups = max(1, w.B // 128)
    per = n // groups
    rng = np.random.default_rng(77)
    idx = [g * 128 + rng.choice(min(128, w.B - g * 128), size=per, replace=False) for g in range(groups)]
    return np.sort(np.concatenate(idx))


@pytest.mark.parametrize("make,n", [(wl.headline, 128), (wl.saturated, 96)], ids=["headline", "saturated"])
def test_fullsize_wide_sample(make, n, capsys):
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    w = make()
    inp = w.inputs()
    dr = DeviceRound(inp, w.knots_n, w.knots_t, w.budget, w.mode)
    dr.run()
    torch.cuda.synchronize()
    out = dr.outputs()
    assert dr.device_status() == 0
    idx = _sample(w, n)
    assert len(idx) == n and (idx < 128).any() and (idx >= 128).any()
    if w.temps is not None:
        assert len(np.unique(np.asarray(w.temps)[idx])) == 4
    rep = parity.Report()
    parity.check_draft(inp, idx, out["x"], out["pd_x"], out["rowmax"], out["rowsum"], rep)
    o = parity.check_verify(inp, idx, out["x"], out["ell"], out["acc"], out["tokens"], out["nout"], out["pt_x"],
                            rep)
    residual = int(np.sum(o.final_kind == 0))
    with capsys.disabled():
        print(f"\n{w.name}: {len(idx)} requests, {residual} residual draws; {rep.summary()}")
    assert residual >= 20
    parity.assert_few_ties(rep)
