"""Confidence calibration on the GPU against the fp64 oracle: the sequential
temperature scaling fit (every candidate's ECE, the chosen temperatures, the
fitted survivals) and the survival ROC-AUC pair counts (exact integers).

Tolerances: the ECEs are fp64 sums of up to N terms in a different order
(per-thread bin columns) than the oracle's index order, so they agree to
about N * 2^-53 relative; 1e-12 absolute is the bar.  A temperature choice
may differ only where the two candidates' oracle ECEs are within that bar (a
near-tie); none occurs on these inputs, so the test asks for equality and
reports the margin.  Scores and bins are fp64 on both sides."""
import numpy as np
import pytest
import torch

from oracle import calibration as C
from speculative_decoding_draft_rank_b200 import _lib, synth, workloads as wl

pytestmark = pytest.mark.gpu

ECE_TOL = 1e-12


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _fit(z, acc, grid, M):
    N, G = z.shape
    K = grid.shape[0]
    ws = torch.zeros(_lib.dspark_sts_workspace_size(N, G, K, M), dtype=torch.uint8, device="cuda")
    f64 = dict(dtype=torch.float64, device="cuda")
    tau = torch.zeros(G, dtype=torch.float32, device="cuda")
    e_raw, e_fit, e_all = torch.zeros(G, **f64), torch.zeros(G, **f64), torch.zeros((G, K), **f64)
    S = torch.zeros((N, G), dtype=torch.float32, device="cuda")
    _lib.dspark_sts_fit(_dev(z), _dev(acc), _dev(grid), M, ws, tau, e_raw, e_fit, e_all, S)
    status = _lib.dspark_get_device_status(ws)
    return (tau.cpu().numpy(), e_raw.cpu().numpy(), e_fit.cpu().numpy(), e_all.cpu().numpy(), S.cpu().numpy(),
            status)


def _check_fit(z, acc, grid, M, expect_status=0):
    tau, e_raw, e_fit, e_all, S, status = _fit(z, acc, grid, M)
    o_tau, o_raw, o_fit, o_all = C.sts_fit(z, acc, grid, M)
    assert status == expect_status
    fin = np.isfinite(o_all)
    assert np.array_equal(fin, np.isfinite(e_all))
    assert np.max(np.abs(e_all[fin] - o_all[fin]), initial=0.0) <= ECE_TOL
    assert np.max(np.abs(e_raw - o_raw)) <= ECE_TOL
    for i in range(z.shape[1]):
        if tau[i] != o_tau[i]:
            kg = int(np.flatnonzero(grid == tau[i])[0])
            ko = int(np.flatnonzero(grid == o_tau[i])[0])
            pytest.fail(f"position {i + 1}: tau {tau[i]} vs oracle {o_tau[i]}, "
                        f"oracle ECE margin {o_all[i, kg] - o_all[i, ko]:.3e}")
    assert np.max(np.abs(e_fit - o_fit)) <= ECE_TOL
    # Fitted survivals: fp64 products rounded to fp32 on both sides; the
    # fp64 values agree to a few ulps, so the fp32 results to 1 ulp.
    oS = C.survival(z, o_tau).astype(np.float32)
    assert np.all(np.abs(S.view(np.int32).astype(np.int64) - oS.view(np.int32).astype(np.int64)) <= 1)
    return tau, e_raw, e_fit


@pytest.mark.parametrize("N,G,K,M,k,seed", [
    (37, 3, 9, 10, 2.0, 0),          # one partial tile of samples, ragged
    (5000, 5, 65, 15, [2.0, 0.7, 1.5, 1.2, 3.0], 1),
    (257, 16, 33, 32, 0.8, 2),       # G = 16, M = 32 (the limits)
    (1, 1, 1, 1, 1.0, 3),            # degenerate: one sample, one candidate, one bin
    (3000, 2, 4096, 7, 1.3, 4),      # K = 4096 candidates
])
def test_sts_fit_matches_oracle(N, G, K, M, k, seed):
    cs = synth.calibration_set(N, G, k=k, seed=seed)
    grid = synth.tau_grid(K) if K > 1 else np.array([1.0], np.float32)
    _check_fit(cs.z, cs.acc, grid, M)


def test_sts_fit_headline_workload():
    w = wl.calibration_headline()
    cs = w.inputs()
    tau, e_raw, e_fit = _check_fit(cs.z, cs.acc, w.grid(), w.M)
    # The head's logits are twice the latent ones: the fit lands next to 2.
    assert np.all(np.abs(np.log(tau / 2.0)) < np.log(1.15)), tau
    assert np.all(e_fit < e_raw)


def test_sts_fit_ties_and_invalid_entries():
    # z = 0: every candidate gives the same ECE bits; the first entry wins.
    z = np.zeros((300, 3), np.float32)
    acc = (np.arange(300) % 4).astype(np.int32)
    _check_fit(z, acc, np.array([0.5, 1.0, 2.0], np.float32), 10)
    # Grid entries that are no temperature: never chosen, flagged.
    cs = synth.calibration_set(2000, 2, k=2.0, seed=5)
    grid = np.array([0.0, -1.0, np.nan, 2.0, np.inf, 1.5], np.float32)
    _check_fit(cs.z, cs.acc, grid, 10, expect_status=_lib.DEV_BAD_VALUE)
    # Every entry invalid: the first is reported, every ECE is +inf.
    tau, _, e_fit, e_all, _, status = _fit(cs.z, cs.acc, np.array([0.0, -2.0], np.float32), 10)
    assert tau[0] == 0.0 and np.all(np.isinf(e_all)) and status & _lib.DEV_BAD_VALUE


def test_sts_fit_accept_counts_out_of_range_are_flagged():
    cs = synth.calibration_set(500, 4, seed=6)
    acc = cs.acc.copy()
    acc[3], acc[77] = -1, 9
    _check_fit(cs.z, acc, synth.tau_grid(17), 10, expect_status=_lib.DEV_ELL_RANGE)


def test_sts_fit_is_deterministic():
    cs = synth.calibration_set(4000, 5, seed=7)
    a = _fit(cs.z, cs.acc, synth.tau_grid(), 15)
    b = _fit(cs.z, cs.acc, synth.tau_grid(), 15)
    for x, y in zip(a[:5], b[:5]):
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8))


def _auc(S, acc):
    N, G = S.shape
    twice = torch.zeros(G, dtype=torch.int64, device="cuda")
    pairs = torch.zeros(G, dtype=torch.int64, device="cuda")
    _lib.dspark_survival_auc(_dev(S), _dev(acc), twice, pairs)
    return twice.cpu().numpy(), pairs.cpu().numpy()


@pytest.mark.parametrize("N,G,seed,rounded", [(37, 3, 0, False), (5000, 5, 1, True), (2049, 2, 2, False),
                                              (16384, 5, 3, False)])
def test_survival_auc_matches_oracle(N, G, seed, rounded):
    cs = synth.calibration_set(N, G, k=1.5, seed=seed)
    S = C.survival(cs.z, np.full(G, 1.5, np.float32)).astype(np.float32)
    if rounded:   # many ties
        S = np.round(S, 2).astype(np.float32)
    twice, pairs = _auc(S, cs.acc)
    y = C.labels_from_accepts(cs.acc, G)
    for i in range(G):
        assert (int(twice[i]), int(pairs[i])) == C.roc_auc(S[:, i].astype(np.float64), y[:, i])


def test_survival_auc_all_one_class():
    S = np.linspace(0, 1, 100, dtype=np.float32).reshape(50, 2)
    twice, pairs = _auc(S, np.full(50, 2, np.int32))   # every sample positive at both positions
    assert np.all(twice == 0) and np.all(pairs == 0)
