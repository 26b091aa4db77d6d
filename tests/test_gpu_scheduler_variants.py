"""Scheduler variants on the GPU against the fp64 oracle: the offline global
search (Theta maximised over every admitted count, no early stop) and static
survival-threshold pruning.  Survivals are cumulative products of random
confidences (with repeated values, so the sort's tie order is exercised);
profiles are the headline's convex knots and step-shaped non-convex ones.
"""
import numpy as np
import pytest
import torch

import parity
from oracle import oracle
from speculative_decoding_draft_rank_b200 import _lib, workloads as wl

pytestmark = pytest.mark.gpu


def _survivals(rng, B, G, ties):
    if ties:
        c = rng.choice(np.float32([1.0, 0.9, 0.75, 0.5]), size=(B, G))
    else:
        c = rng.uniform(0.05, 1.0, size=(B, G)).astype(np.float32)
    return np.cumprod(c, axis=1, dtype=np.float32)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _schedule(S, kn, kt, budget, mode):
    B, G = S.shape
    ws = torch.zeros(_lib.dspark_schedule_workspace_size(B, G), dtype=torch.uint8, device="cuda")
    ell = torch.zeros(B, dtype=torch.int32, device="cuda")
    nadm = torch.zeros(1, dtype=torch.int32, device="cuda")
    theta = torch.zeros(1, dtype=torch.float64, device="cuda")
    order = torch.zeros(B * G, dtype=torch.int32, device="cuda")
    _lib.dspark_schedule(_dev(S), _dev(np.asarray(kn, np.int32)), _dev(np.asarray(kt, np.float64)), budget, mode,
                         ws, ell, nadm, theta, order)
    torch.cuda.synchronize()
    return ell.cpu().numpy(), int(nadm.item()), float(theta.item()), order.cpu().numpy()


PROFILES = {
    "headline": (wl.headline().knots_n, wl.headline().knots_t),
    "step": (np.array([0, 64, 128, 640], np.int32), np.array([100.0, 100.5, 180.0, 200.0])),
    "flat_then_steep": (np.array([0, 300, 301], np.int32), np.array([50.0, 50.0, 120.0])),
}


@pytest.mark.parametrize("B,G", [(256, 5), (37, 3), (1, 16), (4096, 4)])
@pytest.mark.parametrize("profile", list(PROFILES))
@pytest.mark.parametrize("ties", [False, True])
def test_global_search_matches_oracle(B, G, profile, ties):
    rng = np.random.default_rng(B * 7 + G + (1000 if ties else 0))
    S = _survivals(rng, B, G, ties)
    kn, kt = PROFILES[profile]
    for budget in (-1, B * G // 3):
        ell, nadm, theta, order = _schedule(S, kn, kt, budget, _lib.SCHED_GLOBAL_ARGMAX)
        parity.check_schedule(S, ell, nadm, theta, order, kn, kt, budget, oracle.SCHED_GLOBAL_ARGMAX, G,
                              parity.Report())
        # It never admits fewer than the early-stop rule when Theta is unimodal.
        e_ell, e_nadm, _, _ = _schedule(S, kn, kt, budget, _lib.SCHED_GREEDY_EARLY_STOP)
        if profile == "headline":
            assert nadm >= e_nadm


@pytest.mark.parametrize("B,G", [(256, 5), (37, 3), (1, 16), (4096, 4)])
@pytest.mark.parametrize("ties", [False, True])
def test_threshold_matches_oracle(B, G, ties):
    rng = np.random.default_rng(B + G * 13 + (1000 if ties else 0))
    S = _survivals(rng, B, G, ties)
    ws = torch.zeros(_lib.dspark_schedule_workspace_size(B, G), dtype=torch.uint8, device="cuda")
    dS = _dev(S)
    ell = torch.zeros(B, dtype=torch.int32, device="cuda")
    nadm = torch.zeros(1, dtype=torch.int32, device="cuda")
    order = torch.zeros(B * G, dtype=torch.int32, device="cuda")
    thresholds = [0.0, 1.0, 1.5, float(S[0, 0]), float(np.median(S)), float(S.min())]
    for th in thresholds:
        for budget in (-1, 0, B * G // 4):
            _lib.dspark_schedule_threshold(dS, th, budget, ws, ell, nadm, order)
            torch.cuda.synchronize()
            o_ell, o_nadm, o_order = oracle.schedule_threshold(S.astype(np.float64), np.float32(th), budget)
            assert int(nadm.item()) == o_nadm, (th, budget)
            assert np.array_equal(ell.cpu().numpy(), o_ell), (th, budget)
            assert np.array_equal(order.cpu().numpy(), o_order)
            assert _lib.dspark_get_device_status(ws) == 0


# ------------------------------------------------ production scheduler: top-K
def _topk(S, cap, budget):
    B, G = S.shape
    ws = torch.zeros(_lib.dspark_schedule_workspace_size(B, G), dtype=torch.uint8, device="cuda")
    ell = torch.zeros(B, dtype=torch.int32, device="cuda")
    nadm = torch.zeros(1, dtype=torch.int32, device="cuda")
    order = torch.zeros(B * G, dtype=torch.int32, device="cuda")
    capd = torch.tensor([cap], dtype=torch.int32, device="cuda")
    _lib.dspark_schedule_topk(_dev(S), capd, budget, ws, ell, nadm, order)
    torch.cuda.synchronize()
    return ell.cpu().numpy(), int(nadm.item()), order.cpu().numpy(), _lib.dspark_get_device_status(ws)


@pytest.mark.parametrize("B,G", [(256, 5), (37, 3), (1, 16), (4096, 4)])
@pytest.mark.parametrize("ties", [False, True])
def test_topk_matches_oracle(B, G, ties):
    rng = np.random.default_rng(B * 11 + G + (1000 if ties else 0))
    S = _survivals(rng, B, G, ties)
    N = B * G
    for cap in (0, 1, N // 3, N - 1, N, N + 7):
        for budget in (-1, N // 4):
            ell, nadm, order, status = _topk(S, cap, budget)
            oell, onadm, oorder = oracle.schedule_topk(S.astype(np.float64), cap, budget)
            assert status == 0
            assert nadm == onadm and np.array_equal(ell, oell) and np.array_equal(order, oorder)


def test_topk_negative_capacity_is_flagged():
    S = _survivals(np.random.default_rng(5), 16, 4, False)
    ell, nadm, _, status = _topk(S, -3, -1)
    assert nadm == 0 and not ell.any() and status & _lib.DEV_ELL_RANGE


def test_production_scheduler_over_rounds_matches_oracle():
    """Round 0: Algorithm 1's own count; round t >= 1: the global search on
    round t-1's survivals gives the capacity, the top-K of round t's survivals
    the admitted set.  The rounds are replayed from one captured graph whose
    capacity changes between replays."""
    from speculative_decoding_draft_rank_b200.production import ProductionScheduler
    B, G = 256, 5
    rng = np.random.default_rng(21)
    kn, kt = PROFILES["step"]
    ps = ProductionScheduler(B, G, kn, kt, budget=-1)
    S = torch.zeros((B, G), dtype=torch.float32, device="cuda")
    ell = torch.zeros(B, dtype=torch.int32, device="cuda")
    nadm = torch.zeros(1, dtype=torch.int32, device="cuda")
    order = torch.zeros(B * G, dtype=torch.int32, device="cuda")
    st = torch.cuda.Stream()
    rounds = [_survivals(rng, B, G, t % 2 == 1) for t in range(6)]
    # Eager round 0 (no history).
    S.copy_(_dev(rounds[0]))
    torch.cuda.synchronize()
    ps.start_round(st)
    ps.select(S, ell, nadm, order, st)
    st.synchronize()
    ref0 = oracle.schedule(rounds[0].astype(np.float64), kn, kt, -1, oracle.SCHED_GREEDY_EARLY_STOP)
    assert int(nadm.item()) == ref0.n_adm and np.array_equal(ell.cpu().numpy(), ref0.ell)
    # Eager round 1, then rounds 2.. from one graph.
    def one_round():
        ps.start_round(st)
        ps.select(S, ell, nadm, order, st)
    S.copy_(_dev(rounds[1]))
    torch.cuda.synchronize()
    one_round()
    st.synchronize()
    cap, oell, onadm, oorder = oracle.production_schedule(rounds[0].astype(np.float64),
                                                          rounds[1].astype(np.float64), kn, kt)
    assert int(ps.capacity.item()) == cap and int(nadm.item()) == onadm
    assert np.array_equal(ell.cpu().numpy(), oell) and np.array_equal(order.cpu().numpy(), oorder)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        one_round()
    for t in range(2, len(rounds)):
        S.copy_(_dev(rounds[t]))
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            g.replay()
        st.synchronize()
        torch.cuda.synchronize()
        cap, oell, onadm, oorder = oracle.production_schedule(rounds[t - 1].astype(np.float64),
                                                              rounds[t].astype(np.float64), kn, kt)
        assert int(ps.capacity.item()) == cap, t
        assert int(nadm.item()) == onadm and np.array_equal(ell.cpu().numpy(), oell), t
        assert np.array_equal(order.cpu().numpy(), oorder), t
    g.reset()
    assert ps.device_status() == 0
