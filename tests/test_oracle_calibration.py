"""Pins of the calibration oracle (sequential temperature scaling, ECE,
ROC-AUC) to facts that do not come from the oracle itself: hand-worked
examples, a closed form (a head whose logits are k times the true logits is
calibrated exactly at temperature k), special cases, library routines, and
planted mistakes that the pins must catch.

Sources: paperlayer.ai summary of DSpark, §3.2 Confidence-scheduled
verification (STS calibrates the running products left to right by ECE);
menfem.com KB entry, "Key Contributions" and "Results" (raw ROC-AUC
0.81-0.90, ECE 3-8 %, about 1 % after STS)."""
import types

import numpy as np
import pytest

from oracle import calibration as C
from speculative_decoding_draft_rank_b200 import synth


# ------------------------------------------------------------------ pins
def pin_labels(m):
    y = m.labels_from_accepts(np.array([0, 1, 5, 3], np.int32), 5)
    want = np.array([[0, 0, 0, 0, 0], [1, 0, 0, 0, 0], [1, 1, 1, 1, 1], [1, 1, 1, 0, 0]])
    assert np.array_equal(y, want)


def pin_ece_hand(m):
    # Bins of width 0.1: 0.05 -> 0, 0.15 -> 1, 0.95 and 0.97 -> 9.
    # |0 - 0.05| + |1 - 0.15| + |(1 - 0.95) + (1 - 0.97)| = 0.05 + 0.85 + 0.08.
    s = np.array([0.05, 0.15, 0.95, 0.97])
    y = np.array([0, 1, 1, 1])
    for f in (m.ece, m.ece_vec):
        assert f(s, y, 10) == pytest.approx(0.98 / 4, abs=1e-15)
    # Errors of opposite sign inside one bin cancel (ECE, not mean |y - s|):
    # 0.42 and 0.48 share bin 4; (1 - 0.42) + (0 - 0.48) = 0.10.
    assert m.ece_vec(np.array([0.42, 0.48]), np.array([1, 0]), 10) == pytest.approx(0.05, abs=1e-15)
    # The top edge belongs to the last bin; 0.5 with 2 bins to the upper one.
    assert m.ece_vec(np.array([1.0, 0.5]), np.array([1, 0]), 2) == pytest.approx(0.25, abs=1e-15)


def pin_ece_calibrated_zero(m):
    # Every bin's mean label equals its mean score.
    s = np.array([0.25] * 4 + [0.75] * 4)
    y = np.array([1, 0, 0, 0, 1, 1, 0, 1])
    assert m.ece(s, y, 10) == pytest.approx(0.0, abs=1e-15)
    assert m.ece_vec(s, y, 10) == pytest.approx(0.0, abs=1e-15)


def pin_sts_recovers_k(m):
    # Logits k_i * t with acceptance drawn from sigmoid(t): temperature k_i
    # makes every running product the true survival, so the fit lands next
    # to k_i at each position, and only if earlier positions stay fixed at
    # their fitted values.
    k = [2.0, 0.7, 1.5]
    cs = synth.calibration_set(100000, 3, k=k, seed=1)
    tau, e_raw, e_fit, _ = m.sts_fit(cs.z, cs.acc, synth.tau_grid(), 15)
    assert np.all(np.abs(np.log(tau / np.array(k))) < np.log(1.06)), tau
    assert np.all(e_raw > 0.01) and np.all(e_fit < 0.006), (e_raw, e_fit)


def pin_first_minimum(m):
    # z = 0: every temperature gives 1/2, every ECE is the same: the first
    # grid entry is the one chosen.
    z = np.zeros((64, 2), np.float32)
    acc = np.arange(64, dtype=np.int32) % 3
    grid = np.array([0.5, 1.0, 2.0], np.float32)
    tau, _, _, ece_all = m.sts_fit(z, acc, grid, 10)
    assert np.all(ece_all == ece_all[:, :1])
    assert np.array_equal(tau, np.array([0.5, 0.5], np.float32))


def pin_invalid_candidates(m):
    # Entries that are not positive finite numbers are never chosen.
    cs = synth.calibration_set(2000, 2, k=2.0, seed=5)
    grid = np.array([0.0, -1.0, np.nan, 2.0, np.inf], np.float32)
    tau, _, _, ece_all = m.sts_fit(cs.z, cs.acc, grid, 10)
    assert np.array_equal(tau, np.array([2.0, 2.0], np.float32))
    assert np.all(np.isinf(ece_all[:, [0, 1, 2, 4]])) and np.all(np.isfinite(ece_all[:, 3]))


def pin_single_candidate(m):
    # A one-entry grid applies that temperature: the first position's survival
    # is sigmoid(z / tau), here z = tau * log(3) so every score is 3/4.
    tau0 = np.float32(0.5)
    z = np.full((40, 1), np.float32(tau0 * np.log(3.0)), np.float32)
    acc = (np.arange(40) % 4 != 0).astype(np.int32)       # 30 of 40 accepted
    tau, _, e_fit, _ = m.sts_fit(z, acc, np.array([tau0]), 4)
    assert tau[0] == tau0
    assert e_fit[0] == pytest.approx(0.0, abs=1e-7)


def pin_auc(m):
    s = np.array([0.9, 0.8, 0.7, 0.6])
    y = np.array([1, 0, 1, 0])
    assert m.roc_auc(s, y) == (6, 4)           # 3 of 4 pairs ordered
    # A tie counts one half.
    assert m.roc_auc(np.array([0.5, 0.5]), np.array([1, 0])) == (1, 1)
    rng = np.random.default_rng(3)
    s = np.round(rng.random(500), 2)           # many ties
    y = rng.random(500) < s
    twice, pairs = m.roc_auc(s, y)
    from scipy.stats import mannwhitneyu
    u = mannwhitneyu(s[y], s[~y], alternative="two-sided").statistic
    assert twice == int(round(2 * u)) and pairs == int(y.sum()) * int((~y).sum())


PINS = [pin_labels, pin_ece_hand, pin_ece_calibrated_zero, pin_sts_recovers_k, pin_first_minimum,
        pin_invalid_candidates, pin_single_candidate, pin_auc]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(C)


def test_loop_and_vector_ece_agree():
    rng = np.random.default_rng(0)
    s = rng.random(2000)
    y = (rng.random(2000) < s).astype(int)
    assert C.ece(s, y, 15) == C.ece_vec(s, y, 15)


def test_survival_non_increasing_and_ordering():
    cs = synth.calibration_set(5000, 5, k=1.7, seed=2)
    tau, _, _, _ = C.sts_fit(cs.z, cs.acc, synth.tau_grid(), 15)
    S = C.survival(cs.z, tau)
    assert np.all(np.diff(S, axis=1) <= 0)
    # Within a position, a positive temperature keeps the order of the logits'
    # sigmoid factor; at the first position that is the order of S itself.
    o = np.argsort(cs.z[:, 0], kind="stable")
    assert np.all(np.diff(S[o, 0]) >= 0)


def test_generator_acceptance_decays():
    cs = synth.calibration_set(50000, 5, seed=0)
    y = C.labels_from_accepts(cs.acc, 5)
    rate = y.mean(axis=0)
    assert np.all(np.diff(rate) < 0) and rate[0] > 0.7


# ------------------------------------------------------ planted mistakes
MUTANTS = [
    ("tau_multiplies", "e(prev * sigmoid(z[:, i] / t)", "e(prev * sigmoid(z[:, i] * t)"),
    ("label_strict", "acc[:, None] >= np.arange(1, G + 1)", "acc[:, None] > np.arange(1, G + 1)"),
    ("prefix_not_carried", "prev = prev * sigmoid(z[:, i] / float(grid[kstar]))", "prev = prev * sigmoid(z[:, i])"),
    ("bin_rounded", "np.minimum(M - 1, np.floor(s * M)", "np.minimum(M - 1, np.round(s * M)"),
    ("ece_absolute_per_sample", "np.add.at(acc, b, np.asarray(y, dtype=np.float64) - s)",
     "np.add.at(acc, b, np.abs(np.asarray(y, dtype=np.float64) - s))"),
    ("argmin_last", "ece_all[i] == least)[0])", "ece_all[i] == least)[-1])"),
    ("auc_tie_full", "int(np.count_nonzero(p == neg))", "2 * int(np.count_nonzero(p == neg))"),
    ("sigmoid_sign", "1.0 / (1.0 + np.exp(-x))", "1.0 / (1.0 + np.exp(x))"),
]


def _mutant(name, old, new):
    src = open(C.__file__).read()
    assert src.count(old) == 1, name
    mod = types.ModuleType(f"calibration_{name}")
    exec(compile(src.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, old, new):
    m = _mutant(name, old, new)
    caught = []
    for pin in PINS:
        try:
            pin(m)
        except Exception:   # an assertion or a crash both count as caught
            caught.append(pin.__name__)
    assert caught, f"no pin catches {name}"
