"""Plain fp64 restatement of DSpark's confidence calibration.

TEST INFRASTRUCTURE ONLY.  This module is oracle code: only the tests, the
smoke check and the CPU-baseline leg of the benchmark may import it.  It shares
nothing with the CUDA library.

Sources (web pages about arXiv:2607.05147):
  [PL] paperlayer.ai section-by-section summary, §3.2 Confidence-scheduled
       verification: sequential temperature scaling (STS) calibrates the
       cumulative prefix-survival probabilities left to right, minimising the
       expected calibration error (ECE) of the running products of the
       per-position scores, while keeping their ordering.
  [KB] menfem.com knowledge-base entry, "Key Contributions" (post-hoc STS,
       left to right, lowers ECE) and "Results" (raw ROC-AUC 0.81-0.90, ECE
       3-8 %, about 1 % after STS).

Readings where the pages are silent (each is stated again beside the code):
  - the per-position score is c_i = sigmoid(z_i / tau_i) with z_i the linear
    head's logit (w . h + bias), i.e. the temperature divides the logit, as in
    ordinary temperature scaling;
  - the label of position i for a request is "the first i draft tokens were
    all accepted" (A >= i, A the accepted count of a round verified at full
    length), which is the event the prefix survival S_i = prod_{j<=i} c_j
    estimates;
  - ECE uses M equal-width bins on [0, 1] (bin = min(M - 1, floor(s * M))):
    ECE = sum over bins of |sum of (y - s) in the bin| / N;
  - "minimises ECE" is taken over a caller-given grid of candidate
    temperatures, position by position with the earlier positions' fitted
    temperatures held fixed; the first grid entry with the least ECE wins;
  - ROC-AUC counts, over every (positive, negative) pair, 1 when the
    positive scores higher and 1/2 on a tie, divided by the pair count.

Arithmetic: logits and temperatures are widened from fp32 to double; sums run
in index order; exp() is numpy's.
"""
from __future__ import annotations

import numpy as np


def sigmoid(x):
    """Logistic function, fp64."""
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def labels_from_accepts(acc, G):
    """y[n, i-1] = 1 if the first i draft tokens of sample n were accepted
    (A_n >= i), for i = 1..G ([PL] §3.2: the survival of the prefix)."""
    acc = np.asarray(acc, dtype=np.int64)
    return (acc[:, None] >= np.arange(1, G + 1)[None, :]).astype(np.int64)


def ece_bin(s, M):
    """Equal-width bin index of a score in [0, 1]: floor(s * M), the top edge
    folded into the last bin."""
    return min(M - 1, int(np.floor(s * M)))


def ece(s, y, M):
    """Expected calibration error of scores s against 0/1 labels y: the
    count-weighted mean over M equal-width bins of |mean label - mean score|,
    written as sum_bins |sum (y - s)| / N.  Sequential sums in index order."""
    s = np.asarray(s, dtype=np.float64)
    y = np.asarray(y)
    N = s.shape[0]
    acc = [0.0] * M
    for n in range(N):
        acc[ece_bin(s[n], M)] += float(y[n]) - float(s[n])
    tot = 0.0
    for m in range(M):
        tot += abs(acc[m])
    return tot / N


def ece_vec(s, y, M):
    """The same ECE with numpy binning (identical bins, sums in index order
    through np.add.at), for larger N."""
    s = np.asarray(s, dtype=np.float64)
    b = np.minimum(M - 1, np.floor(s * M).astype(np.int64))
    acc = np.zeros(M)
    np.add.at(acc, b, np.asarray(y, dtype=np.float64) - s)
    tot = 0.0
    for m in range(M):
        tot += abs(float(acc[m]))
    return tot / s.shape[0]


def survival(z, tau):
    """S[n, i] = prod_{j<=i} sigmoid(z[n, j] / tau[j]) ([PL] §3.2: the running
    product of the calibrated per-position scores)."""
    z = np.asarray(z, dtype=np.float32).astype(np.float64)
    tau = np.asarray(tau, dtype=np.float32).astype(np.float64)
    N, G = z.shape
    S = np.empty((N, G))
    prev = np.ones(N)
    for i in range(G):
        prev = prev * sigmoid(z[:, i] / tau[i])
        S[:, i] = prev
    return S


def sts_fit(z, acc, tau_grid, M, vectorised=True):
    """Sequential temperature scaling ([PL] §3.2; [KB] Key Contributions).

    For i = 1..G in turn, with tau_1..tau_{i-1} already fixed, every grid
    temperature t gives the candidate survivals S_{i-1} * sigmoid(z_i / t);
    tau_i is the first grid entry whose candidate has the least ECE against
    the labels y_i (A >= i).  A grid entry that is not a positive finite
    number is no temperature: its ECE counts as +inf (chosen only when no
    entry is valid, and then the first).  The ordering of the survivals along a request's
    prefix is kept by construction: every factor lies in (0, 1), so S_i never
    exceeds S_{i-1}.

    Returns (tau [G] as the grid's fp32 values, ece_raw [G] at tau = 1,
    ece_fit [G] at the fitted temperatures, ece_all [G, K] every candidate's
    ECE, the quantity the choice is made on)."""
    z = np.asarray(z, dtype=np.float32).astype(np.float64)
    grid = np.asarray(tau_grid, dtype=np.float32)
    N, G = z.shape
    K = grid.shape[0]
    y = labels_from_accepts(acc, G)
    e = ece_vec if vectorised else ece
    raw = survival(z, np.ones(G, dtype=np.float32))
    ece_raw = np.array([e(raw[:, i], y[:, i], M) for i in range(G)])
    tau = np.empty(G, dtype=np.float32)
    ece_fit = np.empty(G)
    ece_all = np.empty((G, K))
    prev = np.ones(N)
    for i in range(G):
        for k in range(K):
            t = float(grid[k])
            if not (np.isfinite(t) and t > 0.0):
                ece_all[i, k] = np.inf      # not a temperature: never preferred
                continue
            ece_all[i, k] = e(prev * sigmoid(z[:, i] / t), y[:, i], M)
        least = np.min(ece_all[i])
        kstar = int(np.flatnonzero(ece_all[i] == least)[0])   # first of the least
        tau[i] = grid[kstar]
        ece_fit[i] = ece_all[i, kstar]
        prev = prev * sigmoid(z[:, i] / float(grid[kstar]))
    return tau, ece_raw, ece_fit, ece_all


def roc_auc(s, y):
    """ROC-AUC by brute force over every (positive, negative) pair: 1 when the
    positive's score is higher, 1/2 on a tie ([KB] Results reports the raw
    confidence's ROC-AUC).  Returns (2 * the pair score as an integer, the
    pair count); AUC = first / (2 * second).  NaN-free inputs assumed."""
    s = np.asarray(s, dtype=np.float64)
    y = np.asarray(y).astype(bool)
    pos, neg = s[y], s[~y]
    twice = 0
    for p in pos:
        twice += 2 * int(np.count_nonzero(p > neg)) + int(np.count_nonzero(p == neg))
    return twice, int(pos.shape[0]) * int(neg.shape[0])
