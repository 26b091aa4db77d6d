"""The synthetic round workloads: shapes, value distributions and throughput
profiles.  Pure data; the random draws live in ``synth``.

Profiles are piecewise-linear t(n) in microseconds through integer knots
(n_j, t_j) with n_0 = 0, continued past the last knot with the last slope.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import synth

MODE_ALL = 0
MODE_GREEDY_EARLY_STOP = 1


def _profile(t0: float, knots, slopes):
    """Knots n_0 = 0 < n_1 < ... and per-segment slopes -> (knots_n, knots_t)."""
    kn = [0] + list(knots[1:])
    kt = [t0]
    for j in range(1, len(kn)):
        kt.append(kt[-1] + slopes[j - 1] * (kn[j] - kn[j - 1]))
    return np.asarray(kn, np.int32), np.asarray(kt, np.float64)


@dataclass
class Workload:
    name: str
    B: int
    G: int
    V: int
    r: int
    d: int
    dtype: str
    sigma_t: float
    hot: int
    knots_n: np.ndarray
    knots_t: np.ndarray
    budget: int = -1
    mode: int = MODE_GREEDY_EARLY_STOP
    temps: object = None
    seed: int = 0
    extra: dict = field(default_factory=dict)

    def inputs(self) -> synth.RoundInputs:
        return synth.generate(self.B, self.G, self.V, self.r, self.d, self.dtype, seed=self.seed,
                              hot=self.hot, sigma_t=self.sigma_t, temps=self.temps)


def tiny() -> Workload:
    """B=4, G=5, V=1024, r=16, d=64, fp32; budget 12, t(n) = 1 + 0.05 n."""
    kn, kt = _profile(1.0, [0, 20], [0.05])
    return Workload("tiny_b4_g5_v1024_f32", 4, 5, 1024, 16, 64, "f32", 0.3, 8, kn, kt, budget=12)


def qwen_vocab() -> Workload:
    """B=64, G=5, V=151936, r=256, d=2560, bf16; every drafted position verified."""
    kn, kt = _profile(1000.0, [0], [])
    return Workload("qwen_vocab_b64_g5_v151936", 64, 5, 151936, 256, 2560, "bf16", 0.3, 16, kn, kt,
                    mode=MODE_ALL)


def headline() -> Workload:
    """B=256, G=5, V=129280, r=256, d=4096, bf16; profile knots {0,256,512,1024,1536}
    with slopes 0.2/0.5/1.0/2.0 us per token from t(0) = 1000 us."""
    kn, kt = _profile(1000.0, [0, 256, 512, 1024, 1536], [0.2, 0.5, 1.0, 2.0])
    return Workload("headline_b256_g5_v129280", 256, 5, 129280, 256, 4096, "bf16", 0.3, 16, kn, kt)


def saturated() -> Workload:
    """B=1024, G=8, V=129280, bf16; budget 0.5 B G; slope 0.25 us/token to n=2048
    then 0.5 from t(0) = 4000 us; temperatures 0 / 0.6 / 1.0 / 1.2 by quarter."""
    B, G = 1024, 8
    kn, kt = _profile(4000.0, [0, 2048, 4096], [0.25, 0.5])
    temps = np.repeat(np.asarray([0.0, 0.6, 1.0, 1.2], np.float32), B // 4)
    return Workload("saturated_b1024_g8_v129280", B, G, 129280, 256, 4096, "bf16", 0.4, 16, kn, kt,
                    budget=B * G // 2, temps=temps)


def long_block(G: int) -> Workload:
    """B=128, V=151936, r=256, d=2560, bf16, G in {4, 8, 12, 16}; the headline
    profile with its knots scaled by B G / 1280, from t(0) = 500 us."""
    B = 128
    s = B * G / 1280.0
    knots = [0] + [int(round(k * s)) for k in (256, 512, 1024, 1536)]
    kn, kt = _profile(500.0, knots, [0.2, 0.5, 1.0, 2.0])
    return Workload(f"long_block_b128_g{G}_v151936", B, G, 151936, 256, 2560, "bf16", 0.25, 16, kn, kt)


def all_workloads():
    return [tiny(), qwen_vocab(), headline(), saturated()] + [long_block(g) for g in (4, 8, 12, 16)]


@dataclass
class CalibrationWorkload:
    """A sequential-temperature-scaling fit: N verified blocks of G positions,
    K candidate temperatures, M ECE bins; the head's logits are k times the
    latent ones (an over-confident head when k > 1)."""
    name: str
    N: int
    G: int
    K: int
    M: int
    k: float = 2.0
    seed: int = 0

    def inputs(self) -> synth.CalibrationSet:
        return synth.calibration_set(self.N, self.G, k=self.k, seed=self.seed)

    def grid(self) -> np.ndarray:
        return synth.tau_grid(self.K)


def calibration_headline() -> CalibrationWorkload:
    """64 rounds of the headline batch (256 requests) verified at full length
    G = 5: N = 16384 labelled blocks; 65 log-spaced temperatures in [1/4, 4];
    15 bins."""
    return CalibrationWorkload("sts_n16384_g5_k65_m15", 16384, 5, 65, 15)
