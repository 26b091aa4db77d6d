"""Seeded synthetic inputs for one DSpark round.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CUDA path and the CPU oracle are fed from it.

Recipe (one numpy PCG64 child stream per tensor, spawned from
``SeedSequence(seed)``, so every tensor is reproducible on its own and the
large ones can be drawn in fixed-size chunks):

* base logits  [B, G+1, V] ~ N(0, sigma_base^2), plus ``hot`` distinct token
  ids per (b, row) raised by ``hot_boost`` -- the backbone's confident tokens;
* target logits row k (1-based, k = 1..G+1) = base row k + N(0, (sigma_t k)^2),
  so agreement with the draft decays along the block;
* draft logits L = base rows 1..G (the parallel backbone's output);
* Markov factors U [V, r] and W [r, V] ~ N(0, 1/r);
* confidence hidden states h [B, G, d] ~ N(0, 1), weight w [d] ~ N(0, 1/d),
  bias 0;
* x0 [B] uniform over the vocabulary (last committed token per request);
* uniforms u_draft [B, G], u_accept [B, G], u_final [B] in [0, 1), fp32.

bf16 workloads round every float tensor once, to nearest even, on the host;
the device receives the bf16 bit patterns and the oracle the same values
widened exactly to fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

_CHUNK_ROWS = 64  # rows of V drawn per call for the large logit tensors


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns exactly to fp32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class RoundInputs:
    """One round's inputs.  Float tensors are fp32 arrays holding exactly the
    values the device sees; ``bits`` holds the bf16 patterns for bf16 rounds."""
    B: int
    G: int
    V: int
    r: int
    d: int
    dtype: str                    # "f32" or "bf16"
    L: np.ndarray                 # [B, G, V]
    Tlog: np.ndarray              # [B, G+1, V]
    U: np.ndarray                 # [V, r]
    W: np.ndarray                 # [r, V]
    h: np.ndarray                 # [B, G, d]
    w: np.ndarray                 # [d]
    bias: float
    x0: np.ndarray                # [B] int32
    temp: np.ndarray              # [B] fp32
    u_draft: np.ndarray           # [B, G] fp32
    u_accept: np.ndarray          # [B, G] fp32
    u_final: np.ndarray           # [B] fp32
    bits: dict = field(default_factory=dict)


def _normal_rows(rng, rows: int, V: int, scale: float) -> np.ndarray:
    out = np.empty((rows, V), np.float32)
    for s in range(0, rows, _CHUNK_ROWS):
        e = min(rows, s + _CHUNK_ROWS)
        out[s:e] = rng.standard_normal((e - s, V), dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out


def generate(B: int, G: int, V: int, r: int, d: int, dtype: str = "bf16", seed: int = 0,
             sigma_base: float = 2.0, hot: int = 16, hot_boost: float = 6.0,
             sigma_t: float = 0.3, temps=None) -> RoundInputs:
    """Draw one round's inputs.  ``temps``: None (all 1.0), a scalar, or a
    length-B sequence of per-request temperatures."""
    assert dtype in ("f32", "bf16")
    ss = np.random.SeedSequence(seed)
    (s_base, s_hot, s_noise, s_u, s_w, s_h, s_cw, s_x0, s_ud, s_ua, s_uf) = ss.spawn(11)
    gen = lambda s: np.random.Generator(np.random.PCG64(s))

    rows = B * (G + 1)
    base = _normal_rows(gen(s_base), rows, V, sigma_base)
    rh = gen(s_hot)
    for row in range(rows):
        idx = rh.choice(V, size=hot, replace=False)
        base[row, idx] += np.float32(hot_boost)
    base = base.reshape(B, G + 1, V)

    noise = _normal_rows(gen(s_noise), rows, V, 1.0).reshape(B, G + 1, V)
    kscale = (sigma_t * np.arange(1, G + 2, dtype=np.float32)).astype(np.float32)
    noise *= kscale[None, :, None]
    noise += base
    Tlog = noise
    L = np.ascontiguousarray(base[:, :G, :])
    del base

    U = gen(s_u).standard_normal((V, r), dtype=np.float32) * np.float32(1.0 / np.sqrt(r))
    W = gen(s_w).standard_normal((r, V), dtype=np.float32) * np.float32(1.0 / np.sqrt(r))
    h = gen(s_h).standard_normal((B, G, d), dtype=np.float32)
    w = gen(s_cw).standard_normal(d, dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
    x0 = gen(s_x0).integers(0, V, size=B, dtype=np.int64).astype(np.int32)
    u_draft = gen(s_ud).random((B, G), dtype=np.float32)
    u_accept = gen(s_ua).random((B, G), dtype=np.float32)
    u_final = gen(s_uf).random(B, dtype=np.float32)

    if temps is None:
        temp = np.ones(B, np.float32)
    elif np.isscalar(temps):
        temp = np.full(B, temps, np.float32)
    else:
        temp = np.asarray(temps, np.float32)
        assert temp.shape == (B,)

    bits = {}
    if dtype == "bf16":
        for name, arr in (("L", L), ("Tlog", Tlog), ("U", U), ("W", W), ("h", h), ("w", w)):
            bits[name] = bf16_bits(arr)
        L = bf16_to_f32(bits["L"]).reshape(L.shape)
        Tlog = bf16_to_f32(bits["Tlog"]).reshape(Tlog.shape)
        U = bf16_to_f32(bits["U"]).reshape(U.shape)
        W = bf16_to_f32(bits["W"]).reshape(W.shape)
        h = bf16_to_f32(bits["h"]).reshape(h.shape)
        w = bf16_to_f32(bits["w"]).reshape(w.shape)
    return RoundInputs(B, G, V, r, d, dtype, np.ascontiguousarray(L), np.ascontiguousarray(Tlog),
                       U, W, h, w, 0.0, x0, temp, u_draft, u_accept, u_final, bits)


def select_requests(inp: RoundInputs, idx) -> RoundInputs:
    """The inputs of a subset of requests (shared factors kept whole)."""
    idx = np.asarray(idx)
    bits = {k: (v[idx] if k in ("L", "Tlog", "h") else v) for k, v in inp.bits.items()}
    return RoundInputs(len(idx), inp.G, inp.V, inp.r, inp.d, inp.dtype, inp.L[idx], inp.Tlog[idx],
                       inp.U, inp.W, inp.h[idx], inp.w, inp.bias, inp.x0[idx], inp.temp[idx],
                       inp.u_draft[idx], inp.u_accept[idx], inp.u_final[idx], bits)


@dataclass
class CalibrationSet:
    """Labelled confidence-head outputs of N verified draft blocks.

    z [N, G] fp32: the head's logits (w . h + bias) per position;
    acc [N] int32: the accepted count A of each block, verified at full
    length G (positions 1..A accepted, A + 1 rejected when A < G);
    k [G] fp32: the over-confidence factor the logits were scaled by;
    t [N, G] fp32: the latent logits whose logistic law drew acceptance."""
    N: int
    G: int
    z: np.ndarray
    acc: np.ndarray
    k: np.ndarray
    t: np.ndarray


def calibration_set(N: int, G: int, k=2.0, seed: int = 0, mu0: float = 2.5, dmu: float = 0.5,
                    sigma: float = 1.5) -> CalibrationSet:
    """Draw a calibration set with a known miscalibration.

    Recipe (one PCG64 child stream per tensor from ``SeedSequence(seed)``):
    latent logits t[n, i] ~ N(mu0 - dmu * i, sigma^2) for i = 0..G-1, so the
    per-position acceptance falls along the block; independent logistic
    noise e[n, i] ~ Logistic(0, 1); position i passes when e < t (an event of
    probability 1 / (1 + exp(-t)), drawn without evaluating it); A is the
    number of leading passes.  The head reports z = k_i * t: k > 1 is an
    over-confident head (the pages report raw ECE of 3-8 %), k < 1 an
    under-confident one.  ``k`` is a scalar or a length-G sequence."""
    ss = np.random.SeedSequence(seed)
    s_t, s_e = ss.spawn(2)
    gen = lambda s: np.random.Generator(np.random.PCG64(s))
    mu = (np.float32(mu0) - np.float32(dmu) * np.arange(G, dtype=np.float32)).astype(np.float32)
    t = gen(s_t).standard_normal((N, G), dtype=np.float32) * np.float32(sigma) + mu[None, :]
    e = gen(s_e).logistic(0.0, 1.0, size=(N, G)).astype(np.float32)
    passed = e < t
    acc = np.where(passed.all(axis=1), G, np.argmin(passed, axis=1)).astype(np.int32)
    kk = np.broadcast_to(np.asarray(k, dtype=np.float32), (G,)).astype(np.float32)
    z = (t * kk[None, :]).astype(np.float32)
    return CalibrationSet(N, G, np.ascontiguousarray(z), acc, kk, t)


def tau_grid(K: int = 65, lo: float = 0.25, hi: float = 4.0) -> np.ndarray:
    """K log-spaced candidate temperatures from lo to hi (fp32); with the
    defaults the middle entry is exactly 1."""
    g = np.exp(np.linspace(np.log(lo), np.log(hi), K)).astype(np.float32)
    if K % 2 == 1 and abs(np.log(lo) + np.log(hi)) < 1e-12:
        g[K // 2] = np.float32(1.0)
    return g


def rnn_matrix(r: int, seed: int = 0, gain: float = 0.8) -> np.ndarray:
    """A recurrent matrix [r, r] ~ N(0, gain^2 / r) (fp32) for the RNN head:
    with gain < 1 the state update is contractive on average."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0x52])))
    return (g.standard_normal((r, r), dtype=np.float32) * np.float32(gain / np.sqrt(r))).astype(np.float32)
