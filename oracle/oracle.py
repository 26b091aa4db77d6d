"""ctypes front end of the fp64 CPU oracle (``dspark_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU-baseline leg
of the benchmark are the only callers.  The product path never imports this
module, and this module imports nothing from the product package.

The four functions mirror the four stages of one DSpark round (drafting with
the Markov head, confidence/survival, the Algorithm-1 scheduler, rejection-
sampling verification).  Arrays are numpy; float inputs are passed as fp32
(bf16 values are carried exactly in fp32), uniforms as fp64.  The Markov
factor W is taken in the orientation the method writes it, [r, V].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dspark_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SCHED_ALL = 0
SCHED_GREEDY_EARLY_STOP = 1
SCHED_GLOBAL_ARGMAX = 2  # offline search without early stop (negative control)

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with plain gcc -O2 (no fast-math, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        use_library(build())
    return _lib


def use_library(path: str) -> None:
    """Point the front end at a compiled oracle (the tests load deliberately
    broken copies this way to show that the pins catch them)."""
    global _lib
    lib = ctypes.CDLL(path)
    for name in ("dspark_oracle_draft", "dspark_oracle_draft_head", "dspark_oracle_confidence",
                 "dspark_oracle_schedule", "dspark_oracle_verify", "dspark_oracle_verify_head"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib


def source_path() -> str:
    return _SRC


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: oracle returned status {rc}")


@dataclass
class DraftResult:
    x: np.ndarray        # [B, G] int32
    pd: np.ndarray       # [B, G] p_d(x)
    rowmax: np.ndarray   # [B, G] max_v (L + Delta)_v, before the temperature
    rowsum: np.ndarray   # [B, G] sum_v exp(z_v - max z), z = (L + Delta) / T
    margin: np.ndarray   # [B, G] decision margin


def draft(L, U, W, x0, temp, u_draft, force_x=None, A=None) -> DraftResult:
    """Semi-autoregressive drafting.  L [B,G,V], U [V,r], W [r,V], x0 [B],
    temp [B], u_draft [B,G]; A [r,r] selects the RNN head (state
    h_k = tanh(h_{k-1} A + U[x_{k-1}]), bias h_k W), None the Markov head."""
    L = _f32(L); U = _f32(U); W = _f32(W)
    B, G, V = L.shape
    r = U.shape[1]
    assert U.shape == (V, r) and W.shape == (r, V)
    Ar = _f32(A) if A is not None else None
    assert Ar is None or Ar.shape == (r, r)
    x0 = _i32(x0); temp = _f32(temp); u = _f64(u_draft)
    fx = _i32(force_x) if force_x is not None else None
    x = np.zeros((B, G), np.int32)
    pd = np.zeros((B, G)); rm = np.zeros((B, G)); rs = np.zeros((B, G)); mg = np.zeros((B, G))
    rc = _load().dspark_oracle_draft_head(B, G, V, r, _p(L), _p(U), _p(Ar), _p(W), _p(x0), _p(temp), _p(u),
                                          _p(fx), _p(x), _p(pd), _p(rm), _p(rs), _p(mg))
    _check(rc, "draft")
    return DraftResult(x, pd, rm, rs, mg)


def rnn_states(U, A, x0, x):
    """The RNN head's states h_1..h_G [B, G, r] (fp64) along the drafted
    tokens x [B, G] from x0 [B]: h_k = tanh(h_{k-1} A + U[x_{k-1}])."""
    U = _f32(U); A = _f32(A); x0 = _i32(x0); x = _i32(x)
    B, G = x.shape
    V, r = U.shape
    h = np.zeros((B, G, r))
    rc = _load().dspark_oracle_rnn_states(B, G, V, r, _p(U), _p(A), _p(x0), _p(x), _p(h))
    _check(rc, "rnn_states")
    return h


def confidence(h, w, bias=0.0, tau=None):
    """Linear confidence head and prefix survival.  h [B,G,d], w [d] -> (c, S) fp64 [B,G]."""
    h = _f32(h); w = _f32(w)
    B, G, d = h.shape
    t = _f64(tau) if tau is not None else None
    c = np.zeros((B, G)); S = np.zeros((B, G))
    rc = _load().dspark_oracle_confidence(B, G, d, _p(h), _p(w), ctypes.c_double(bias), _p(t),
                                          _p(c), _p(S))
    _check(rc, "confidence")
    return c, S


@dataclass
class ScheduleResult:
    ell: np.ndarray          # [B] admitted prefix length per request
    n_adm: int               # admitted candidates
    theta: float             # objective at the admitted count
    order: np.ndarray        # [B*G] sorted candidate indices (idx = i*B + b)
    margin_theta: float      # relative objective change at the stop point (+inf: no stop comparison)
    margin_gap: float        # survival gap across the cut
    margins: np.ndarray      # [B*G] relative objective change of every comparison made (NaN: not made)


def schedule(S, knots_n, knots_t, budget=-1, mode=SCHED_GREEDY_EARLY_STOP, force_n=-1) -> ScheduleResult:
    """Algorithm-1 admission over survivals S [B,G] against profile knots."""
    S = _f64(S)
    B, G = S.shape
    kn = _i32(knots_n); kt = _f64(knots_t)
    ell = np.zeros(B, np.int32); order = np.zeros(B * G, np.int32)
    n_adm = ctypes.c_int(0); th = ctypes.c_double(0); mth = ctypes.c_double(0); mgap = ctypes.c_double(0)
    margins = np.zeros(B * G)
    rc = _load().dspark_oracle_schedule(B, G, _p(S), len(kn), _p(kn), _p(kt), int(budget), int(mode),
                                        int(force_n), _p(ell), ctypes.byref(n_adm), ctypes.byref(th),
                                        _p(order), ctypes.byref(mth), ctypes.byref(mgap), _p(margins))
    _check(rc, "schedule")
    return ScheduleResult(ell, n_adm.value, th.value, order, mth.value, mgap.value, margins)


def schedule_threshold(S, threshold, budget=-1):
    """Static-threshold pruning over survivals S [B,G]: the sorted candidates
    with S >= threshold, at most `budget`.  Returns (ell [B], n_adm, order)."""
    S = _f64(S)
    B, G = S.shape
    ell = np.zeros(B, np.int32); order = np.zeros(B * G, np.int32)
    n_adm = ctypes.c_int(0)
    rc = _load().dspark_oracle_schedule_threshold(B, G, _p(S), ctypes.c_double(float(threshold)), int(budget),
                                                  _p(ell), ctypes.byref(n_adm), _p(order))
    _check(rc, "schedule_threshold")
    return ell, n_adm.value, order


def schedule_topk(S, capacity, budget=-1):
    """Dynamic top-K admission over survivals S [B,G]: the first `capacity`
    candidates of the stable order (clamped to [0, B*G]), at most `budget`.
    Returns (ell [B], n_adm, order)."""
    S = _f64(S)
    B, G = S.shape
    ell = np.zeros(B, np.int32); order = np.zeros(B * G, np.int32)
    n_adm = ctypes.c_int(0)
    rc = _load().dspark_oracle_schedule_topk(B, G, _p(S), int(capacity), int(budget), _p(ell),
                                             ctypes.byref(n_adm), _p(order))
    _check(rc, "schedule_topk")
    return ell, n_adm.value, order


def production_schedule(S_prev, S_cur, knots_n, knots_t, budget=-1):
    """The production scheduler's two steps for one round: the capacity from
    the previous round's survivals (the global search of Theta over the
    profile, which copes with non-smooth capacity curves), then the top-K of
    the current round's candidates.  Returns (capacity, ell, n_adm, order)."""
    cap = schedule(S_prev, knots_n, knots_t, budget, SCHED_GLOBAL_ARGMAX).n_adm
    ell, n_adm, order = schedule_topk(S_cur, cap, budget)
    return cap, ell, n_adm, order


@dataclass
class VerifyResult:
    acc: np.ndarray          # [B] accepted count A
    tokens: np.ndarray       # [B, G+1] emitted tokens, -1 padded
    nout: np.ndarray         # [B] A + 1
    pt_x: np.ndarray         # [B, G] p_t(x_k) for admitted k
    pd_x: np.ndarray         # [B, G] p_d(x_k) for admitted k
    margin_acc: np.ndarray   # [B, G]
    margin_fin: np.ndarray   # [B]
    final_kind: np.ndarray   # [B] 0 residual, 1 bonus, 2 greedy, 3 empty residual


def verify(Tlog, L, U, W, x0, x, temp, u_accept, u_final, ell, force_accept=None, A=None) -> VerifyResult:
    """Rejection-sampling verification over the admitted prefixes (A: the
    RNN head's recurrent matrix, as for draft; None for the Markov head)."""
    Tlog = _f32(Tlog); L = _f32(L); U = _f32(U); W = _f32(W)
    Ar = _f32(A) if A is not None else None
    B, G1, V = Tlog.shape
    G = G1 - 1
    r = U.shape[1]
    assert L.shape == (B, G, V) and U.shape == (V, r) and W.shape == (r, V)
    x0 = _i32(x0); x = _i32(x); temp = _f32(temp)
    ua = _f64(u_accept); uf = _f64(u_final); ell = _i32(ell)
    fa = _i32(force_accept) if force_accept is not None else None
    acc = np.zeros(B, np.int32); tok = np.zeros((B, G + 1), np.int32); nout = np.zeros(B, np.int32)
    ptx = np.zeros((B, G)); pdx = np.zeros((B, G)); ma = np.zeros((B, G)); mf = np.zeros(B)
    kind = np.zeros(B, np.int32)
    rc = _load().dspark_oracle_verify_head(B, G, V, r, _p(Tlog), _p(L), _p(U), _p(Ar), _p(W), _p(x0), _p(x),
                                           _p(temp), _p(ua), _p(uf), _p(ell), _p(fa), _p(acc), _p(tok),
                                           _p(nout), _p(ptx), _p(pdx), _p(ma), _p(mf), _p(kind))
    _check(rc, "verify")
    return VerifyResult(acc, tok, nout, ptx, pdx, ma, mf, kind)
