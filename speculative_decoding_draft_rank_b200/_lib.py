"""ctypes binding of libdspark (the C ABI declared in include/dspark.h).

Argument marshalling only: torch tensors supply device pointers and sizes,
torch streams supply the cudaStream_t.  Every step of the round runs in the
library's CUDA kernels; there is no fallback.  Importing this module on a
machine without the built library, or calling it without a CUDA device,
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdspark.so")

DSPARK_F32 = 0
DSPARK_BF16 = 1
SCHED_ALL = 0
SCHED_GREEDY_EARLY_STOP = 1
SCHED_GLOBAL_ARGMAX = 2
SCHED_THRESHOLD = 3
SCHED_TOPK = 4

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED_DTYPE", 3: "WORKSPACE", 4: "CUDA", 5: "TIMEOUT"}
DEV_TOKEN_RANGE, DEV_ELL_RANGE, DEV_BAD_TEMP, DEV_TIMEOUT, DEV_BAD_VALUE = 0x1, 0x2, 0x4, 0x8, 0x10

EXPORTS = ("dspark_version", "dspark_draft_workspace_size", "dspark_draft_markov", "dspark_confidence",
           "dspark_schedule_workspace_size", "dspark_schedule", "dspark_verify_workspace_size",
           "dspark_verify", "dspark_get_device_status", "dspark_clear_device_status",
           "dspark_draft_noalloc_max_scratch", "dspark_draft_markov_noalloc", "dspark_schedule_threshold",
           "dspark_sts_workspace_size", "dspark_sts_fit", "dspark_survival_auc", "dspark_schedule_topk",
           "dspark_draft_noalloc_device_status", "dspark_draft_rnn", "dspark_verify_rnn", "dspark_get_near_ties",
           "dspark_exp2_fma", "dspark_gather_admitted_targets")


class DsparkError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} returned {status} ({STATUS.get(status, '?')})")
        self.status = status


_lib = None
_vp, _i, _f, _sz, _d = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_double


def load() -> ctypes.CDLL:
    """Load libdspark.so from the package directory (build it first with
    ``python -m speculative_decoding_draft_rank_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libdspark.so is not built ({LIB_PATH}); run the package build step")
    lib = ctypes.CDLL(LIB_PATH)
    lib.dspark_version.restype = ctypes.c_char_p
    lib.dspark_draft_workspace_size.restype = _sz
    lib.dspark_draft_workspace_size.argtypes = [_i] * 5
    lib.dspark_draft_markov.restype = _i
    lib.dspark_draft_markov.argtypes = [_vp] * 6 + [_i] * 5 + [_vp, _sz] + [_vp] * 5
    lib.dspark_confidence.restype = _i
    lib.dspark_confidence.argtypes = [_vp, _vp, _f, _vp, _i, _i, _i, _i, _vp, _vp, _vp]
    lib.dspark_schedule_workspace_size.restype = _sz
    lib.dspark_schedule_workspace_size.argtypes = [_i, _i]
    lib.dspark_schedule.restype = _i
    lib.dspark_schedule.argtypes = [_vp, _i, _i, _vp, _vp, _i, _i, _i, _vp, _sz, _vp, _vp, _vp, _vp, _vp]
    lib.dspark_schedule_threshold.restype = _i
    lib.dspark_schedule_threshold.argtypes = [_vp, _i, _i, _f, _i, _vp, _sz, _vp, _vp, _vp, _vp]
    lib.dspark_verify_workspace_size.restype = _sz
    lib.dspark_verify_workspace_size.argtypes = [_i] * 5
    lib.dspark_verify.restype = _i
    lib.dspark_verify.argtypes = [_vp] * 13 + [_i] * 5 + [_vp, _sz] + [_vp] * 5
    lib.dspark_get_device_status.restype = _i
    lib.dspark_get_device_status.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.dspark_exp2_fma.restype = _i
    lib.dspark_exp2_fma.argtypes = [_vp, _vp, _i, _vp]
    lib.dspark_get_near_ties.restype = _i
    lib.dspark_get_near_ties.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32)]
    lib.dspark_clear_device_status.restype = _i
    lib.dspark_clear_device_status.argtypes = [_vp, _vp]
    lib.dspark_draft_noalloc_max_scratch.restype = _sz
    lib.dspark_draft_noalloc_max_scratch.argtypes = []
    lib.dspark_draft_markov_noalloc.restype = _i
    lib.dspark_draft_markov_noalloc.argtypes = [_vp] * 6 + [_i] * 5 + [_vp] * 5
    lib.dspark_draft_rnn.restype = _i
    lib.dspark_draft_rnn.argtypes = [_vp] * 7 + [_i] * 5 + [_vp, _sz] + [_vp] * 6
    lib.dspark_verify_rnn.restype = _i
    lib.dspark_verify_rnn.argtypes = [_vp] * 12 + [_i] * 5 + [_vp, _sz] + [_vp] * 5
    lib.dspark_draft_noalloc_device_status.restype = _i
    lib.dspark_draft_noalloc_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.dspark_schedule_topk.restype = _i
    lib.dspark_schedule_topk.argtypes = [_vp, _i, _i, _vp, _i, _vp, _sz, _vp, _vp, _vp, _vp]
    lib.dspark_sts_workspace_size.restype = _sz
    lib.dspark_sts_workspace_size.argtypes = [_i] * 4
    lib.dspark_sts_fit.restype = _i
    lib.dspark_sts_fit.argtypes = [_vp] * 3 + [_i] * 4 + [_vp, _sz] + [_vp] * 6
    lib.dspark_survival_auc.restype = _i
    lib.dspark_survival_auc.argtypes = [_vp, _vp, _i, _i, _vp, _vp, _vp]
    lib.dspark_gather_admitted_targets.restype = _i
    lib.dspark_gather_admitted_targets.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp]
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libdspark takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libdspark takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return DSPARK_BF16
    if t.dtype == torch.float32:
        return DSPARK_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _call(fn, *args):
    st = getattr(load(), fn)(*args)
    if st != 0:
        raise DsparkError(fn, st)


def version() -> str:
    return load().dspark_version().decode()


def dspark_draft_workspace_size(B, G, V, r, dtype) -> int:
    return int(load().dspark_draft_workspace_size(B, G, V, r, dtype))


def dspark_schedule_workspace_size(B, G) -> int:
    return int(load().dspark_schedule_workspace_size(B, G))


def dspark_verify_workspace_size(B, G, V, r, dtype) -> int:
    return int(load().dspark_verify_workspace_size(B, G, V, r, dtype))


def dspark_draft_markov(L, U, Wt, x0, temp, u_draft, ws, x_out, pd_x_out, rowmax_out, rowsum_out,
                        stream=None):
    B, G, V = L.shape
    r = U.shape[1]
    _call("dspark_draft_markov", _ptr(L), _ptr(U), _ptr(Wt), _ptr(x0), _ptr(temp), _ptr(u_draft), B, G, V,
          r, _dtype(L), _ptr(ws), ws.numel() * ws.element_size(), _ptr(x_out), _ptr(pd_x_out),
          _ptr(rowmax_out), _ptr(rowsum_out), _stream(stream))


def dspark_draft_rnn(L, U, Arec, Wt, x0, temp, u_draft, ws, x_out, pd_x_out, rowmax_out, rowsum_out, H_out,
                     stream=None):
    """Drafting with the RNN head: Arec [r, r] bf16 recurrent matrix; H_out
    [B, G, r] fp32 receives the state that biased every position."""
    B, G, V = L.shape
    r = U.shape[1]
    _call("dspark_draft_rnn", _ptr(L), _ptr(U), _ptr(Arec), _ptr(Wt), _ptr(x0), _ptr(temp), _ptr(u_draft), B, G,
          V, r, _dtype(L), _ptr(ws), ws.numel() * ws.element_size(), _ptr(x_out), _ptr(pd_x_out), _ptr(rowmax_out),
          _ptr(rowsum_out), _ptr(H_out), _stream(stream))


def dspark_verify_rnn(Tlog, L, H, Wt, x, pd_x, rowmax, rowsum, temp, u_accept, u_final, ell, ws, acc_out,
                      tokens_out, nout_out, pt_x_out=None, stream=None):
    """Verification of RNN-head drafts (the states H from dspark_draft_rnn)."""
    B, G1, V = Tlog.shape
    r = H.shape[2]
    _call("dspark_verify_rnn", _ptr(Tlog), _ptr(L), _ptr(H), _ptr(Wt), _ptr(x), _ptr(pd_x), _ptr(rowmax),
          _ptr(rowsum), _ptr(temp), _ptr(u_accept), _ptr(u_final), _ptr(ell), B, G1 - 1, V, r, _dtype(Tlog),
          _ptr(ws), ws.numel() * ws.element_size(), _ptr(acc_out), _ptr(tokens_out), _ptr(nout_out),
          _ptr(pt_x_out), _stream(stream))


def dspark_draft_noalloc_max_scratch() -> int:
    return int(load().dspark_draft_noalloc_max_scratch())


def dspark_draft_markov_noalloc(L, U, Wt, x0, temp, u_draft, x_out, pd_x_out, rowmax_out, rowsum_out,
                                stream=None):
    """Drafting with the library's own fixed scratch instead of a workspace."""
    B, G, V = L.shape
    r = U.shape[1]
    _call("dspark_draft_markov_noalloc", _ptr(L), _ptr(U), _ptr(Wt), _ptr(x0), _ptr(temp), _ptr(u_draft), B,
          G, V, r, _dtype(L), _ptr(x_out), _ptr(pd_x_out), _ptr(rowmax_out), _ptr(rowsum_out), _stream(stream))


def dspark_draft_noalloc_device_status(stream=None) -> int:
    """Status word of the last allocation-free drafting call on `stream`
    (synchronises the stream)."""
    out = ctypes.c_uint32(0)
    _call("dspark_draft_noalloc_device_status", _stream(stream), ctypes.byref(out))
    return int(out.value)


def dspark_confidence(h, w, bias, tau, c_out, S_out, stream=None):
    B, G, d = h.shape
    _call("dspark_confidence", _ptr(h), _ptr(w), ctypes.c_float(bias), _ptr(tau), B, G, d, _dtype(h),
          _ptr(c_out), _ptr(S_out), _stream(stream))


def dspark_schedule(S, knots_n, knots_t, budget, mode, ws, ell_out, n_adm_out, theta_out, order_out=None,
                    stream=None):
    B, G = S.shape
    _call("dspark_schedule", _ptr(S), B, G, _ptr(knots_n), _ptr(knots_t), knots_n.numel(), int(budget),
          int(mode), _ptr(ws), ws.numel() * ws.element_size(), _ptr(ell_out), _ptr(n_adm_out),
          _ptr(theta_out), _ptr(order_out), _stream(stream))


def dspark_schedule_threshold(S, threshold, budget, ws, ell_out, n_adm_out, order_out=None, stream=None):
    """Static-threshold pruning: the sorted candidates with S >= threshold."""
    B, G = S.shape
    _call("dspark_schedule_threshold", _ptr(S), B, G, ctypes.c_float(threshold), int(budget), _ptr(ws),
          ws.numel() * ws.element_size(), _ptr(ell_out), _ptr(n_adm_out), _ptr(order_out), _stream(stream))


def dspark_schedule_topk(S, capacity, budget, ws, ell_out, n_adm_out, order_out=None, stream=None):
    """Dynamic top-K: the first *capacity (a device int32) candidates of the
    stable order by S."""
    B, G = S.shape
    _call("dspark_schedule_topk", _ptr(S), B, G, _ptr(capacity), int(budget), _ptr(ws),
          ws.numel() * ws.element_size(), _ptr(ell_out), _ptr(n_adm_out), _ptr(order_out), _stream(stream))


def dspark_verify(Tlog, L, U, Wt, x0, x, pd_x, rowmax, rowsum, temp, u_accept, u_final, ell, ws, acc_out,
                  tokens_out, nout_out, pt_x_out=None, stream=None):
    B, G1, V = Tlog.shape
    r = U.shape[1]
    _call("dspark_verify", _ptr(Tlog), _ptr(L), _ptr(U), _ptr(Wt), _ptr(x0), _ptr(x), _ptr(pd_x),
          _ptr(rowmax), _ptr(rowsum), _ptr(temp), _ptr(u_accept), _ptr(u_final), _ptr(ell), B, G1 - 1, V, r,
          _dtype(Tlog), _ptr(ws), ws.numel() * ws.element_size(), _ptr(acc_out), _ptr(tokens_out),
          _ptr(nout_out), _ptr(pt_x_out), _stream(stream))


def dspark_sts_workspace_size(N, G, K, n_bins) -> int:
    return int(load().dspark_sts_workspace_size(N, G, K, n_bins))


def dspark_sts_fit(z, acc, tau_grid, n_bins, ws, tau_out, ece_raw_out=None, ece_fit_out=None, ece_all_out=None,
                   S_out=None, stream=None):
    """Sequential temperature scaling: z [N, G] f32 logits, acc [N] int32,
    tau_grid [K] f32 candidates -> tau_out [G] f32 (and the optional ECEs,
    fp64, and fitted survivals S_out [N, G] f32)."""
    N, G = z.shape
    K = tau_grid.shape[0]
    _call("dspark_sts_fit", _ptr(z), _ptr(acc), _ptr(tau_grid), N, G, K, int(n_bins), _ptr(ws),
          ws.numel() * ws.element_size(), _ptr(tau_out), _ptr(ece_raw_out), _ptr(ece_fit_out), _ptr(ece_all_out),
          _ptr(S_out), _stream(stream))


def dspark_survival_auc(S, acc, twice_out, pairs_out, stream=None):
    """ROC-AUC pair counts per position: twice_out, pairs_out [G] int64
    tensors (uint64 bit patterns); AUC = twice / (2 * pairs)."""
    N, G = S.shape
    _call("dspark_survival_auc", _ptr(S), _ptr(acc), N, G, _ptr(twice_out), _ptr(pairs_out), _stream(stream))


def dspark_get_device_status(ws, stream=None) -> int:
    out = ctypes.c_uint32(0)
    _call("dspark_get_device_status", _ptr(ws), _stream(stream), ctypes.byref(out))
    return int(out.value)


def dspark_get_near_ties(ws, stream=None):
    """(drafting, verification) near-tie counts of a workspace since its last
    clear (synchronises the stream)."""
    d, v = ctypes.c_uint32(0), ctypes.c_uint32(0)
    _call("dspark_get_near_ties", _ptr(ws), _stream(stream), ctypes.byref(d), ctypes.byref(v))
    return int(d.value), int(v.value)


def dspark_gather_admitted_targets(Tlog_host, Tlog_dev, ell, stream=None):
    """Enqueue one kernel that copies rows 0..ell[b] of every request of the
    pinned host target logits [B, G+1, V] into the device buffer of the same
    layout; ell: the device int32 [B] of admitted lengths."""
    if Tlog_host.is_cuda or not Tlog_host.is_pinned() or not Tlog_host.is_contiguous():
        raise ValueError("Tlog_host must be a contiguous pinned host tensor")
    if Tlog_host.shape != Tlog_dev.shape or Tlog_host.dtype != Tlog_dev.dtype or ell.dtype != torch.int32:
        raise ValueError("Tlog_host and Tlog_dev differ in shape or dtype, or ell is not int32")
    B, G1, V = Tlog_dev.shape
    _call("dspark_gather_admitted_targets", ctypes.c_void_p(Tlog_host.data_ptr()), _ptr(Tlog_dev), _ptr(ell), B,
          G1 - 1, V, _dtype(Tlog_dev), _stream(stream))


def dspark_exp2_fma(x, y, stream=None):
    """y = 2^x (float32 device tensors of equal size) by the library's FMA-pipe polynomial."""
    _call("dspark_exp2_fma", _ptr(x), _ptr(y), int(x.numel()), _stream(stream))


def dspark_clear_device_status(ws, stream=None):
    _call("dspark_clear_device_status", _ptr(ws), _stream(stream))
