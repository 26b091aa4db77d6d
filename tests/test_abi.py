"""The C ABI without a GPU: the library loads, exports every entry point that
include/dspark.h declares, and rejects bad arguments on the host with the
documented status codes (no CUDA call is reached on these paths)."""
import ctypes
import os
import re
import subprocess

import pytest

from speculative_decoding_draft_rank_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dspark.h")

FAKE = ctypes.c_void_p(0x100000)      # never dereferenced: every call below fails host checks first
FAKE_WS = ctypes.c_void_p(0x200000)   # 256-byte aligned


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(dspark_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_exports_match_header(lib):
    declared = _declared()
    assert declared, "no declarations parsed"
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (dspark_\w+)$", out, re.M))
    assert set(declared) <= exported, set(declared) - exported
    assert set(_lib.EXPORTS) == set(declared)
    for name in declared:
        assert hasattr(lib, name)


def test_version(lib):
    assert "sm_100a" in _lib.version()


def test_workspace_queries(lib):
    assert _lib.dspark_draft_workspace_size(256, 5, 129280, 256, _lib.DSPARK_BF16) > 0
    assert _lib.dspark_verify_workspace_size(256, 5, 129280, 256, _lib.DSPARK_BF16) > 0
    assert _lib.dspark_schedule_workspace_size(1024, 8) > 0
    assert _lib.dspark_draft_workspace_size(0, 5, 1000, 16, 0) == 0
    assert _lib.dspark_draft_workspace_size(4, 17, 1000, 16, 0) == 0
    assert _lib.dspark_draft_workspace_size(4, 5, 1, 16, 0) == 0
    assert _lib.dspark_draft_workspace_size(4, 5, 1000, 24, _lib.DSPARK_BF16) == 0  # r % 16
    assert _lib.dspark_schedule_workspace_size(4096, 16) == 0                    # B*G > 16384


def _draft(lib, B=4, G=5, V=1024, r=16, dtype=0, ws=FAKE_WS, ws_bytes=1 << 30, null=None):
    args = [FAKE] * 6
    if null is not None:
        args[null] = None
    return lib.dspark_draft_markov(*args, B, G, V, r, dtype, ws, ws_bytes, FAKE, FAKE, FAKE, FAKE, None)


def test_draft_argument_checks(lib):
    assert _draft(lib, B=0) == 1
    assert _draft(lib, G=0) == 1
    assert _draft(lib, G=17) == 1
    assert _draft(lib, V=1) == 1
    assert _draft(lib, r=24, dtype=1) == 1
    assert _draft(lib, dtype=7) == 2
    for k in range(6):
        assert _draft(lib, null=k) == 1
    assert _draft(lib, ws=None) == 3
    assert _draft(lib, ws=ctypes.c_void_p(0x200010)) == 3          # misaligned
    assert _draft(lib, ws_bytes=16) == 3                           # too small


def test_bf16_arrays_must_be_16_byte_aligned(lib):
    """bf16 rows are moved by TMA and 16-byte vector loads: a bf16 array that
    does not start on a 16-byte boundary is refused on the host."""
    odd = ctypes.c_void_p(0x200008)
    for k in range(3):   # L, U, Wt
        args = [FAKE] * 6
        args[k] = odd
        assert lib.dspark_draft_markov(*args, 4, 5, 1024, 16, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, FAKE,
                                       None) == 1
        assert lib.dspark_draft_markov_noalloc(*args, 4, 5, 1024, 16, 1, FAKE, FAKE, FAKE, FAKE, None) == 1
    f = lib.dspark_verify
    for k in range(4):   # Tlog, L, U, Wt
        args = [FAKE] * 13
        args[k] = odd
        assert f(*args, 4, 5, 1024, 16, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, None, None) == 1
    # fp32 arrays have no such rule (the CUDA-core paths check alignment themselves).
    args = [odd] + [FAKE] * 5
    assert lib.dspark_draft_markov(*args, 4, 5, 1024, 16, 0, FAKE_WS, 16, FAKE, FAKE, FAKE, FAKE, None) == 3


def test_schedule_and_confidence_checks(lib):
    f = lib.dspark_schedule
    assert f(FAKE, 4, 5, FAKE, FAKE, 0, -1, 1, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE, None, None) == 1  # P = 0
    assert f(FAKE, 4, 5, FAKE, FAKE, 65, -1, 1, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 4, 5, FAKE, FAKE, 2, -1, 9, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE, None, None) == 1  # mode
    assert f(FAKE, 4096, 8, FAKE, FAKE, 2, -1, 1, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE, None, None) == 1
    assert f(FAKE, 4, 5, FAKE, FAKE, 2, -1, 1, None, 1 << 20, FAKE, FAKE, FAKE, None, None) == 3
    assert f(FAKE, 4, 5, FAKE, FAKE, 2, -1, 3, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE, None, None) == 1  # threshold mode
    assert f(FAKE, 4, 5, FAKE, FAKE, 2, -1, 4, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE, None, None) == 1
    h = lib.dspark_schedule_threshold
    assert h(FAKE, 0, 5, ctypes.c_float(0.5), -1, FAKE_WS, 1 << 20, FAKE, FAKE, None, None) == 1    # B = 0
    assert h(FAKE, 4096, 8, ctypes.c_float(0.5), -1, FAKE_WS, 1 << 20, FAKE, FAKE, None, None) == 1  # B*G
    assert h(FAKE, 4, 5, ctypes.c_float(float("nan")), -1, FAKE_WS, 1 << 20, FAKE, FAKE, None, None) == 1
    assert h(None, 4, 5, ctypes.c_float(0.5), -1, FAKE_WS, 1 << 20, FAKE, FAKE, None, None) == 1
    assert h(FAKE, 4, 5, ctypes.c_float(0.5), -1, None, 1 << 20, FAKE, FAKE, None, None) == 3
    g = lib.dspark_confidence
    assert g(FAKE, FAKE, ctypes.c_float(0), None, 4, 5, 0, 0, FAKE, FAKE, None) == 1   # d = 0
    assert g(FAKE, FAKE, ctypes.c_float(0), None, 4, 5, 8, 3, FAKE, FAKE, None) == 2   # dtype
    assert g(None, FAKE, ctypes.c_float(0), None, 4, 5, 8, 0, FAKE, FAKE, None) == 1


def test_verify_argument_checks(lib):
    f = lib.dspark_verify
    ok = [FAKE] * 13
    assert f(*ok, 4, 5, 1024, 16, 0, None, 1 << 30, FAKE, FAKE, FAKE, None, None) == 3
    bad = list(ok)
    bad[12] = None
    assert f(*bad, 4, 5, 1024, 16, 0, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, None, None) == 1
    assert f(*ok, 4, 5, 1024, 16, 0, FAKE_WS, 1 << 30, None, FAKE, FAKE, None, None) == 1


def test_injected_failure(lib, monkeypatch):
    """Host-side fault injection: the named entry point returns the given
    status without enqueuing any work."""
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_draft_markov=4")
    assert _draft(lib) == 4
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_schedule=5")
    assert lib.dspark_schedule(FAKE, 4, 5, FAKE, FAKE, 2, -1, 1, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE, None,
                               None) == 5
    with pytest.raises(_lib.DsparkError) as ei:
        _lib._call("dspark_schedule", FAKE, 4, 5, FAKE, FAKE, 2, -1, 1, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE,
                   None, None)
    assert ei.value.status == 5


def test_calibration_argument_checks(lib):
    assert lib.dspark_sts_workspace_size(16384, 5, 65, 15) > 0
    assert lib.dspark_sts_workspace_size(0, 5, 65, 15) == 0
    assert lib.dspark_sts_workspace_size(16, 17, 65, 15) == 0
    assert lib.dspark_sts_workspace_size(16, 5, 4097, 15) == 0
    assert lib.dspark_sts_workspace_size(16, 5, 65, 33) == 0
    assert lib.dspark_sts_workspace_size(16, 5, 65, 0) == 0

    def fit(N=64, G=5, K=9, M=15, ws=FAKE_WS, ws_bytes=1 << 20, null=None):
        args = [FAKE, FAKE, FAKE]
        if null is not None and null < 3:
            args[null] = None
        return lib.dspark_sts_fit(*args, N, G, K, M, ws, ws_bytes, FAKE if null != 3 else None, None, None, None,
                                  None, None)

    assert fit(N=0) == 1 and fit(G=0) == 1 and fit(G=17) == 1 and fit(K=0) == 1 and fit(M=33) == 1
    for k in range(4):
        assert fit(null=k) == 1
    assert fit(ws=None) == 3
    assert fit(ws=ctypes.c_void_p(0x200010)) == 3
    assert fit(ws_bytes=256) == 3
    assert lib.dspark_survival_auc(FAKE, FAKE, 0, 5, FAKE, FAKE, None) == 1
    assert lib.dspark_survival_auc(FAKE, FAKE, 16, 17, FAKE, FAKE, None) == 1
    assert lib.dspark_survival_auc(None, FAKE, 16, 5, FAKE, FAKE, None) == 1
    assert lib.dspark_survival_auc(FAKE, FAKE, 16, 5, None, FAKE, None) == 1


def test_schedule_topk_argument_checks(lib):
    def topk(B=8, G=5, cap=FAKE, ws=FAKE_WS, ws_bytes=1 << 20, S=FAKE, ell=FAKE, nadm=FAKE):
        return lib.dspark_schedule_topk(S, B, G, cap, -1, ws, ws_bytes, ell, nadm, None, None)

    assert topk(B=0) == 1 and topk(G=17) == 1 and topk(B=4096, G=8) == 1
    assert topk(cap=None) == 1 and topk(S=None) == 1 and topk(ell=None) == 1 and topk(nadm=None) == 1
    assert topk(ws=None) == 3 and topk(ws=ctypes.c_void_p(0x200010)) == 3 and topk(ws_bytes=8) == 3
    # mode 4 needs its capacity: the plain scheduler entry rejects it.
    assert lib.dspark_schedule(FAKE, 8, 5, FAKE, FAKE, 2, -1, 4, FAKE_WS, 1 << 20, FAKE, FAKE, FAKE, None,
                               None) == 1



def test_injected_failure_on_variant_entries(lib, monkeypatch):
    """The calibration and top-K entry points honour host-side injection too
    (they fail before touching any pointer)."""
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_sts_fit=4")
    assert lib.dspark_sts_fit(FAKE, FAKE, FAKE, 64, 5, 9, 15, FAKE_WS, 1 << 20, FAKE, None, None, None, None,
                              None) == 4
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_survival_auc=5")
    assert lib.dspark_survival_auc(FAKE, FAKE, 64, 5, FAKE, FAKE, None) == 5
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_schedule_topk=4")
    assert lib.dspark_schedule_topk(FAKE, 8, 5, FAKE, -1, FAKE_WS, 1 << 20, FAKE, FAKE, None, None) == 4


def test_injected_failure_on_verify_and_noalloc(lib, monkeypatch):
    """Verification, allocation-free drafting and its status getter honour
    host-side injection too (they fail before touching any pointer)."""
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_verify=4")
    assert lib.dspark_verify(*([FAKE] * 13), 4, 5, 1024, 16, 0, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, None,
                             None) == 4
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_draft_markov_noalloc=5")
    assert lib.dspark_draft_markov_noalloc(*([FAKE] * 6), 4, 5, 1024, 16, 0, FAKE, FAKE, FAKE, FAKE, None) == 5
    # An injection names one entry point only.
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_draft_markov=5")
    assert lib.dspark_draft_markov_noalloc(*([FAKE] * 6), 0, 5, 1024, 16, 0, FAKE, FAKE, FAKE, FAKE, None) == 1


def test_noalloc_argument_checks(lib):
    """The allocation-free entry point applies the same host checks as the
    workspace one."""
    f = lib.dspark_draft_markov_noalloc
    assert f(*([FAKE] * 6), 0, 5, 1024, 16, 0, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(*([FAKE] * 6), 4, 17, 1024, 16, 0, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(*([FAKE] * 6), 4, 5, 1024, 24, 1, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(*([FAKE] * 6), 4, 5, 1024, 16, 7, FAKE, FAKE, FAKE, FAKE, None) == 2
    for k in range(6):
        args = [FAKE] * 6
        args[k] = None
        assert f(*args, 4, 5, 1024, 16, 0, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert lib.dspark_draft_noalloc_device_status(None, None) == 1


def test_rnn_entry_point_checks(lib, monkeypatch):
    """The RNN head's entry points: bf16 only, r <= 256, every pointer
    present, 16-byte aligned bf16 arrays and states, a large enough
    workspace; host-side injection."""
    d = lib.dspark_draft_rnn
    v = lib.dspark_verify_rnn
    ok7 = [FAKE] * 7
    assert d(*ok7, 4, 5, 1024, 16, 0, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 2   # fp32
    assert d(*ok7, 4, 5, 1024, 272, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1  # r > 256
    assert d(*ok7, 4, 5, 1024, 16, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, FAKE, None, None) == 1   # no H_out
    assert d(*ok7, 4, 5, 1024, 16, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, FAKE, ctypes.c_void_p(0x200008),
             None) == 1                                                                            # misaligned H
    assert d(*ok7, 4, 5, 1024, 16, 1, FAKE_WS, 16, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 3        # workspace
    for k in range(7):
        args = list(ok7)
        args[k] = None
        assert d(*args, 4, 5, 1024, 16, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    ok12 = [FAKE] * 12
    assert v(*ok12, 4, 5, 1024, 16, 0, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, None, None) == 2
    assert v(*ok12, 4, 5, 1024, 272, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, None, None) == 1
    bad = list(ok12)
    bad[2] = None   # the states
    assert v(*bad, 4, 5, 1024, 16, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, None, None) == 1
    assert v(*ok12, 4, 5, 1024, 16, 1, None, 1 << 30, FAKE, FAKE, FAKE, None, None) == 3
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_draft_rnn=4")
    assert d(*ok7, 4, 5, 1024, 16, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 4
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_verify_rnn=5")
    assert v(*ok12, 4, 5, 1024, 16, 1, FAKE_WS, 1 << 30, FAKE, FAKE, FAKE, None, None) == 5


def test_gather_admitted_targets_checks(lib, monkeypatch):
    """The admitted target rows from host memory: the host checks reject an
    unknown dtype, bad sizes and a null pointer before any CUDA call (the
    pointer checks that follow need a GPU); host-side injection."""
    f = lib.dspark_gather_admitted_targets
    assert f(FAKE, FAKE, FAKE, 4, 5, 1024, 7, None) == 2
    assert f(FAKE, FAKE, FAKE, 0, 5, 1024, 1, None) == 1
    assert f(FAKE, FAKE, FAKE, 4097, 5, 1024, 1, None) == 1
    assert f(FAKE, FAKE, FAKE, 4, 0, 1024, 1, None) == 1
    assert f(FAKE, FAKE, FAKE, 4, 17, 1024, 1, None) == 1
    assert f(FAKE, FAKE, FAKE, 4, 5, 0, 1, None) == 1
    assert f(FAKE, FAKE, FAKE, 4, 5, (1 << 24) + 1, 1, None) == 1
    for k in range(3):
        args = [FAKE, FAKE, FAKE]
        args[k] = None
        assert f(*args, 4, 5, 1024, 1, None) == 1
    monkeypatch.setenv("DSPARK_INJECT_ERROR", "dspark_gather_admitted_targets=4")
    assert f(FAKE, FAKE, FAKE, 4, 5, 1024, 1, None) == 4
