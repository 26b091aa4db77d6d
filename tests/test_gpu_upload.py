"""Target rows from host memory (dspark_gather_admitted_targets) and the
round fed from host memory (DeviceRound.run_from_host).

The target forward yields rows only for the admitted positions, so a round
fed from the host copies rows 0..ell_b of each request and nothing else.
These tests check that the gather copies exactly those rows (the rest of the
device buffer keeps a NaN sentinel), that it refuses sources it cannot
address, and that a round whose device target buffer holds NaN everywhere
else gives the same results as the round on fully resident inputs:
verification reads no row past ell_b.
"""
import numpy as np
import pytest
import torch

from speculative_decoding_draft_rank_b200 import _lib, synth, workloads as wl
from speculative_decoding_draft_rank_b200.round import DeviceRound

pytestmark = pytest.mark.gpu


def _ell_patterns(B, G, rng):
    yield np.full(B, G, np.int32)                   # one run over the whole buffer
    yield np.zeros(B, np.int32)                     # the bonus rows only
    e = rng.integers(0, G + 1, B).astype(np.int32)
    e[: B // 3] = G                                 # a long run at the start
    e[-1] = G                                       # the last request ends the buffer
    yield e
    e = rng.integers(0, G + 1, B).astype(np.int32)
    e[::2] = G                                      # runs of two
    yield e


@pytest.mark.parametrize("dtype,B,G,V", [(torch.bfloat16, 37, 5, 1000), (torch.float32, 9, 3, 1288),
                                         (torch.bfloat16, 256, 8, 4104), (torch.bfloat16, 5, 2, 1001),
                                         (torch.float32, 3, 4, 1001)])
def test_gather_copies_exactly_the_admitted_rows(dtype, B, G, V):
    rng = np.random.default_rng(B * G + V)
    host = torch.from_numpy(rng.standard_normal((B, G + 1, V), dtype=np.float32)).to(dtype).pin_memory()
    dev = torch.empty((B, G + 1, V), dtype=dtype, device="cuda")
    for ell in _ell_patterns(B, G, rng):
        dev.fill_(float("nan"))
        # Out-of-range lengths are clamped to [0, G] on the device.
        e = ell.copy()
        e[0] = G + 3 if ell[0] == G else ell[0]
        e[-1] = -2 if ell[-1] == 0 else ell[-1]
        _lib.dspark_gather_admitted_targets(host, dev, torch.from_numpy(e).cuda())
        torch.cuda.synchronize()
        got = dev.cpu()
        keep = torch.arange(G + 1)[None, :] <= torch.from_numpy(ell)[:, None].long()   # [B, G+1]
        assert torch.equal(got[keep], host[keep])
        assert torch.isnan(got[~keep].float()).all()


def test_gather_refuses_pageable_or_device_sources():
    B, G, V = 4, 3, 64
    dev = torch.zeros((B, G + 1, V), dtype=torch.bfloat16, device="cuda")
    ell = torch.ones(B, dtype=torch.int32, device="cuda")
    pageable = torch.ones((B, G + 1, V), dtype=torch.bfloat16)
    f = _lib.load().dspark_gather_admitted_targets
    import ctypes
    assert f(ctypes.c_void_p(pageable.data_ptr()), ctypes.c_void_p(dev.data_ptr()),
             ctypes.c_void_p(ell.data_ptr()), B, G, V, _lib.DSPARK_BF16, None) == 1
    other = torch.ones_like(dev)
    assert f(ctypes.c_void_p(other.data_ptr()), ctypes.c_void_p(dev.data_ptr()),
             ctypes.c_void_p(ell.data_ptr()), B, G, V, _lib.DSPARK_BF16, None) == 1
    pinned = pageable.pin_memory()
    pinned_dst = torch.zeros_like(pinned).pin_memory()
    assert f(ctypes.c_void_p(pinned.data_ptr()), ctypes.c_void_p(pinned_dst.data_ptr()),
             ctypes.c_void_p(ell.data_ptr()), B, G, V, _lib.DSPARK_BF16, None) == 1
    torch.cuda.synchronize()
    assert int(dev.float().abs().sum()) == 0


@pytest.mark.parametrize("make", [wl.tiny, wl.headline, lambda: wl.long_block(8)])
def test_round_from_host_matches_resident_round(make):
    w = make()
    inp = w.inputs()
    ref = DeviceRound(inp, w.knots_n, w.knots_t, w.budget, w.mode)
    ref.run()
    torch.cuda.synchronize()
    want = ref.outputs()
    del ref
    dr = DeviceRound(inp, w.knots_n, w.knots_t, w.budget, w.mode, pinned_host=True)
    for k in DeviceRound.ROUND_INPUTS + ("Tlog",):
        dr.t[k].fill_(float("nan") if dr.t[k].is_floating_point() else 0)
    st = torch.cuda.Stream()
    dr.run_from_host(st)
    st.synchronize()
    h2d, d2h = dr.host_round_bytes()
    got = dr.outputs()
    for k in ("x", "ell", "acc", "tokens", "nout"):
        assert np.array_equal(got[k], want[k]), k
    for k in ("pd_x", "rowmax", "rowsum", "S", "pt_x"):
        assert np.array_equal(got[k], want[k]), k
    for k, v in dr.host_out.items():
        assert np.array_equal(v.numpy(), want[k]), k
    ell = want["ell"].astype(np.int64)
    elem = 2 if inp.dtype == "bf16" else 4
    small = sum(dr.host[k].numel() * dr.host[k].element_size() for k in DeviceRound.ROUND_INPUTS)
    assert h2d == small + int((ell + 1).sum()) * inp.V * elem
    assert d2h == sum(v.numel() * v.element_size() for v in dr.host_out.values())
    # The rows past ell_b were never copied: they still hold the sentinel.
    T = dr.t["Tlog"].float().cpu()
    keep = torch.arange(inp.G + 1)[None, :] <= torch.from_numpy(ell)[:, None]
    assert torch.isnan(T[~keep]).all()
    assert dr.device_status() == 0
