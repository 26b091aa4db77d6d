"""Drafting through the entry point that allocates nothing.

Callers such as an inference engine's plugin (handed only inputs and outputs
at enqueue time, with all memory planned ahead) or a latency-critical serving
loop (which must not call cudaMalloc, as it can synchronise the device) use
dspark_draft_markov_noalloc instead of dspark_draft_markov.  It keeps its
scratch in a fixed device array inside the library.  This file runs last so
that a failure here leaves every other test already run; it passes alone in a
fresh process and after the rest.
"""
import numpy as np
import pytest
import torch

from speculative_decoding_draft_rank_b200 import _lib, synth

pytestmark = pytest.mark.gpu

ATOL = 1e-5  # the parity tolerance the other GPU tests use for probabilities


def _device_inputs(inp):
    dev = torch.device("cuda")
    if inp.dtype == "bf16":
        cvt = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        L, U, Wt = cvt(inp.bits["L"]), cvt(inp.bits["U"]), cvt(np.ascontiguousarray(inp.bits["W"].T))
    else:
        cvt = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)
        L, U, Wt = cvt(inp.L), cvt(inp.U), cvt(np.ascontiguousarray(inp.W.T))
    small = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return L, U, Wt, small(inp.x0), small(inp.temp), small(inp.u_draft)


def _outputs(B, G):
    dev = torch.device("cuda")
    return (torch.full((B, G), -7, dtype=torch.int32, device=dev),
            *(torch.full((B, G), -7.0, dtype=torch.float32, device=dev) for _ in range(3)))


@pytest.mark.parametrize("dtype,B,G,V,r", [("bf16", 256, 5, 12000, 256), ("bf16", 37, 3, 5008, 80),
                                           ("f32", 9, 4, 3001, 16), ("bf16", 256, 5, 129280, 256)])
def test_noalloc_matches_workspace_entry_point(dtype, B, G, V, r):
    temps = np.tile(np.float32([1.0, 0.0, 0.7, 1.3]), B)[:B]
    inp = synth.generate(B, G, V, r, 8, dtype, seed=B + V, hot=8, temps=temps)
    L, U, Wt, x0, temp, ud = _device_inputs(inp)
    code = _lib.DSPARK_BF16 if dtype == "bf16" else _lib.DSPARK_F32
    ws = torch.zeros(_lib.dspark_draft_workspace_size(B, G, V, r, code) + 256, dtype=torch.uint8,
                     device="cuda")
    ref = _outputs(B, G)
    _lib.dspark_draft_markov(L, U, Wt, x0, temp, ud, ws, *ref)
    for call in range(2):  # two calls in a row share (and reuse) the library's scratch
        got = _outputs(B, G)
        _lib.dspark_draft_markov_noalloc(L, U, Wt, x0, temp, ud, *got)
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref[0]), f"call {call}: draft tokens differ"
        for name, g, w in zip(("p_d(x)", "row max", "Z"), got[1:], ref[1:]):
            assert torch.allclose(g, w, atol=ATOL, rtol=0), f"call {call}: {name} differs"
    assert _lib.dspark_get_device_status(ws) == 0
    assert _lib.dspark_draft_noalloc_device_status() == 0


def test_noalloc_rejects_rounds_beyond_its_scratch():
    cap = _lib.dspark_draft_noalloc_max_scratch()
    B, G, V, r = 4096, 4, 1 << 20, 512
    assert _lib.dspark_draft_workspace_size(B, G, V, r, _lib.DSPARK_BF16) > cap
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(16, dtype=torch.int32, device="cuda")
    f = torch.zeros(16, dtype=torch.float32, device="cuda")
    st = _lib.load().dspark_draft_markov_noalloc(
        _lib._ptr(dummy), _lib._ptr(dummy), _lib._ptr(dummy), _lib._ptr(idx), _lib._ptr(f), _lib._ptr(f), B, G, V,
        r, _lib.DSPARK_BF16, _lib._ptr(idx), _lib._ptr(f), _lib._ptr(f), _lib._ptr(f), None)
    assert st == 3  # DSPARK_ERR_WORKSPACE, before any work is enqueued


def test_noalloc_reports_a_wait_that_ran_out(monkeypatch):
    """A bounded wait that runs out inside the allocation-free call is
    reported through its status getter, and the next call (which clears the
    word) succeeds with the normal budget."""
    B, G, V, r = 130, 3, 4104, 64
    inp = synth.generate(B, G, V, r, 8, "bf16", seed=3, hot=8)
    L, U, Wt, x0, temp, ud = _device_inputs(inp)
    ws = torch.zeros(_lib.dspark_draft_workspace_size(B, G, V, r, _lib.DSPARK_BF16), dtype=torch.uint8,
                     device="cuda")
    ref = _outputs(B, G)
    _lib.dspark_draft_markov(L, U, Wt, x0, temp, ud, ws, *ref)
    monkeypatch.setenv("DSPARK_WAIT_BUDGET_CYCLES", "200")
    got = _outputs(B, G)
    _lib.dspark_draft_markov_noalloc(L, U, Wt, x0, temp, ud, *got)
    assert _lib.dspark_draft_noalloc_device_status() & _lib.DEV_TIMEOUT
    monkeypatch.delenv("DSPARK_WAIT_BUDGET_CYCLES")
    _lib.dspark_draft_markov_noalloc(L, U, Wt, x0, temp, ud, *got)
    assert _lib.dspark_draft_noalloc_device_status() == 0
    assert torch.equal(got[0], ref[0])
