"""The FMA-pipe polynomial 2^x that the verification row pass uses for one
exponential in four (dspark_exp2_fma), against fp64 2^x: relative error
within 4e-7 on [-125, 0] (about that of the special-function unit's ex2),
at the integers too, and clamped to 2^-125 (to the same accuracy) below -125."""
import numpy as np
import pytest
import torch

from speculative_decoding_draft_rank_b200 import _lib

pytestmark = pytest.mark.gpu


def _run(x: np.ndarray) -> np.ndarray:
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    yd = torch.empty_like(xd)
    _lib.dspark_exp2_fma(xd, yd)
    torch.cuda.synchronize()
    return yd.cpu().numpy()


def test_relative_error_on_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(-125.0, 0.0, 1 << 20), rng.uniform(-1.0, 0.0, 1 << 18),
                        -np.arange(0, 125, dtype=np.float64) - 0.5, np.array([0.0, -0.49999997, -0.5, -0.50000006])])
    x32 = x.astype(np.float32)
    y = _run(x32).astype(np.float64)
    ref = np.exp2(x32.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= 4e-7, (rel.max(), x32[np.argmax(rel)])


def test_integers_and_clamp():
    x = -np.arange(0, 126, dtype=np.float32)
    y = _run(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.abs(y - ref) <= 4e-7 * ref)
    low = _run(np.array([-126.0, -200.0, -1e30, -np.inf], np.float32)).astype(np.float64)
    assert np.all(np.abs(low - 2.0 ** -125) <= 4e-7 * 2.0 ** -125)


def test_odd_length():
    x = np.linspace(-3.0, 0.0, 7, dtype=np.float32)
    y = _run(x)
    assert np.allclose(y, np.exp2(x.astype(np.float64)), rtol=4e-7, atol=0)
