"""Pins of the oracle's RNN draft head (paperlayer.ai summary of DSpark, §3.1
Semi-autoregressive generation: the RNN head keeps a recurrent state that
summarises the whole prefix of the block; menfem.com KB entry, "Key
Contributions": an RNN head with the full within-block history beside the
Markov head).  The pages give no equations; the oracle's reading is
h_k = tanh(h_{k-1} A + U[x_{k-1}]), h_0 = 0, bias h_k W.  What the pages and
the mathematics fix about it, and what these tests hold it to:

* with A = 0 the state is tanh(U[x_{k-1}]): the head is the Markov head with
  the factor tanh(U) (pinned against the Markov oracle, itself pinned);
* the bias depends on the whole prefix, not only on the previous token;
* verification with the RNN head keeps the target law exactly (the exact
  enumeration of every uniform's outcomes), which needs drafting and
  verification to agree on p_d.
The orientation of A (h A rather than A h) is a convention the pages do not
fix; the GPU path is held to the oracle's."""
import numpy as np
import pytest

import enum_harness as eh
from oracle import oracle
from speculative_decoding_draft_rank_b200 import synth


def _tiny(seed, B, G, V, r):
    rng = np.random.default_rng(seed)
    L = rng.normal(0, 1.5, (B, G, V)).astype(np.float32)
    U = rng.uniform(-0.9, 0.9, (V, r)).astype(np.float32)
    W = rng.normal(0, 1.0, (r, V)).astype(np.float32)
    x0 = rng.integers(0, V, B).astype(np.int32)
    u = rng.random((B, G))
    return rng, L, U, W, x0, u


@pytest.mark.parametrize("T", [1.0, 0.7, 0.0])
def test_zero_recurrence_is_the_markov_head_with_tanh_factor(T):
    rng, L, U, W, x0, u = _tiny(1, 6, 4, 40, 8)
    temp = np.full(6, T, np.float32)
    A0 = np.zeros((8, 8), np.float32)
    rnn = oracle.draft(L, U, W, x0, temp, u, A=A0)
    Um = np.tanh(U.astype(np.float64)).astype(np.float32)
    mk = oracle.draft(L, Um, W, x0, temp, u, force_x=rnn.x)   # follow the RNN's tokens
    # tanh(U) rounded to fp32 moves the bias by ~1e-7: decisions agree
    # unless their margin is that small.
    sure = rnn.margin > 1e-5
    mk_free = oracle.draft(L, Um, W, x0, temp, u)
    assert np.array_equal(rnn.x[sure.all(axis=1)], mk_free.x[sure.all(axis=1)])
    np.testing.assert_allclose(rnn.pd, mk.pd, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(rnn.rowmax, mk.rowmax, rtol=0, atol=1e-5)
    # Verification too.
    ell = np.full(6, 4, np.int32)
    ua, uf = rng.random((6, 4)), rng.random(6)
    T1 = rng.normal(0, 1.5, (6, 5, 40)).astype(np.float32)
    vr = oracle.verify(T1, L, U, W, x0, rnn.x, temp, ua, uf, ell, A=A0)
    vm = oracle.verify(T1, L, Um, W, x0, rnn.x, temp, ua, uf, ell, force_accept=None)
    ok = (vr.margin_acc > 1e-5).all(axis=1) & (vr.margin_fin > 1e-5)
    assert np.array_equal(vr.tokens[ok], vm.tokens[ok])
    np.testing.assert_allclose(np.nan_to_num(vr.pd_x), np.nan_to_num(vm.pd_x), rtol=1e-5, atol=1e-7)


def test_bias_depends_on_the_whole_prefix():
    # Two requests that differ only in x_0, both forced to the same x_1, x_2:
    # the Markov head's position-3 distribution depends on x_2 alone, the RNN
    # head's on the whole prefix.
    rng, L, U, W, x0, u = _tiny(2, 2, 3, 16, 4)
    L[1] = L[0]
    x0 = np.array([3, 11], np.int32)
    force = np.array([[5, 7, -1], [5, 7, -1]], np.int32)
    temp = np.ones(2, np.float32)
    A = synth.rnn_matrix(4, seed=3, gain=0.9)
    mk = oracle.draft(L, U, W, x0, temp, u, force_x=force)
    rn = oracle.draft(L, U, W, x0, temp, u, force_x=force, A=A)
    assert mk.rowmax[0, 2] == mk.rowmax[1, 2] and mk.rowsum[0, 2] == mk.rowsum[1, 2]
    assert abs(rn.rowmax[0, 2] - rn.rowmax[1, 2]) > 1e-6 or abs(rn.rowsum[0, 2] - rn.rowsum[1, 2]) > 1e-6
    # Position 1 sees only x_0 in both heads; the state there is tanh(U[x_0]).
    assert rn.rowmax[0, 0] != rn.rowmax[1, 0]


@pytest.mark.parametrize("seed,V,G,r,T", [(0, 3, 3, 2, 1.0), (1, 4, 2, 3, float(np.float32(0.7))),
                                          (2, 5, 2, 2, float(np.float32(1.4)))])
def test_rnn_head_keeps_the_target_law(seed, V, G, r, T):
    rng = np.random.default_rng(300 + seed)
    Lrows = rng.normal(0, 1.5, (G, V)).astype(np.float32)
    U = rng.normal(0, 1.0, (V, r)).astype(np.float32)
    W = rng.normal(0, 1.0, (r, V)).astype(np.float32)
    A = rng.normal(0, 1.0, (r, r)).astype(np.float32)
    target = eh.random_target(rng, V, G)
    for ell in range(G + 1):
        sc = eh.Scenario(Lrows, U, W, int(rng.integers(0, V)), T, target, ell_fixed=ell, A=A)
        law = sc.output_law()
        assert eh.preservation_error(law, target, T, V) < 1e-12


def test_rnn_and_markov_drafts_differ_when_the_state_carries():
    # A sanity check that the recurrence is live: the same inputs with A != 0
    # give a different bias than with A = 0 from position 2 on, never at
    # position 1 (h_1 = tanh(U[x_0]) for every A).
    rng, L, U, W, x0, u = _tiny(4, 5, 4, 30, 6)
    temp = np.ones(5, np.float32)
    A = synth.rnn_matrix(6, seed=9)
    a = oracle.draft(L, U, W, x0, temp, u, A=np.zeros((6, 6), np.float32))
    b = oracle.draft(L, U, W, x0, temp, u, A=A, force_x=a.x)
    assert np.array_equal(a.rowmax[:, 0], b.rowmax[:, 0]) and np.array_equal(a.rowsum[:, 0], b.rowsum[:, 0])
    assert np.all(np.abs(a.rowmax[:, 1:] - b.rowmax[:, 1:]) > 0)


def test_states_with_zero_recurrence_are_tanh_of_the_factor_rows():
    # A = 0: h_k = tanh(U[x_{k-1}]) exactly as numpy's tanh gives it.
    rng, L, U, W, x0, u = _tiny(5, 4, 3, 20, 6)
    x = rng.integers(0, 20, (4, 3)).astype(np.int32)
    h = oracle.rnn_states(U, np.zeros((6, 6), np.float32), x0, x)
    prev = np.concatenate([x0[:, None], x[:, :-1]], axis=1)
    np.testing.assert_allclose(h, np.tanh(U.astype(np.float64)[prev]), rtol=0, atol=1e-15)


def test_states_match_the_drafting_bias():
    # The state the drafting stage used is the one rnn_states reports: with
    # W = identity (V = r) and L = 0, row max and log Z of a greedy row are
    # max_c h_k[c] and 0.
    rng = np.random.default_rng(6)
    r = 5
    U = rng.uniform(-1, 1, (r, r)).astype(np.float32)
    W = np.eye(r, dtype=np.float32)
    A = synth.rnn_matrix(r, seed=7)
    L = np.zeros((3, 4, r), np.float32)
    x0 = np.array([0, 2, 4], np.int32)
    d = oracle.draft(L, U, W, x0, np.zeros(3, np.float32), rng.random((3, 4)), A=A)
    h = oracle.rnn_states(U, A, x0, d.x)
    np.testing.assert_allclose(d.rowmax, h.max(axis=2), rtol=0, atol=1e-15)
    assert np.array_equal(d.x, h.argmax(axis=2))


def test_rnn_states_refuse_tokens_outside_the_vocabulary():
    """The states entry indexes U by token: a token outside [0, V) (either
    the committed one or a drafted one) or an empty batch is an argument
    error, not an out-of-bounds read."""
    rng = np.random.default_rng(3)
    V, r, G = 6, 4, 3
    U = rng.normal(0, 1, (V, r)).astype(np.float32)
    A = np.zeros((r, r), np.float32)
    ok_x0, ok_x = np.array([1, 2], np.int32), np.array([[0, 5, 3], [1, 1, 1]], np.int32)
    oracle.rnn_states(U, A, ok_x0, ok_x)
    for x0, x in ((np.array([6, 2], np.int32), ok_x), (np.array([-1, 2], np.int32), ok_x),
                  (ok_x0, np.array([[0, 6, 3], [1, 1, 1]], np.int32)),
                  (ok_x0, np.array([[0, 1, 3], [-2, 1, 1]], np.int32))):
        with pytest.raises(ValueError):
            oracle.rnn_states(U, A, x0, x)
    with pytest.raises(ValueError):
        oracle.rnn_states(U, A, np.zeros(0, np.int32), np.zeros((0, G), np.int32))
