"""Pins of the LM-head + unmask oracle.

The projection is pinned by a pure-Python triple loop on tiny inputs and by
closed forms (an identity head returns the hidden states; a head whose row v*
is a multiple of the hidden state gives that token the logit alpha * |h|^2);
the composition with Algorithm 2 by a hand-derived case and by the
single-spike commit threshold of the unmask pins.
"""

import math

import numpy as np

from oracle.lmhead import lmhead_logits, lmhead_unmask

RNG = np.random.default_rng(11)


def test_projection_matches_triple_loop():
    h = RNG.standard_normal((3, 5))
    W = RNG.standard_normal((7, 5))
    ref = [[sum(h[r][k] * W[v][k] for k in range(5)) for v in range(7)] for r in range(3)]
    np.testing.assert_allclose(lmhead_logits(h, W), np.array(ref), rtol=0, atol=1e-13)


def test_identity_head_returns_hidden_states():
    h = RNG.standard_normal((4, 6))
    np.testing.assert_array_equal(lmhead_logits(h, np.eye(6)), h)


def test_row_selection():
    h = RNG.standard_normal((5, 4))
    W = RNG.standard_normal((3, 4))
    np.testing.assert_array_equal(lmhead_logits(h, W, rows=[4, 1]), lmhead_logits(h, W)[[4, 1]])


def test_aligned_row_gets_alpha_norm_squared():
    h = RNG.standard_normal((1, 8))
    W = np.zeros((6, 8))
    W[4] = 0.5 * h[0]
    l = lmhead_logits(h, W)
    assert math.isclose(l[0, 4], 0.5 * float(h[0] @ h[0]), rel_tol=1e-15)
    assert (l[0, [0, 1, 2, 3, 5]] == 0).all()


def test_spike_commit_threshold_through_the_head():
    # V - 1 zero logits and one logit s: conf = e^s / (e^s + V - 1); commit iff
    # s > ln(gamma (V - 1) / (1 - gamma))
    V, gamma = 64, 0.9
    s_star = math.log(gamma * (V - 1) / (1 - np.float32(gamma)))
    for s, expect in ((s_star - 1e-3, False), (s_star + 1e-3, True)):
        h = np.array([[math.sqrt(s)]])
        W = np.zeros((V, 1))
        W[17, 0] = math.sqrt(s)
        res = lmhead_unmask(h, W, np.array([1]), gamma)
        assert res["tokens"][0] == 17
        assert bool(res["commit"][0]) == expect
        assert math.isclose(res["conf"][0], math.exp(s) / (math.exp(s) + V - 1), rel_tol=1e-12)


def test_unmasked_rows_are_not_predicted():
    h = RNG.standard_normal((4, 3))
    W = RNG.standard_normal((10, 3))
    res = lmhead_unmask(h, W, np.array([0, 1, 0, 1]), 0.5)
    assert res["tokens"][0] == -1 and res["tokens"][2] == -1
    assert not res["commit"][0] and not res["commit"][2]
    assert np.isnan(res["logits"][0]).all()
    assert res["tokens"][1] == int(np.argmax(h[1] @ W.T))


def test_hand_case_with_fallback():
    # two blocks of two rows; logits chosen so nothing passes gamma = 0.99 in
    # block 0 (the row of higher confidence commits by the fallback) and row 3
    # passes in block 1
    h = np.eye(4)
    W = np.array([[2.0, 0.0, 0.0, 0.0],
                  [0.0, 1.0, 0.0, 9.0],
                  [0.0, 0.0, 0.0, 0.0]])
    # logits rows: r0 = (2,0,0), r1 = (0,1,0), r2 = (0,0,0), r3 = (0,9,0)
    res = lmhead_unmask(h, W, np.ones(4), 0.99, block_S=2, commit_at_least_one=True)
    assert res["tokens"].tolist() == [0, 1, 0, 1]
    c0 = math.exp(2) / (math.exp(2) + 2)
    c1 = math.e / (math.e + 2)
    assert math.isclose(res["conf"][0], c0) and math.isclose(res["conf"][1], c1)
    assert res["commit"].tolist() == [True, False, False, True]
