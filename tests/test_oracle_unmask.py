"""Pins for the float64 unmasking oracle.

* hand-enumerated commit sets on vocabularies of at most 8 tokens
  (tests/golden/unmask_small.json, derivations in the file);
* closed forms: V equal logits give conf = 1/V and token 0; one spike s over
  zeros gives conf = e^s / (e^s + V - 1), so the commit flips at
  s* = ln(gamma (V - 1) / (1 - gamma));
* library routines: scipy.special.softmax for the top probability, NumPy
  argmax (first occurrence) for the token;
* invariants: adding a constant to a row changes neither token nor confidence;
  unmasked rows are never committed.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle.unmask import confidence_unmask, top2_gap

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "unmask_small.json")


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_enumerated_cases(case):
    logits = np.asarray(case["logits"], dtype=np.float32)
    res = confidence_unmask(logits, np.asarray(case["mask"]), case["gamma"],
                            block_S=case["block_S"] or None,
                            commit_at_least_one=case["commit_at_least_one"])
    assert res["tokens"].tolist() == case["tokens"]
    assert res["commit"].astype(int).tolist() == case["commit"]
    if "fallback" in case:
        assert res["fallback"].astype(int).tolist() == case["fallback"]
    m = np.asarray(case["mask"]).astype(bool)
    assert (res["mask_out"] == (m & ~res["commit"])).all()


@pytest.mark.parametrize("V", [1, 2, 7, 1024, 131072])
def test_equal_logits_closed_form(V):
    x = np.full((2, V), 0.75, dtype=np.float32)
    res = confidence_unmask(x, np.ones(2), 0.9)
    assert res["tokens"].tolist() == [0, 0]
    np.testing.assert_allclose(res["conf"], 1.0 / V, rtol=1e-14)
    assert res["commit"].tolist() == ([True, True] if V == 1 else [False, False])


@pytest.mark.parametrize("V,gamma", [(8, 0.9), (1024, 0.9), (131072, 0.95)])
def test_single_spike_closed_form(V, gamma):
    thr = math.log(gamma * (V - 1) / (1 - gamma))
    spikes = np.array([thr - 0.5, thr - 0.01, thr + 0.01, thr + 0.5, 0.3], dtype=np.float32)
    x = np.zeros((len(spikes), V), dtype=np.float32)
    pos = [V - 1, 3 % V, 0, V // 2, 5 % V]
    for r, (s, p) in enumerate(zip(spikes, pos)):
        x[r, p] = s
    res = confidence_unmask(x, np.ones(len(spikes)), gamma)
    for r, (s, p) in enumerate(zip(spikes.astype(np.float64), pos)):
        expect = math.exp(s) / (math.exp(s) + V - 1)
        assert abs(res["conf"][r] - expect) < 1e-13
        assert res["tokens"][r] == p
        assert res["commit"][r] == (s > thr)


def test_matches_library_softmax_and_argmax():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 4096)) * math.sqrt(2)).astype(np.float32)
    x[np.arange(64), rng.integers(0, 4096, 64)] += rng.uniform(0, 16, 64).astype(np.float32)
    mask = rng.integers(0, 2, 64)
    res = confidence_unmask(x, mask, 0.9)
    p = scipy.special.softmax(x.astype(np.float64), axis=1)
    m = mask.astype(bool)
    np.testing.assert_allclose(res["conf"][m], p.max(axis=1)[m], rtol=1e-12)
    assert (res["tokens"][m] == np.argmax(x, axis=1)[m]).all()
    assert (res["tokens"][~m] == -1).all() and not res["commit"][~m].any()
    assert (res["commit"] == (m & (p.max(axis=1) > np.float32(0.9)))).all()


def test_shift_invariance():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((16, 500)).astype(np.float32)
    a = confidence_unmask(x, np.ones(16), 0.5)
    b = confidence_unmask(x.astype(np.float64) + 1000.0, np.ones(16), 0.5)
    assert (a["tokens"] == b["tokens"]).all()
    np.testing.assert_allclose(a["conf"], b["conf"], rtol=1e-12)


def test_threshold_is_float32_gamma():
    # conf exactly 0.5 against gamma = 0.5: equal in every precision, no commit
    r = confidence_unmask(np.zeros((1, 2), np.float32), [1], 0.5)
    assert not r["commit"][0]


def test_fallback_commits_one_per_unfinished_block():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((64, 256)).astype(np.float32)  # nothing reaches 0.9
    mask = np.ones(64)
    mask[16:32] = 0  # block 1 already finished
    res = confidence_unmask(x, mask, 0.9, block_S=16, commit_at_least_one=True)
    per_block = res["commit"].reshape(4, 16).sum(1).tolist()
    assert per_block == [1, 0, 1, 1]
    for blk in (0, 2, 3):
        sl = slice(16 * blk, 16 * blk + 16)
        assert np.argmax(res["commit"][sl]) == np.nanargmax(res["conf"][sl])


def test_top2_gap():
    x = np.array([[1, 3, 3, 0], [0, 5, 1, 2]], dtype=np.float32)
    np.testing.assert_array_equal(top2_gap(x), [0.0, 3.0])


def test_top2_gap_single_token_vocabulary():
    assert np.isinf(top2_gap(np.zeros((3, 1), np.float32))).all()
