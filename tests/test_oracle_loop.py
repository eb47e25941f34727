"""Pins for the block refinement loop oracle (Algorithm 1's inner loop).

Invariants the pages fix ("Technical summary: Nemotron-TwoTower",
§Methodology > Generation process, and §Training and conditioning >
Sampling): committed tokens stay committed, the masked set only shrinks, and
with the one-commit-per-step fallback a block of S positions finishes within
S steps. A two-position case is enumerated by hand.
"""

import numpy as np

from oracle.loop import block_loop


def test_invariants_random_logits():
    rng = np.random.default_rng(1)
    B, S, V, T = 8, 16, 512, 16
    cache = {}

    def step_logits(t):
        if t not in cache:
            x = rng.standard_normal((B * S, V)).astype(np.float32)
            x[np.arange(B * S), rng.integers(0, V, B * S)] += rng.uniform(0, 12, B * S).astype(np.float32)
            cache[t] = x
        return cache[t]

    res = block_loop(step_logits, np.ones(B * S), 0.9, S, T, commit_at_least_one=True)
    assert not res["mask"].any()
    assert sum(res["per_step"]) == B * S
    assert (res["commit_step"] >= 0).all() and (res["tokens"] >= 0).all()
    # every unfinished block commits at least one position per step
    cs = res["commit_step"].reshape(B, S)
    for b in range(B):
        last = cs[b].max()
        for t in range(last + 1):
            assert (cs[b] == t).sum() >= 1
    # a committed token is the argmax of the logits at its commit step
    for r in range(B * S):
        assert res["tokens"][r] == int(np.argmax(cache[int(res["commit_step"][r])][r]))


def test_hand_enumerated_two_positions():
    # step 0: row 0 conf = e^8/(e^8+1) > 0.9 commits (token 0); row 1 conf 0.5 stays
    # step 1: row 1 conf = 1/2 again, nothing passes -> fallback commits row 1 (token 0)
    x0 = np.array([[8, 0], [0, 0]], dtype=np.float32)
    x1 = np.array([[0, 9], [0, 0]], dtype=np.float32)  # row 0 is no longer read
    res = block_loop(lambda t: [x0, x1][t], np.ones(2), 0.9, 2, 5, commit_at_least_one=True)
    assert res["tokens"].tolist() == [0, 0]
    assert res["commit_step"].tolist() == [0, 1]
    assert res["per_step"] == [1, 1] and res["steps"] == 2


def test_without_fallback_may_stop_with_masked_rows():
    x = np.zeros((4, 8), dtype=np.float32)  # conf 1/8 everywhere
    res = block_loop(lambda t: x, np.ones(4), 0.9, 4, 3, commit_at_least_one=False)
    assert res["steps"] == 3 and res["mask"].all() and res["per_step"] == [0, 0, 0]
