"""Pins of the self-speculative verification oracle.

Causal block attention: with no prefix it is torch's causal scaled-dot-product
attention in float64 (a library routine); the last block position sees every
block key, so it equals the bidirectional block attention there; S = 1 makes
the two modes equal; a pure-Python brute force on tiny inputs. Commit rule:
hand-enumerated blocks, and the lossless property - every committed token is
the autoregressive (argmax) token.
"""

import math

import numpy as np
import pytest

from oracle.attention import block_attention
from oracle.spec import causal_block_attention, verify_commit

RNG = np.random.default_rng(31)


def _inp(B=2, S=5, H_q=4, H_kv=2, d=8, lens=(3, 0)):
    q = RNG.standard_normal((B, S, H_q, d))
    kb, vb = RNG.standard_normal((B, S, H_kv, d)), RNG.standard_normal((B, S, H_kv, d))
    R = max(1, sum(lens))
    kp, vp = RNG.standard_normal((R, H_kv, d)), RNG.standard_normal((R, H_kv, d))
    off = np.concatenate([[0], np.cumsum(lens)[:-1]])
    return q, kp, vp, kb, vb, np.array(lens), off


def test_no_prefix_is_causal_sdpa():
    torch = pytest.importorskip("torch")
    q, kp, vp, kb, vb, L, off = _inp(lens=(0, 0))
    o, _ = causal_block_attention(q, kp, vp, kb, vb, L, off)
    g = q.shape[2] // kb.shape[2]
    Q = torch.tensor(q).permute(0, 2, 1, 3)
    K = torch.tensor(kb).repeat_interleave(g, dim=2).permute(0, 2, 1, 3)
    V = torch.tensor(vb).repeat_interleave(g, dim=2).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)


def test_last_position_equals_bidirectional():
    args = _inp()
    oc, lc = causal_block_attention(*args)
    ob, lb = block_attention(*args)
    np.testing.assert_allclose(oc[:, -1], ob[:, -1], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lc[:, :, -1], lb[:, :, -1], rtol=1e-13, atol=1e-13)
    assert not np.allclose(oc[:, 0], ob[:, 0])


def test_one_position_block_equals_bidirectional():
    args = _inp(S=1)
    oc, lc = causal_block_attention(*args)
    ob, lb = block_attention(*args)
    np.testing.assert_allclose(oc, ob, rtol=1e-13, atol=1e-13)


def test_brute_force():
    q, kp, vp, kb, vb, L, off = _inp(B=1, S=3, H_q=2, H_kv=1, d=2, lens=(2,))
    o, _ = causal_block_attention(q, kp, vp, kb, vb, L, off)
    for i in range(3):
        keys = [kp[0, 0], kp[1, 0]] + [kb[0, j, 0] for j in range(i + 1)]
        vals = [vp[0, 0], vp[1, 0]] + [vb[0, j, 0] for j in range(i + 1)]
        for h in range(2):
            s = [sum(q[0, i, h, k] * kk[k] for k in range(2)) / math.sqrt(2) for kk in keys]
            m = max(s)
            w = [math.exp(x - m) for x in s]
            ref = [sum(w[j] * vals[j][k] for j in range(len(w))) / sum(w) for k in range(2)]
            np.testing.assert_allclose(o[0, i, h], ref, rtol=1e-12)


def _logits_for(tokens, V=6):
    x = np.zeros((len(tokens), V))
    for r, t in enumerate(tokens):
        x[r, t] = 3.0
    return x


@pytest.mark.parametrize("ar,draft,n,commit", [
    ([1, 2, 3, 4], [1, 2, 3, 4], 4, [1, 1, 1, 1]),     # whole draft accepted
    ([1, 2, 3, 4], [0, 2, 3, 4], 0, [1, 0, 0, 0]),     # first token wrong: AR token at 0
    ([1, 2, 3, 4], [1, 2, 5, 4], 2, [1, 1, 1, 0]),     # match, match, mismatch (AR token), rest waits
    ([1, 2, 3, 4], [1, 2, 3, 0], 3, [1, 1, 1, 1]),     # mismatch at the last position
])
def test_commit_rule_hand_cases(ar, draft, n, commit):
    res = verify_commit(_logits_for(ar), np.array(draft), S=4)
    assert res["n_accept"].tolist() == [n]
    assert res["commit"].astype(int).tolist() == commit
    assert res["tokens"].tolist() == ar


def test_ties_take_the_lowest_id_and_blocks_are_independent():
    x = np.zeros((4, 5))
    x[0, [2, 4]] = 1.0     # tie: token 2
    x[1, 0] = 1.0
    x[2, 3] = 1.0
    x[3, 1] = 1.0
    res = verify_commit(x, np.array([2, 0, 3, 2]), S=2)
    assert res["tokens"].tolist() == [2, 0, 3, 1]
    assert res["n_accept"].tolist() == [2, 1]
    assert res["commit"].tolist() == [True, True, True, True]


def test_committed_tokens_are_the_autoregressive_ones():
    x = RNG.standard_normal((40, 50))
    ar = x.argmax(1)
    draft = ar.copy()
    draft[RNG.random(40) < 0.3] = 7
    res = verify_commit(x, draft, S=8)
    for b in range(5):
        n = res["n_accept"][b]
        assert (draft[b * 8:b * 8 + n] == ar[b * 8:b * 8 + n]).all()
        assert n == 8 or draft[b * 8 + n] != ar[b * 8 + n]
    assert (res["tokens"] == ar).all()
