"""Pins for the float64 attention oracle, against things other than itself.

Each test ties the oracle to a library routine, a closed form, an invariant
the pages fix, or brute force on tiny inputs:

* the operation is softmax(q K^T / sqrt(d)) V over prefix ++ block keys
  (torch scaled_dot_product_attention in float64, grouped heads via
  enable_gqa, which repeats each KV head over its contiguous query group);
* prefix_len = 0 leaves full bidirectional attention over the block
  ("Technical summary: Nemotron-TwoTower", §Methodology > Architecture);
* S = 1 is ordinary causal decode attention of one query over the prefix and
  itself ("Nemotron-Labs Diffusion", AR mode as the correctness reference);
* shuffling the block positions shuffles the outputs (no mask, no position
  encoding inside the block);
* splitting the keys and merging by log-sum-exp gives the unsplit result;
* q = 0 gives the mean of the values and lse = log(number of keys).
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle.attention import attend, block_attention, block_attention_rows, lse_combine


def _inputs(B, S, H_q, H_kv, d, lens, seed, pad=0, std=1.0):
    g = torch.Generator().manual_seed(seed)
    lens = list(lens)
    off = [0]
    for L in lens:
        off.append(off[-1] + L + pad)
    R = max(off[-1], 1)
    t = lambda *s: (torch.randn(*s, generator=g, dtype=torch.float64) * std)
    return dict(
        q=t(B, S, H_q, d),
        k_prefix=t(R, H_kv, d),
        v_prefix=t(R, H_kv, d),
        k_blk=t(B, S, H_kv, d),
        v_blk=t(B, S, H_kv, d),
        prefix_len=np.array(lens, dtype=np.int64),
        prefix_offset=np.array(off, dtype=np.int64),
    )


def _run(inp, scale=None):
    return block_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["k_blk"],
                           inp["v_blk"], inp["prefix_len"], inp["prefix_offset"], scale=scale)


def _sdpa_reference(inp, scale=None):
    """torch SDPA (float64, CPU) over the concatenated keys, per sequence."""
    q = inp["q"]
    B, S, H_q, d = q.shape
    outs = []
    for b in range(B):
        L = int(inp["prefix_len"][b])
        off = int(inp["prefix_offset"][b])
        K = torch.cat([inp["k_prefix"][off:off + L], inp["k_blk"][b]], 0)  # [L+S, H_kv, d]
        V = torch.cat([inp["v_prefix"][off:off + L], inp["v_blk"][b]], 0)
        o = torch.nn.functional.scaled_dot_product_attention(
            q[b].permute(1, 0, 2)[None], K.permute(1, 0, 2)[None], V.permute(1, 0, 2)[None],
            scale=scale, enable_gqa=True)
        outs.append(o[0].permute(1, 0, 2))
    return torch.stack(outs).numpy()


CASES = [
    # B, S, H_q, H_kv, d, lens
    (1, 4, 2, 1, 8, [5]),
    (2, 3, 6, 2, 4, [0, 9]),
    (3, 16, 8, 2, 16, [37, 1, 128]),
    (2, 32, 4, 4, 8, [200, 3]),
    (1, 1, 3, 1, 8, [17]),
]


@pytest.mark.parametrize("case", CASES)
def test_matches_sdpa_over_concatenation(case):
    B, S, H_q, H_kv, d, lens = case
    inp = _inputs(B, S, H_q, H_kv, d, lens, seed=11 + B + S)
    o, _ = _run(inp)
    ref = _sdpa_reference(inp)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_explicit_scale_matches_sdpa():
    inp = _inputs(2, 5, 4, 2, 8, [7, 12], seed=3)
    o, _ = _run(inp, scale=0.37)
    np.testing.assert_allclose(o, _sdpa_reference(inp, scale=0.37), rtol=0, atol=1e-12)


def test_prefix_len_zero_is_full_bidirectional_attention():
    inp = _inputs(2, 16, 8, 2, 16, [0, 0], seed=5)
    o, _ = _run(inp)
    for b in range(2):
        ref = torch.nn.functional.scaled_dot_product_attention(
            inp["q"][b].permute(1, 0, 2)[None], inp["k_blk"][b].permute(1, 0, 2)[None],
            inp["v_blk"][b].permute(1, 0, 2)[None], is_causal=False, enable_gqa=True)
        np.testing.assert_allclose(o[b], ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("L", [0, 1, 9, 64])
def test_block_of_one_is_causal_decode(L):
    """S = 1: the single block token is the newest position of a causal LM."""
    H_q, H_kv, d = 4, 2, 8
    inp = _inputs(1, 1, H_q, H_kv, d, [L], seed=40 + L)
    o, _ = _run(inp)
    g = torch.Generator().manual_seed(99)
    q_prev = torch.randn(L, H_q, d, generator=g, dtype=torch.float64)
    Q = torch.cat([q_prev, inp["q"][0]], 0)                       # [L+1, H_q, d]
    K = torch.cat([inp["k_prefix"][:L], inp["k_blk"][0]], 0)      # [L+1, H_kv, d]
    V = torch.cat([inp["v_prefix"][:L], inp["v_blk"][0]], 0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.permute(1, 0, 2)[None], K.permute(1, 0, 2)[None], V.permute(1, 0, 2)[None],
        is_causal=True, enable_gqa=True)[0].permute(1, 0, 2)
    np.testing.assert_allclose(o[0, 0], ref[L].numpy(), rtol=0, atol=1e-12)


def test_block_permutation_equivariance():
    inp = _inputs(2, 16, 8, 2, 16, [33, 70], seed=7)
    o, lse = _run(inp)
    perm = torch.randperm(16, generator=torch.Generator().manual_seed(1))
    pin = dict(inp)
    for k in ("q", "k_blk", "v_blk"):
        pin[k] = inp[k][:, perm]
    o2, lse2 = _run(pin)
    np.testing.assert_allclose(o2, o[:, perm.numpy()], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse[:, :, perm.numpy()], rtol=0, atol=1e-12)


def test_split_and_lse_merge_equals_whole():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((6, 16))
    K = rng.standard_normal((300, 16)) * 2.0
    V = rng.standard_normal((300, 16))
    o, lse = attend(q, K, V, 0.25)
    for cuts in ([150], [1, 299], [10, 64, 200, 250]):
        edges = [0] + cuts + [300]
        parts = [attend(q, K[a:b], V[a:b], 0.25) for a, b in zip(edges[:-1], edges[1:])]
        o2, lse2 = lse_combine([p[0] for p in parts], [p[1] for p in parts])
        np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)


def test_zero_query_closed_form():
    inp = _inputs(2, 4, 4, 2, 8, [10, 3], seed=9)
    inp["q"][:] = 0
    o, lse = _run(inp)
    for b in range(2):
        L, off = int(inp["prefix_len"][b]), int(inp["prefix_offset"][b])
        for h in range(4):
            kv = h // 2
            V = torch.cat([inp["v_prefix"][off:off + L, kv], inp["v_blk"][b, :, kv]], 0)
            np.testing.assert_allclose(o[b, :, h], V.mean(0).numpy()[None].repeat(4, 0),
                                       rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[b, h], math.log(L + 4), rtol=0, atol=1e-13)


def test_unused_padding_rows_are_never_read():
    base = _inputs(3, 8, 4, 2, 8, [5, 0, 11], seed=21)
    padded = _inputs(3, 8, 4, 2, 8, [5, 0, 11], seed=21, pad=4)
    # copy the valid rows of base into the padded layout, fill the gaps with huge values
    for k in ("k_prefix", "v_prefix"):
        padded[k][:] = 1e6
        for b in range(3):
            L = int(base["prefix_len"][b])
            s0, s1 = int(base["prefix_offset"][b]), int(padded["prefix_offset"][b])
            padded[k][s1:s1 + L] = base[k][s0:s0 + L]
    for k in ("q", "k_blk", "v_blk"):
        padded[k] = base[k]
    o, lse = _run(base)
    o2, lse2 = _run(padded)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_brute_force_triple_loop_tiny():
    """Pure-Python loops over keys, no NumPy reductions, on tiny inputs."""
    for seed, (B, S, H_q, H_kv, d, lens) in enumerate([(1, 2, 2, 1, 3, [3]), (2, 3, 4, 2, 4, [0, 5]),
                                                      (1, 4, 3, 3, 2, [9])]):
        inp = _inputs(B, S, H_q, H_kv, d, lens, seed=100 + seed)
        o, lse = _run(inp)
        sc = 1.0 / math.sqrt(d)
        g = H_q // H_kv
        for b in range(B):
            L, off = int(inp["prefix_len"][b]), int(inp["prefix_offset"][b])
            for h in range(H_q):
                kv = h // g
                keys = [inp["k_prefix"][off + j, kv].tolist() for j in range(L)] + \
                       [inp["k_blk"][b, j, kv].tolist() for j in range(S)]
                vals = [inp["v_prefix"][off + j, kv].tolist() for j in range(L)] + \
                       [inp["v_blk"][b, j, kv].tolist() for j in range(S)]
                for i in range(S):
                    qi = inp["q"][b, i, h].tolist()
                    sc_list = [sum(qi[t] * k[t] for t in range(d)) * sc for k in keys]
                    mx = max(sc_list)
                    w = [math.exp(s - mx) for s in sc_list]
                    z = sum(w)
                    for t in range(d):
                        ref = sum(w[j] * vals[j][t] for j in range(len(keys))) / z
                        assert abs(o[b, i, h, t] - ref) < 1e-12
                    assert abs(lse[b, h, i] - (mx + math.log(z))) < 1e-12


def test_sampled_rows_match_full_oracle():
    inp = _inputs(2, 8, 8, 2, 16, [40, 7], seed=31)
    o, lse = _run(inp)
    picks = [(0, 0, 0), (1, 7, 7), (0, 3, 5), (1, 2, 1)]
    o2, l2 = block_attention_rows(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["k_blk"],
                                  inp["v_blk"], inp["prefix_len"], inp["prefix_offset"], picks)
    for n, (b, i, h) in enumerate(picks):
        np.testing.assert_allclose(o2[n], o[b, i, h], rtol=0, atol=1e-14)
        assert abs(l2[n] - lse[b, h, i]) < 1e-14


def test_accepts_bf16_tensors_exactly():
    g = torch.Generator().manual_seed(0)
    q = torch.randn(1, 2, 2, 8, generator=g).to(torch.bfloat16)
    kp = torch.randn(4, 1, 8, generator=g).to(torch.bfloat16)
    kb = torch.randn(1, 2, 1, 8, generator=g).to(torch.bfloat16)
    o, _ = block_attention(q, kp, kp, kb, kb, [4], [0, 4])
    ref, _ = block_attention(q.double().numpy(), kp.double().numpy(), kp.double().numpy(),
                             kb.double().numpy(), kb.double().numpy(), [4], [0, 4])
    np.testing.assert_array_equal(o, ref)
