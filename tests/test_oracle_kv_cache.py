"""Pins of the block-commit (prefix-cache append) oracle.

"Technical summary: Nemotron-TwoTower", §Methodology > Generation process,
fourth bullet: after a block commits, the next block's prefix is the old
prefix followed by the committed block. The first pin states exactly that
through the (separately pinned) attention oracle: attention of a new block over
the appended cache equals attention over a cache laid out from scratch with
the concatenated rows. The others are invariants and edge cases of the layout.
"""

import numpy as np
import pytest

from oracle.attention import block_attention
from oracle.kv_cache import kv_append

RNG = np.random.default_rng(7)


def _cache(lens, cap, H_kv=2, d=8, junk=True):
    """Packed cache with `cap` rows reserved per sequence; rows past each
    sequence's length hold junk that a correct reader never uses."""
    B = len(lens)
    off = np.arange(B, dtype=np.int64) * cap
    rows = B * cap
    k = RNG.standard_normal((rows, H_kv, d)) if junk else np.zeros((rows, H_kv, d))
    v = RNG.standard_normal((rows, H_kv, d)) if junk else np.zeros((rows, H_kv, d))
    return k, v, np.array(lens, dtype=np.int32), off, np.full(B, cap, dtype=np.int64)


def test_next_block_sees_old_prefix_then_committed_block():
    B, S, H_q, H_kv, d = 3, 4, 4, 2, 8
    lens = [5, 0, 9]
    k, v, L, off, cap = _cache(lens, cap=16, H_kv=H_kv, d=d)
    k_new = RNG.standard_normal((B, S, H_kv, d))
    v_new = RNG.standard_normal((B, S, H_kv, d))
    k2, v2, L2, skipped = kv_append(k, v, k_new, v_new, L, off, cap)
    assert skipped == []
    # the same cache laid out from scratch: sequence b's rows are its old
    # prefix rows followed by the committed block, packed back to back
    ks, vs, offs = [], [], [0]
    for b in range(B):
        ks.append(np.concatenate([k[off[b]:off[b] + lens[b]], k_new[b]], axis=0))
        vs.append(np.concatenate([v[off[b]:off[b] + lens[b]], v_new[b]], axis=0))
        offs.append(offs[-1] + lens[b] + S)
    k_ref, v_ref = np.concatenate(ks), np.concatenate(vs)
    lens_ref = np.array(lens) + S
    q = RNG.standard_normal((B, S, H_q, d))
    kb = RNG.standard_normal((B, S, H_kv, d))
    vb = RNG.standard_normal((B, S, H_kv, d))
    o1, l1 = block_attention(q, k2, v2, kb, vb, L2, off)
    o2, l2 = block_attention(q, k_ref, v_ref, kb, vb, lens_ref, np.array(offs[:-1]))
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
    assert L2.tolist() == (np.array(lens) + S).tolist()


def test_only_the_appended_rows_change():
    B, S = 4, 3
    k, v, L, off, cap = _cache([2, 7, 0, 4], cap=12)
    kn = RNG.standard_normal((B, S, 2, 8))
    vn = RNG.standard_normal((B, S, 2, 8))
    sel = np.array([1, 0, 1, 1], dtype=np.uint8)
    k2, v2, L2, skipped = kv_append(k, v, kn, vn, L, off, cap, seq_mask=sel)
    assert skipped == []
    changed = np.zeros(k.shape[0], dtype=bool)
    for b in range(B):
        if sel[b]:
            lo = off[b] + L[b]
            changed[lo:lo + S] = True
            assert np.array_equal(k2[lo:lo + S], kn[b]) and np.array_equal(v2[lo:lo + S], vn[b])
    assert np.array_equal(k2[~changed], k[~changed]) and np.array_equal(v2[~changed], v[~changed])
    assert L2.tolist() == [L[0] + S, L[1], L[2] + S, L[3] + S]


def test_two_appends_equal_one_append_of_both_blocks():
    k, v, L, off, cap = _cache([3, 1], cap=20)
    a_k, a_v = RNG.standard_normal((2, 4, 2, 8)), RNG.standard_normal((2, 4, 2, 8))
    b_k, b_v = RNG.standard_normal((2, 4, 2, 8)), RNG.standard_normal((2, 4, 2, 8))
    k1, v1, L1, _ = kv_append(k, v, a_k, a_v, L, off, cap)
    k1, v1, L1, _ = kv_append(k1, v1, b_k, b_v, L1, off, cap)
    k2, v2, L2, _ = kv_append(k, v, np.concatenate([a_k, b_k], 1), np.concatenate([a_v, b_v], 1),
                              L, off, cap)
    assert np.array_equal(k1, k2) and np.array_equal(v1, v2) and np.array_equal(L1, L2)


@pytest.mark.parametrize("lens,cap,S,skip", [
    ([12], 16, 4, []),        # exactly fills the reserved rows
    ([13], 16, 4, [0]),       # one row too many
    ([0], 3, 4, [0]),         # block larger than the reservation
    ([-1], 16, 4, [0]),       # negative length
])
def test_capacity_edges(lens, cap, S, skip):
    k, v, L, off, capa = _cache([max(x, 0) for x in lens], cap=cap)
    L = np.array(lens, dtype=np.int32)
    kn, vn = RNG.standard_normal((1, S, 2, 8)), RNG.standard_normal((1, S, 2, 8))
    k2, v2, L2, skipped = kv_append(k, v, kn, vn, L, off, capa)
    assert skipped == skip
    if skip:
        assert np.array_equal(k2, k) and np.array_equal(v2, v) and np.array_equal(L2, L)
    else:
        assert L2[0] == lens[0] + S
        assert np.array_equal(k2[lens[0]:lens[0] + S], kn[0])


def test_bf16_tensors_copy_bit_patterns():
    torch = pytest.importorskip("torch")
    k = torch.randn(10, 2, 8).to(torch.bfloat16)
    kn = torch.randn(1, 3, 2, 8).to(torch.bfloat16)
    k2, _, L2, _ = kv_append(k, k, kn, kn, torch.tensor([4], dtype=torch.int32),
                             torch.tensor([0]), torch.tensor([10]))
    assert np.array_equal(k2[4:7], kn[0].view(torch.int16).numpy())
    assert np.array_equal(k2[:4], k[:4].view(torch.int16).numpy())
    assert L2.tolist() == [7]


def test_overflow_into_the_next_sequence_is_refused():
    # sequence 0 would spill into rows reserved for sequence 1 (still inside
    # the array): it is skipped and sequence 1 keeps its rows
    k, v, L, off, cap = _cache([6, 2], cap=8)
    kn, vn = RNG.standard_normal((2, 4, 2, 8)), RNG.standard_normal((2, 4, 2, 8))
    k2, v2, L2, skipped = kv_append(k, v, kn, vn, L, off, cap)
    assert skipped == [0]
    assert L2.tolist() == [6, 6]
    assert np.array_equal(k2[:10], k[:10]) and np.array_equal(v2[:10], v[:10])
    assert np.array_equal(k2[10:14], kn[1])
