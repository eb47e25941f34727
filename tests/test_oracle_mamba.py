"""Pins of the block-local bidirectional Mamba scan oracle.

The recurrence is pinned against an independent formulation: the same scan
written as a sum over tokens with cumulative decays (the quadratic, attention-
like form of a scalar-decay state-space model), evaluated with matrix algebra
rather than a loop. Plus: the reverse half equals the forward recurrence run on
the reversed block from a zero state, the one-token closed form, the group
mapping, and the boundary state's exact contribution.
"""

import numpy as np
import pytest

from oracle.mamba import batch_block_scan, block_scan

RNG = np.random.default_rng(21)


def _inputs(S=5, H=4, P=3, N=6, G=2, scale=1.0):
    x = RNG.standard_normal((S, H, P))
    dt = RNG.uniform(0.05, 0.5, (S, H))
    dt_r = RNG.uniform(0.05, 0.5, (S, H))
    Bm, Cm = RNG.standard_normal((S, G, N)), RNG.standard_normal((S, G, N))
    B_r, C_r = RNG.standard_normal((S, G, N)), RNG.standard_normal((S, G, N))
    A, A_r = -RNG.uniform(0.5, 3.0, H), -RNG.uniform(0.5, 3.0, H)
    Dskip = RNG.standard_normal(H)
    h0 = RNG.standard_normal((H, P, N)) * scale
    return x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0


def _quadratic(x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0):
    S, H, P = x.shape
    G = Bm.shape[1]
    y = np.zeros((S, H, P))
    for h in range(H):
        g = h // (H // G)
        la = np.cumsum(dt[:, h] * A[h])           # log prod_{r<=t} a_r
        la_r = np.cumsum(dt_r[:, h] * A_r[h])
        t, s = np.meshgrid(np.arange(S), np.arange(S), indexing="ij")
        # forward: coefficient of token s in y[t] is prod_{r=s+1..t} a_r (s <= t)
        Lf = np.where(s <= t, np.exp(la[t] - la[s]), 0.0)
        Mf = Lf * (Cm[:, g] @ Bm[:, g].T) * dt[None, :, h]
        y[:, h] = Mf @ x[:, h] + np.exp(la)[:, None] * (Cm[:, g] @ h0[h].T) + Dskip[h] * x[:, h]
        # reverse: coefficient of token s >= t is prod_{r=t..s-1} a'_r
        Lr = np.where(s >= t, np.exp((la_r[s] - dt_r[s, h] * A_r[h]) - (la_r[t] - dt_r[t, h] * A_r[h])), 0.0)
        Mr = Lr * (C_r[:, g] @ B_r[:, g].T) * dt_r[None, :, h]
        y[:, h] += Mr @ x[:, h]
    return y


@pytest.mark.parametrize("shape", [(5, 4, 3, 6, 2), (1, 2, 2, 4, 1), (9, 6, 4, 8, 3), (16, 8, 4, 16, 8)])
def test_recurrence_equals_quadratic_form(shape):
    S, H, P, N, G = shape
    args = _inputs(S, H, P, N, G)
    np.testing.assert_allclose(block_scan(*args), _quadratic(*args), rtol=1e-10, atol=1e-10)


def test_reverse_half_is_forward_scan_of_reversed_block():
    x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0 = _inputs(S=7)
    zero = np.zeros_like(dt)
    rev_part = block_scan(x, zero, Bm, Cm, dt_r, B_r, C_r, A, A_r, 0 * Dskip, 0 * h0)
    fwd_of_reversed = block_scan(x[::-1], dt_r[::-1], B_r[::-1], C_r[::-1], zero, Bm, Cm, A_r, A,
                                 0 * Dskip, 0 * h0)
    np.testing.assert_allclose(rev_part, fwd_of_reversed[::-1], rtol=1e-12, atol=1e-12)


def test_one_token_closed_form():
    x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0 = _inputs(S=1, H=2, P=3, N=4, G=1)
    y = block_scan(x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0)
    for h in range(2):
        a = np.exp(dt[0, h] * A[h])
        ref = (a * h0[h] + dt[0, h] * np.outer(x[0, h], Bm[0, 0])) @ Cm[0, 0] + Dskip[h] * x[0, h]
        ref += dt_r[0, h] * x[0, h] * float(B_r[0, 0] @ C_r[0, 0])
        np.testing.assert_allclose(y[0, h], ref, rtol=1e-13)


def test_group_mapping_is_contiguous():
    args = list(_inputs(S=4, H=4, P=2, N=3, G=2))
    y0 = block_scan(*args)
    args[2] = args[2].copy()
    args[2][:, 1] += 1.0          # group 1's B: heads 2 and 3 only
    y1 = block_scan(*args)
    assert np.array_equal(y0[:, :2], y1[:, :2])
    assert not np.allclose(y0[:, 2:], y1[:, 2:])


def test_boundary_state_enters_linearly_and_only_forward():
    x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0 = _inputs(S=6)
    y1 = block_scan(x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0)
    y0 = block_scan(x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, 0 * h0)
    H = x.shape[1]
    for h in range(H):
        g = h // (H // Bm.shape[1])
        decay = np.exp(np.cumsum(dt[:, h] * A[h]))
        np.testing.assert_allclose(y1[:, h] - y0[:, h], decay[:, None] * (Cm[:, g] @ h0[h].T),
                                   rtol=1e-12, atol=1e-12)


def test_batch_is_per_sequence():
    args = [np.stack([a, a2]) for a, a2 in zip(_inputs(), _inputs())]
    shared = [args[7][0], args[8][0], args[9][0]]
    full = args[:7] + shared + [args[10]]
    y = batch_block_scan(*full)
    for b in range(2):
        yb = block_scan(*[a[b] for a in args[:7]], *shared, args[10][b])
        assert np.array_equal(y[b], yb)
