"""Oracle of the block-local bidirectional Mamba scan (test infrastructure
only).

"Training Hybrid Block Diffusion Language Models with Partial
Bidirectionality", §Methodology (partial bidirectionality, cache-aligned
objective): a Mamba layer keeps, for the finished prefix, only a forward
boundary state (its recurrent state after the prefix); inside the active
denoising block the layer mixes in both directions, but the reverse scan is
confined to the block, so the cached prefix state never depends on the noisy
block or the diffusion step. "Technical summary: Nemotron-TwoTower",
§Methodology: the backbone's Mamba layers are Mamba-2.

The recurrence is not printed on the pages; this restates the published
Mamba-2 selective state-space recurrence (scalar decay per head, grouped B/C)
in the plainest reading:

  forward, from the cached boundary state h_fwd[-1] = h0 (per head, P x N):
      h_fwd[t] = exp(dt[t] * A) * h_fwd[t-1] + dt[t] * outer(x[t], B[t])
      y_fwd[t] = h_fwd[t] @ C[t] + Dskip * x[t]
  reverse, inside the block only, from zero after its last token:
      h_rev[t] = exp(dt_r[t] * A_r) * h_rev[t+1] + dt_r[t] * outer(x[t], B_r[t])
      y_rev[t] = h_rev[t] @ C_r[t]
  y[t] = y_fwd[t] + y_rev[t]

x [S, H, P] is shared by both directions; each direction has its own step
sizes dt (already positive, i.e. after the softplus), decay A (< 0) and
projections B, C [S, G, N]; head h uses group h // (H / G). The boundary state
is an input and is not updated (the block is not committed yet).

Plain float64 loops in the recurrence's own order.
"""

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        import torch

        x = x.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def block_scan(x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0):
    """One block of one sequence. Shapes: x [S,H,P]; dt, dt_r [S,H];
    Bm, Cm, B_r, C_r [S,G,N]; A, A_r, Dskip [H]; h0 [H,P,N].
    Returns y [S,H,P] (float64)."""
    x, dt, Bm, Cm = _f64(x), _f64(dt), _f64(Bm), _f64(Cm)
    dt_r, B_r, C_r = _f64(dt_r), _f64(B_r), _f64(C_r)
    A, A_r, Dskip, h0 = _f64(A), _f64(A_r), _f64(Dskip), _f64(h0)
    S, H, P = x.shape
    G = Bm.shape[1]
    hpg = H // G
    y = np.zeros((S, H, P))
    for h in range(H):
        g = h // hpg
        state = h0[h].copy()
        for t in range(S):
            state = np.exp(dt[t, h] * A[h]) * state + dt[t, h] * np.outer(x[t, h], Bm[t, g])
            y[t, h] += state @ Cm[t, g] + Dskip[h] * x[t, h]
        state = np.zeros_like(h0[h])
        for t in range(S - 1, -1, -1):
            state = np.exp(dt_r[t, h] * A_r[h]) * state + dt_r[t, h] * np.outer(x[t, h], B_r[t, g])
            y[t, h] += state @ C_r[t, g]
    return y


def batch_block_scan(x, dt, Bm, Cm, dt_r, B_r, C_r, A, A_r, Dskip, h0):
    """The same for B sequences: every input gains a leading batch axis except
    A, A_r, Dskip (shared by the layer). Returns y [B,S,H,P]."""
    x = _f64(x)
    return np.stack([block_scan(x[b], _f64(dt)[b], _f64(Bm)[b], _f64(Cm)[b], _f64(dt_r)[b],
                                _f64(B_r)[b], _f64(C_r)[b], A, A_r, Dskip, _f64(h0)[b])
                     for b in range(x.shape[0])])
