"""Oracle of committing a finished block into the prefix cache (test
infrastructure only).

"Technical summary: Nemotron-TwoTower", §Methodology > Generation process,
fourth bullet: once a block has been refined enough it is committed, the
context tower takes the new clean tokens into its state, and the process
repeats for the next block. So the next block's prefix is the old prefix
followed by the committed block, and the context tower's keys and values of
those S tokens extend the cache that the denoiser reads. Here those K/V are an
input (the context tower is a model this repository does not run); the
operation places them after each sequence's old prefix rows and lengthens the
prefix by S.

Layout (the same one the attention oracle reads): packed rows
[prefix_rows, H_kv, d]; sequence b owns rows prefix_offset[b] ..
prefix_offset[b] + prefix_capacity[b] - 1, of which the first prefix_len[b]
are valid. A selected sequence whose new rows would leave its own rows or the
array is skipped and reported; nothing of it changes.

Plain NumPy array copies: no arithmetic, so every value is reproduced bit for
bit whatever its dtype.
"""

import numpy as np


def _np(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: only when a tensor is handed in

        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().copy()  # bit pattern, copied exactly
        return x.numpy().copy()
    return np.array(x, copy=True)


def kv_append(k_prefix, v_prefix, k_new, v_new, prefix_len, prefix_offset, prefix_capacity,
              seq_mask=None):
    """Returns (k_prefix', v_prefix', prefix_len', skipped): new arrays after the
    append, and the list of selected sequences that were skipped because their
    new rows do not fit. Values are copied by bit pattern (bf16 tensors are
    handled as int16 bit patterns), so the result is exact."""
    k = _np(k_prefix)
    v = _np(v_prefix)
    kn = _np(k_new)
    vn = _np(v_new)
    L = np.asarray(_np(prefix_len), dtype=np.int64).copy()
    off = np.asarray(_np(prefix_offset), dtype=np.int64)
    cap = np.asarray(_np(prefix_capacity), dtype=np.int64)
    B, S = kn.shape[0], kn.shape[1]
    rows = k.shape[0]
    sel = np.ones(B, dtype=bool) if seq_mask is None else np.asarray(_np(seq_mask)) != 0
    skipped = []
    for b in range(B):
        if not sel[b]:
            continue
        lo = off[b] + L[b]
        fits = (L[b] >= 0 and off[b] >= 0 and cap[b] >= 0 and L[b] + S <= cap[b]
                and lo + S <= rows and L[b] + S <= 2**31 - 1)
        if not fits:
            skipped.append(b)
            continue
        k[lo:lo + S] = kn[b]
        v[lo:lo + S] = vn[b]
        L[b] += S
    return k, v, L.astype(np.int32), skipped
