"""Oracle of self-speculative verification (test infrastructure only).

"Nemotron-Labs Diffusion", self-speculation mode (LinearSpec): the model drafts
a block bidirectionally (the diffusion step), then checks the draft causally
(the autoregressive step), and every position of the matching prefix commits;
at temperature 0 the result is the one autoregressive decoding gives.

Two parts:

* causal_block_attention - the verification pass's attention: block position
  i attends to the whole clean prefix and to the block's keys 0 .. i only
  (causal inside the block, the mask of an autoregressive pass over the
  drafted tokens); otherwise exactly block_attention.
* verify_commit - the commit rule. Readings (the page states the rule in one
  sentence): row i of the logits is the autoregressive prediction of block
  position i (the caller aligns them); a_i = its argmax (lowest id on ties);
  n = the number of leading positions with a_i == draft_i; positions 0 .. n-1
  commit with their (equal) tokens, and, when n < S, position n also commits
  with a_n - the token the autoregressive pass itself produces there, which
  keeps the result identical to autoregressive decoding at temperature 0
  (standard speculative verification). Later positions stay uncommitted.
"""

import numpy as np

from .attention import _f64, _i64, attend, kv_head_of


def causal_block_attention(q, k_prefix, v_prefix, k_blk, v_blk, prefix_len, prefix_offset,
                           scale=None):
    """As block_attention, but block position i sees block keys 0 .. i only.
    Returns (o [B, S, H_q, d], lse [B, H_q, S]) in float64."""
    q, k_blk, v_blk = _f64(q), _f64(k_blk), _f64(v_blk)
    k_prefix, v_prefix = _f64(k_prefix), _f64(v_prefix)
    prefix_len, prefix_offset = _i64(prefix_len), _i64(prefix_offset)
    B, S, H_q, d = q.shape
    H_kv = k_blk.shape[2]
    g = H_q // H_kv
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d)
    o = np.empty((B, S, H_q, v_blk.shape[3]))
    lse = np.empty((B, H_q, S))
    for b in range(B):
        L, off = int(prefix_len[b]), int(prefix_offset[b])
        for h in range(H_q):
            kv = kv_head_of(h, g, H_kv)
            for i in range(S):
                K = np.concatenate([k_prefix[off:off + L, kv], k_blk[b, :i + 1, kv]], axis=0)
                V = np.concatenate([v_prefix[off:off + L, kv], v_blk[b, :i + 1, kv]], axis=0)
                o_i, l_i = attend(q[b, i, h][None, :], K, V, scale)
                o[b, i, h] = o_i[0]
                lse[b, h, i] = l_i[0]
    return o, lse


def verify_commit(logits, draft, S):
    """logits [B*S, V] (row i of block b predicts its position i), draft int
    [B*S]. Returns dict: tokens int64 [B*S] (the argmax of every row), commit
    bool [B*S], n_accept int64 [B] (length of the matching prefix)."""
    x = _f64(logits)
    d = np.asarray(draft.detach().cpu().numpy() if hasattr(draft, "detach") else draft,
                   dtype=np.int64)
    rows = x.shape[0]
    tokens = np.empty(rows, dtype=np.int64)
    for r in range(rows):
        tokens[r] = int(np.flatnonzero(x[r] == x[r].max())[0])
    B = rows // S
    commit = np.zeros(rows, dtype=bool)
    n_accept = np.zeros(B, dtype=np.int64)
    for b in range(B):
        n = 0
        while n < S and tokens[b * S + n] == d[b * S + n]:
            n += 1
        n_accept[b] = n
        commit[b * S:b * S + n] = True
        if n < S:
            commit[b * S + n] = True  # the autoregressive token at the first mismatch
    return {"tokens": tokens, "commit": commit, "n_accept": n_accept}
