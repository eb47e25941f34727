"""Float64 oracle for the denoiser's block attention (test infrastructure only).

What is computed, and where it comes from:

* "Technical summary: Nemotron-TwoTower", §Methodology > Architecture, item 2:
  the denoiser tower uses bidirectional attention among the tokens of the
  current noisy block and keeps a causal cross-attention to the same layer of
  the frozen context tower.
* Same page, §Methodology > Generation process, third bullet: at every layer
  the denoiser attends to the context-tower KV cache of the past blocks and to
  the current block's bidirectional KV.
* "Training Hybrid Block Diffusion Language Models with Partial
  Bidirectionality", §Methodology (cache-aligned objective): the prefix cache
  is a function of the clean prefix only, so it is an input here, never an
  output.

Readings where the pages are silent (each is listed with its reason in the
design notes of this repository):

* every block query sees all L_b prefix keys (the prefix lies wholly in the
  past, so "causal" holds at block granularity and needs no mask);
* every one of the S block keys is attended, still-masked positions included;
* one softmax over the concatenation prefix ++ block;
* score scale 1/sqrt(d) unless given;
* grouped-query heads map contiguously: query head h reads KV head h // g,
  g = H_q / H_kv;
* no position encoding inside this operation (the caller applies it).

Everything is float64. Inputs are upcast exactly (bf16 and fp32 values are
exactly representable in float64).
"""

import numpy as np


def _f64(x):
    """Exact upcast of a NumPy array or a torch tensor to a float64 array."""
    if hasattr(x, "detach"):  # torch tensor, any dtype / device
        x = x.detach().to("cpu")
        import torch  # local: only used when a tensor is handed in

        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _i64(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.asarray(x, dtype=np.int64)


def kv_head_of(h, g, H_kv):
    """Contiguous grouped-query mapping: query head h reads KV head h // g."""
    return h // g


def attend(q, K, V, scale):
    """Softmax attention of the rows of q over the key/value rows K, V.

    q: [n, d], K: [m, d], V: [m, dv] (float64). Returns (o [n, dv], lse [n]).
    o = softmax(q K^T * scale) V, computed stably by subtracting the row max;
    lse = max + log(sum(exp(s - max))) is the natural-log normaliser of the
    scores, the quantity that lets attention over disjoint key sets be merged.
    """
    s = (q @ K.T) * scale  # [n, m]
    mx = s.max(axis=1, keepdims=True)
    p = np.exp(s - mx)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ V) / l
    lse = mx[:, 0] + np.log(l[:, 0])
    return o, lse


def lse_combine(o_parts, lse_parts):
    """Merge attention results computed over disjoint key sets.

    For parts s with normalised outputs o_s and log-normalisers lse_s:
    M = max_s lse_s, w_s = exp(lse_s - M),
    o = sum_s w_s o_s / sum_s w_s, lse = M + log(sum_s w_s).
    This is the exact identity behind splitting a long prefix into chunks.

    o_parts: [P, n, dv], lse_parts: [P, n]. Returns (o [n, dv], lse [n]).
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    M = lse_parts.max(axis=0)
    w = np.exp(lse_parts - M[None, :])
    den = w.sum(axis=0)
    o = (w[:, :, None] * o_parts).sum(axis=0) / den[:, None]
    return o, M + np.log(den)


def block_attention(q, k_prefix, v_prefix, k_blk, v_blk, prefix_len,
                    prefix_offset, scale=None):
    """One denoiser attention step of the active block, per sequence.

    Shapes (row-major, last index fastest):
      q            [B, S, H_q, d]   block queries
      k_prefix     [R, H_kv, d]     packed clean-prefix keys (all sequences)
      v_prefix     [R, H_kv, d]     packed clean-prefix values
      k_blk, v_blk [B, S, H_kv, d]  the active block's own keys / values
      prefix_len   [B]              valid prefix rows of sequence b
      prefix_offset[B] (or [B+1])   first packed row of sequence b
    For every b, query head h (KV head kv = h // g) and block position i:
      keys   = k_prefix[off_b : off_b + L_b, kv] ++ k_blk[b, :, kv]
      values = v_prefix[off_b : off_b + L_b, kv] ++ v_blk[b, :, kv]
      o[b, i, h], lse[b, h, i] = attend(q[b, i, h], keys, values, scale)
    Returns (o [B, S, H_q, d] float64, lse [B, H_q, S] float64).
    """
    q = _f64(q)
    k_prefix = _f64(k_prefix)
    v_prefix = _f64(v_prefix)
    k_blk = _f64(k_blk)
    v_blk = _f64(v_blk)
    prefix_len = _i64(prefix_len)
    prefix_offset = _i64(prefix_offset)
    B, S, H_q, d = q.shape
    H_kv = k_blk.shape[2]
    if H_q % H_kv != 0:
        raise ValueError("H_q must be a multiple of H_kv")
    g = H_q // H_kv
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d)
    o = np.empty((B, S, H_q, v_blk.shape[3]), dtype=np.float64)
    lse = np.empty((B, H_q, S), dtype=np.float64)
    for b in range(B):
        L = int(prefix_len[b])
        off = int(prefix_offset[b])
        for h in range(H_q):
            kv = kv_head_of(h, g, H_kv)
            K = np.concatenate([k_prefix[off:off + L, kv, :], k_blk[b, :, kv, :]], axis=0)
            V = np.concatenate([v_prefix[off:off + L, kv, :], v_blk[b, :, kv, :]], axis=0)
            o_bh, lse_bh = attend(q[b, :, h, :], K, V, scale)
            o[b, :, h, :] = o_bh
            lse[b, h, :] = lse_bh
    return o, lse


def block_attention_rows(q, k_prefix, v_prefix, k_blk, v_blk, prefix_len,
                         prefix_offset, picks, scale=None):
    """The same as block_attention, for a sample of output rows only.

    picks: iterable of (b, i, h). Returns (o [n, d], lse [n]) in pick order.
    Used to check very large workloads, where the full oracle would not finish,
    on a sample of outputs that are each computed on their own.
    """
    B, S, H_q, d = q.shape
    H_kv = k_blk.shape[2]
    g = H_q // H_kv
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d)
    prefix_len = _i64(prefix_len)
    prefix_offset = _i64(prefix_offset)
    out_o, out_l = [], []
    for (b, i, h) in picks:
        L = int(prefix_len[b])
        off = int(prefix_offset[b])
        kv = kv_head_of(h, g, H_kv)
        K = np.concatenate([_f64(k_prefix[off:off + L, kv, :]), _f64(k_blk[b, :, kv, :])], axis=0)
        V = np.concatenate([_f64(v_prefix[off:off + L, kv, :]), _f64(v_blk[b, :, kv, :])], axis=0)
        o_r, l_r = attend(_f64(q[b, i, h, :])[None, :], K, V, scale)
        out_o.append(o_r[0])
        out_l.append(l_r[0])
    return np.stack(out_o), np.asarray(out_l)
