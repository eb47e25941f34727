"""Oracle of the LM head fused with confidence unmasking (test
infrastructure only).

The step right before confidence unmasking ("Technical summary:
Nemotron-TwoTower", §Training and conditioning > Sampling, Algorithm 2: the
denoiser predicts every masked token in parallel, and a token commits when its
confidence is higher than gamma): the prediction of position r is the
vocabulary projection of its final hidden state,
    l[r, v] = sum_k hidden[r, k] * W[v, k],
followed by the full-vocabulary softmax whose argmax and top probability
Algorithm 2 uses. Fusing the projection with the reduction changes nothing in
what is computed; it only keeps the [rows, V] logits out of memory.

Readings where the pages are silent: the head is a plain bias-free linear map
(no softcap, no temperature, no scaling), W is [V, D] row-major (one vocabulary
row per token), and only masked positions are predicted.

float64 throughout: bf16 inputs upcast exactly; each logit is the exact
product sum up to float64 rounding (far below the float32 rounding the GPU's
accumulation carries).
"""

import numpy as np

from .unmask import confidence_unmask


def _f64(x):
    if hasattr(x, "detach"):
        import torch

        x = x.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def lmhead_logits(hidden, w_vocab, rows=None):
    """l = hidden @ W^T in float64: hidden [R, D], W [V, D] -> [R, V] (or the
    listed rows only)."""
    h = _f64(hidden)
    if rows is not None:
        h = h[np.asarray(rows, dtype=np.int64)]
    return h @ _f64(w_vocab).T


def lmhead_unmask(hidden, w_vocab, mask, gamma, block_S=None, commit_at_least_one=False):
    """Algorithm 2 on the projected logits of the masked rows: the same result
    dict as confidence_unmask, plus the float64 logits of every row under
    "logits" (unmasked rows: NaN), which the tests use to bound rounding."""
    m = np.asarray(mask.detach().cpu().numpy() if hasattr(mask, "detach") else mask).astype(bool)
    V = int(w_vocab.shape[0])
    logits = np.full((m.shape[0], V), np.nan)
    idx = np.flatnonzero(m)
    if idx.size:
        logits[idx] = lmhead_logits(hidden, w_vocab, rows=idx)
    safe = np.where(m[:, None], logits, 0.0)  # unmasked rows are never looked at
    res = confidence_unmask(safe, m, gamma, block_S=block_S,
                            commit_at_least_one=commit_at_least_one)
    res["logits"] = logits
    return res
