"""Float64 oracle for confidence unmasking (test infrastructure only).

"Technical summary: Nemotron-TwoTower", §Training and conditioning >
Sampling (Algorithm 2): at every step the denoiser predicts all masked tokens
in parallel; tokens whose confidence is higher than the threshold gamma are
committed, the uncertain ones stay masked, so the number committed per step
adapts. "Nemotron-Labs Diffusion", diffusion mode (FastDiffuser): a 32-token
block is filled over several denoising steps, a confidence threshold deciding
which tokens commit at each step.

Readings where the pages are silent:

* confidence = the largest softmax probability of the position's full-
  vocabulary distribution at temperature 1, i.e. the probability of the argmax
  token: conf = exp(l_tok - logsumexp(l)) = 1 / sum_v exp(l_v - max_v l);
* greedy token = the argmax, lowest vocabulary index on exact ties;
* strict comparison conf > gamma ("higher than the threshold");
* the threshold is the float32 value of gamma, upcast;
* optional per-block fallback (an opt-in build assumption, not from the
  pages): when a block still has masked positions and none passes gamma, the
  masked position of highest confidence commits (lowest position on ties);
* committed tokens are final (never re-masked).
"""

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        import torch

        x = x.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _bool(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.asarray(x).astype(bool)


def confidence_unmask(logits, mask, gamma, block_S=None, commit_at_least_one=False):
    """Algorithm 2 on a batch of positions.

    logits [rows, V] (float32 values; upcast exactly), mask [rows] (nonzero =
    still masked), gamma (float; rounded to float32 as the threshold).
    block_S groups consecutive rows into blocks for the optional fallback.

    Returns a dict of NumPy arrays, one entry per row:
      tokens   int64    argmax token of masked rows, -1 for unmasked rows
      conf     float64  confidence of masked rows, NaN for unmasked rows
      commit   bool     masked and conf > gamma (or chosen by the fallback)
      mask_out bool     mask and not commit
      fallback bool     committed by the fallback rule
    """
    x = _f64(logits)
    m = _bool(mask)
    rows, V = x.shape
    thr = float(np.float32(gamma))
    tokens = np.full(rows, -1, dtype=np.int64)
    conf = np.full(rows, np.nan, dtype=np.float64)
    commit = np.zeros(rows, dtype=bool)
    fallback = np.zeros(rows, dtype=bool)
    for r in range(rows):
        if not m[r]:
            continue
        row = x[r]
        mx = row.max()
        tok = int(np.flatnonzero(row == mx)[0])  # lowest index on ties
        z = np.exp(row - mx).sum()
        tokens[r] = tok
        conf[r] = 1.0 / z
        commit[r] = conf[r] > thr
    if commit_at_least_one:
        if not block_S or block_S <= 0:
            raise ValueError("the fallback needs block_S > 0")
        for start in range(0, rows, block_S):
            sl = slice(start, min(start + block_S, rows))
            masked = np.flatnonzero(m[sl])
            if masked.size == 0 or commit[sl].any():
                continue
            c = conf[sl][masked]
            best = masked[int(np.flatnonzero(c == c.max())[0])]  # lowest position on ties
            commit[start + best] = True
            fallback[start + best] = True
    return {
        "tokens": tokens,
        "conf": conf,
        "commit": commit,
        "mask_out": m & ~commit,
        "fallback": fallback,
    }


def top2_gap(logits):
    """Per row: largest logit minus the second largest (0 on a tie).

    Rows whose gap is below 1e-6 have no stable argmax between two
    implementations that round differently; parity reports them separately.
    """
    x = _f64(logits)
    if x.shape[1] < 2:  # one token: no runner-up, the argmax is unique
        return np.full(x.shape[0], np.inf)
    part = np.partition(x, x.shape[1] - 2, axis=1)
    return part[:, -1] - part[:, -2]
