"""Float64 oracle for the block refinement loop (test infrastructure only).

"Technical summary: Nemotron-TwoTower", §Methodology > Generation process
(Algorithm 1): a new block starts as S masked tokens; the denoiser refines it
over up to T steps; a block that is refined enough (by the confidence
threshold) is committed, after which the context tower absorbs it and the next
block starts. Only the inner refinement loop of one block position per
sequence is restated here.

Per step t (0-based), with the step's fresh inputs:
  1. run the attention of the step (its output does not feed the synthetic
     logits of the workload, so the loop's integer state depends only on the
     logits and the mask);
  2. confidence_unmask on the still-masked positions, with the per-block
     fallback when requested;
  3. committed positions leave the masked set, their token is final.
Stop when no sequence has a masked position, or after T steps.
"""

import numpy as np

from .unmask import confidence_unmask


def block_loop(step_logits, mask0, gamma, S, T, commit_at_least_one=True):
    """Run Algorithm 1's inner loop on per-step logits.

    step_logits: callable t -> logits [B*S, V] for step t.
    mask0: initial mask [B*S] (normally all ones).
    Returns dict with
      tokens      int64 [B*S]  final token per position (-1 if never committed)
      commit_step int64 [B*S]  step at which the position committed (-1 never)
      per_step    list of int  number of positions committed at each step
      steps       int          steps taken
      mask        bool [B*S]   final mask
    """
    mask = np.asarray(mask0).astype(bool).copy()
    n = mask.shape[0]
    tokens = np.full(n, -1, dtype=np.int64)
    commit_step = np.full(n, -1, dtype=np.int64)
    per_step = []
    steps = 0
    for t in range(T):
        if not mask.any():
            break
        res = confidence_unmask(step_logits(t), mask, gamma, block_S=S,
                                commit_at_least_one=commit_at_least_one)
        c = res["commit"]
        tokens[c] = res["tokens"][c]
        commit_step[c] = t
        per_step.append(int(c.sum()))
        mask = res["mask_out"]
        steps += 1
    return {
        "tokens": tokens,
        "commit_step": commit_step,
        "per_step": per_step,
        "steps": steps,
        "mask": mask,
    }
