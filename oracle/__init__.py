"""Float64 CPU oracle for one denoising step of a block-diffusion LM.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, obviously-correct
restatement of what the denoise step computes, written from the source pages:

* "Technical summary: Nemotron-TwoTower" (gist.science, 2606.26493),
  §Methodology > Architecture (frozen causal context tower, denoiser with
  bidirectional block attention plus layer-aligned causal cross-attention),
  §Methodology > Generation process (Algorithm 1: S masked tokens refined over
  T steps, attending to the context-tower KV of past blocks and the current
  block's bidirectional KV), and §Training and conditioning > Sampling
  (Algorithm 2: confidence unmasking with threshold gamma), and the fourth
  bullet of §Generation process (a committed block extends the prefix that the
  next block attends to: the prefix-cache append).
* "Training Hybrid Block Diffusion Language Models with Partial
  Bidirectionality" (gist.science, 2607.02805), §Methodology: the clean-prefix
  cache depends only on the prefix, never on the diffusion step, so the
  denoiser reads it and never writes it.
* "Nemotron-Labs Diffusion" (molayo1419.me), diffusion mode (FastDiffuser):
  32-token blocks filled by iterative denoising with a confidence threshold.
* The LM head in front of Algorithm 2 (``lmhead``) and the block-local
  bidirectional Mamba scan of the partial-bidirectionality page (``mamba``),
  and self-speculative verification (``spec``: "Nemotron-Labs Diffusion",
  self-speculation mode), each restated in its module with its readings.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import it. The CUDA product path
(``block_diffusion_lm_bd_b200``) shares no code with it and never imports it.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against library routines, closed forms, invariants, brute force and
hand-enumerated golden cases. Whole-pipeline numbers against the pages are
"parity unpinned": the pages print no worked numeric example for this path.
"""

from .attention import attend, block_attention, lse_combine
from .unmask import confidence_unmask, top2_gap
from .loop import block_loop
from .kv_cache import kv_append
from .lmhead import lmhead_logits, lmhead_unmask
from .mamba import batch_block_scan, block_scan
from .spec import causal_block_attention, verify_commit

__all__ = [
    "attend",
    "block_attention",
    "lse_combine",
    "confidence_unmask",
    "top2_gap",
    "block_loop",
    "kv_append",
    "lmhead_logits",
    "lmhead_unmask",
    "block_scan",
    "batch_block_scan",
    "causal_block_attention",
    "verify_commit",
]
