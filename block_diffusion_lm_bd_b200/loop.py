"""The block refinement loop: Algorithm 1's inner loop over one block.

"Technical summary: Nemotron-TwoTower", Methodology > Generation process: a
new block starts as S masked tokens and the denoiser refines it over up to T
steps; each step attends to the context-tower KV of the past blocks and the
block's own KV, then commits (Training and conditioning > Sampling,
Algorithm 2) the positions whose confidence is higher than gamma. Committed
tokens are final.

Host orchestration only: every step is one bd_attn_step and one bd_unmask
(mask updated in place, optional per-block fallback); when the block is done,
commit_block is one bd_kv_append: the block's clean K/V (the context tower's,
supplied by the caller) join the prefix cache, so the next block's prefix is
the old one followed by this block (Generation process, fourth bullet). Committed tokens
accumulate in one tokens buffer because bd_unmask leaves the rows that are no
longer masked untouched. The only synchronisation per step is the read-back
of the mask (one byte per position) that decides whether to stop.
"""

import numpy as np
import torch

from . import api


class BlockLoop:
    """State and buffers of the refinement loop of B blocks of S positions.

    step_inputs(t) -> dict with the step's device tensors: q, k_prefix,
    v_prefix, k_blk, v_blk, prefix_len, prefix_offset and logits [B*S, V].
    """

    def __init__(self, B, S, H_q, H_kv, d, V, gamma, device, commit_at_least_one=True,
                 stream=None):
        self.B, self.S, self.V, self.gamma = B, S, V, gamma
        self.fallback = commit_at_least_one
        self.stream = stream
        rows = B * S
        dev = torch.device(device)
        self.mask = torch.ones(rows, dtype=torch.uint8, device=dev)
        self.tokens = torch.full((rows,), -1, dtype=torch.int32, device=dev)
        self.conf = torch.full((rows,), float("nan"), dtype=torch.float32, device=dev)
        self.commit = torch.zeros(rows, dtype=torch.uint8, device=dev)
        self.o = torch.empty((B, S, H_q, d), dtype=torch.float32, device=dev)
        self.lse = torch.empty((B, H_q, S), dtype=torch.float32, device=dev)
        self.ws_attn = torch.empty(api.attn_workspace_bytes(B, S, H_q, H_kv, d), dtype=torch.uint8,
                                   device=dev)
        self.ws_unmask = torch.empty(api.unmask_workspace_bytes(rows, V), dtype=torch.uint8,
                                     device=dev)
        self.mask_host = torch.empty(rows, dtype=torch.uint8).pin_memory()
        self.commit_step = np.full(rows, -1, dtype=np.int64)
        self.per_step = []

    def reset(self):
        self.mask.fill_(1)
        self.tokens.fill_(-1)
        self.commit_step[:] = -1
        self.per_step = []

    def step(self, inp):
        """One denoise step; returns the number of positions still masked."""
        api.attn_step(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["k_blk"], inp["v_blk"],
                      inp["prefix_len"], inp["prefix_offset"], o=self.o, lse=self.lse,
                      workspace=self.ws_attn, stream=self.stream)
        api.unmask(inp["logits"], self.mask, self.gamma, block_S=self.S,
                   commit_at_least_one=self.fallback, tokens_out=self.tokens,
                   conf_out=self.conf, commit_out=self.commit, mask_out=self.mask,
                   workspace=self.ws_unmask, stream=self.stream)
        self.mask_host.copy_(self.mask, non_blocking=True)
        (self.stream or torch.cuda.current_stream(self.mask.device)).synchronize()
        m = self.mask_host.numpy().astype(bool)
        t = len(self.per_step)
        prev = self.commit_step < 0
        newly = prev & ~m
        self.commit_step[newly] = t
        self.per_step.append(int(newly.sum()))
        return int(m.sum())

    def commit_block(self, cache, k_clean, v_clean, prefix_capacity, seq_mask=None):
        """Append the committed block's clean K/V [B,S,H_kv,d] to the prefix
        cache in `cache` (k_prefix, v_prefix, prefix_len, prefix_offset);
        prefix_len grows by S for every selected sequence."""
        api.kv_append(cache["k_prefix"], cache["v_prefix"], k_clean, v_clean, cache["prefix_len"],
                      cache["prefix_offset"], prefix_capacity, seq_mask=seq_mask,
                      stream=self.stream)

    def run(self, step_inputs, T):
        """Run up to T steps; stop when every position is committed."""
        steps = 0
        for t in range(T):
            remaining = self.step(step_inputs(t))
            steps += 1
            if remaining == 0:
                break
        return steps
