"""GPU parity of the block refinement loop (Algorithm 1's inner loop).

Each step of the GPU loop (bd_attn_step + bd_unmask with the per-block
fallback, mask updated in place) is compared with the float64 oracle given the
same input mask (teacher forcing: a row whose confidence lies within 1e-6 of
gamma may legitimately differ and is excluded, as in the unmask tests). Loop
invariants ("Technical summary: Nemotron-TwoTower", Generation process): the
masked set only shrinks, committed tokens are final, and with the fallback
every unfinished block commits at least one position per step, so a block of
S positions finishes within S steps.
"""

import numpy as np
import pytest
import torch

from block_diffusion_lm_bd_b200 import workloads
from block_diffusion_lm_bd_b200.loop import BlockLoop
from oracle.attention import block_attention
from oracle.unmask import confidence_unmask
from _util import ATTN_TOL, attn_err, compare_unmask, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _inputs(w, step, base):
    inp = dict(base)
    inp.update(workloads.attention_inputs(w, device=DEV, step=step, block_only=True))
    inp["logits"] = workloads.logits(w, device=DEV, step=step)
    return inp


def _run_and_check(w, T, check_steps, check_attn_step0=False):
    base = workloads.attention_inputs(w, device=DEV)
    loop = BlockLoop(w.B, w.S, w.H_q, w.H_kv, w.d, w.V, w.gamma, DEV,
                     commit_at_least_one=w.commit_at_least_one)
    rows = w.B * w.S
    prev_mask = np.ones(rows, dtype=bool)
    tokens_ref = np.full(rows, -1, dtype=np.int64)
    for t in range(T):
        inp = _inputs(w, t, base)
        mask_in = loop.mask.clone()
        remaining = loop.step(inp)
        if t == 0 and check_attn_step0:
            ro, _ = block_attention(inp["q"], base["k_prefix"], base["v_prefix"], inp["k_blk"],
                                    inp["v_blk"], base["prefix_len_host"], base["prefix_offset_host"])
            err, _ = attn_err(to_np(loop.o), ro)
            assert err <= ATTN_TOL[w.dtype], err
        m_in = mask_in.cpu().numpy().astype(bool)
        m_out = loop.mask.cpu().numpy().astype(bool)
        commit = loop.commit.cpu().numpy().astype(bool)
        # invariants
        assert not (m_out & ~m_in).any(), "a committed position was re-masked"
        assert (m_out == (m_in & ~commit)).all()
        for blk in range(w.B):
            sl = slice(blk * w.S, (blk + 1) * w.S)
            if m_in[sl].any():
                assert commit[sl].sum() >= 1, f"step {t}: unfinished block {blk} committed nothing"
        if t < check_steps:
            ref = confidence_unmask(inp["logits"].cpu().numpy(), m_in, w.gamma, block_S=w.S,
                                    commit_at_least_one=w.commit_at_least_one)
            res = {"tokens": loop.tokens.clone(), "conf": loop.conf.clone(), "commit": loop.commit}
            # tokens / conf of rows masked at this step were written by this step
            compare_unmask(res, ref, inp["logits"].cpu().numpy(), m_in, w.gamma, w.S,
                           w.commit_at_least_one)
            tokens_ref[ref["commit"]] = ref["tokens"][ref["commit"]]
        prev_mask = m_out
        if remaining == 0:
            break
    return loop, t + 1, prev_mask


def test_small_loop_matches_oracle_every_step():
    w = workloads.WORKLOADS[4].with_(B=8, prefix_len=300, V=4096)
    loop, steps, mask = _run_and_check(w, T=16, check_steps=16, check_attn_step0=True)
    assert not mask.any() and steps <= w.S
    assert sum(loop.per_step) == w.B * w.S
    assert (loop.tokens.cpu().numpy() >= 0).all()


def test_full_size_loop_invariants_and_first_steps():
    w = workloads.WORKLOADS[4]
    loop, steps, mask = _run_and_check(w, T=w.steps, check_steps=2)
    assert not mask.any(), "with the fallback every block finishes within T = S steps"
    assert steps <= w.steps
    assert sum(loop.per_step) == w.B * w.S
    assert (loop.commit_step >= 0).all()
    print(f"loop: {steps} steps, committed per step {loop.per_step}, "
          f"tokens per step {w.B * w.S / steps:.1f}")


def test_commit_block_appends_to_the_prefix_cache():
    """Algorithm 1's tail: after the loop, the block's clean K/V join the prefix
    cache (bit-exact against the oracle); the next step's attention then reads
    a prefix longer by S."""
    from oracle.kv_cache import kv_append

    w = workloads.WORKLOADS[4].with_(B=4, prefix_len=200, V=4096)
    base = workloads.attention_inputs(w, device=DEV, pad_rows=w.S)
    cap = (base["prefix_offset"][1:] - base["prefix_offset"][:-1]).contiguous()
    loop = BlockLoop(w.B, w.S, w.H_q, w.H_kv, w.d, w.V, w.gamma, DEV, commit_at_least_one=True)
    steps = loop.run(lambda t: _inputs(w, t, base), w.steps)
    assert steps <= w.S and not loop.mask.any()
    g = torch.Generator(device=DEV).manual_seed(77)
    kc = torch.randn(w.B, w.S, w.H_kv, w.d, device=DEV, generator=g).to(w.dtype)
    vc = torch.randn(w.B, w.S, w.H_kv, w.d, device=DEV, generator=g).to(w.dtype)
    ref = kv_append(base["k_prefix"], base["v_prefix"], kc, vc, base["prefix_len"],
                    base["prefix_offset"][:w.B], cap)
    loop.commit_block(base, kc, vc, cap)
    torch.cuda.synchronize()
    assert (base["k_prefix"].cpu().view(torch.int16).numpy() == ref[0]).all()
    assert (base["v_prefix"].cpu().view(torch.int16).numpy() == ref[1]).all()
    assert base["prefix_len"].cpu().tolist() == [200 + w.S] * w.B
