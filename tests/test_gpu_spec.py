"""GPU parity of self-speculative verification: the causal-in-block attention
(bd_attn_step_ex with BD_ATTN_BLOCK_CAUSAL, tensor-core and CUDA-core paths)
against the oracle's causal_block_attention, and bd_spec_verify's commit rule
against verify_commit (bit-exact tokens, accepted lengths and commits; blocks
holding a row whose top-two logits are closer than 1e-6 are left out and
counted, as in the unmask tests)."""

import numpy as np
import pytest
import torch

from block_diffusion_lm_bd_b200 import api, workloads
from oracle.spec import causal_block_attention, verify_commit
from oracle.unmask import top2_gap
from _util import ATTN_TOL, LSE_TOL, attn_err, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _attn(inp, causal=True):
    o, lse = api.attn_step(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["k_blk"], inp["v_blk"],
                           inp["prefix_len"], inp["prefix_offset"], block_causal=causal)
    torch.cuda.synchronize()
    assert api.get_device_status() == 0
    return o, lse


@pytest.mark.parametrize("dtype,B,S,H_q,H_kv,d,lens", [
    (torch.bfloat16, 3, 16, 32, 8, 128, [0, 300, 1000]),       # q rows spread over quadrants
    (torch.bfloat16, 2, 32, 32, 8, 128, [129, 0]),             # 128 packed rows
    (torch.bfloat16, 2, 64, 2, 1, 128, [0, 77]),               # S = 64 block tile
    (torch.bfloat16, 2, 16, 8, 2, 64, [10, 513]),              # d = 64: CUDA-core path
    (torch.float32, 2, 16, 8, 2, 64, [0, 260]),                # fp32: CUDA-core path
    (torch.float32, 1, 40, 4, 4, 128, [100]),                  # S = 40 over two key chunks
])
def test_causal_attention_matches_oracle(dtype, B, S, H_q, H_kv, d, lens):
    base = workloads.WORKLOADS[0 if dtype == torch.float32 else 1]
    w = base.with_(B=B, S=S, H_q=H_q, H_kv=H_kv, d=d)
    inp = workloads.attention_inputs(w, device=DEV, lens=lens)
    o, lse = _attn(inp)
    ro, rl = causal_block_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["k_blk"],
                                    inp["v_blk"], inp["prefix_len_host"], inp["prefix_offset_host"])
    err, raw = attn_err(to_np(o), ro)
    assert err <= ATTN_TOL[dtype], (err, raw)
    assert float(np.abs(to_np(lse) - rl).max()) <= LSE_TOL[dtype]


def test_causal_flag_off_is_the_bidirectional_step():
    w = workloads.WORKLOADS[1].with_(B=2)
    inp = workloads.attention_inputs(w, device=DEV, lens=[500, 70])
    o1, _ = _attn(inp, causal=False)
    o2, l2 = api.attn_step(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["k_blk"], inp["v_blk"],
                           inp["prefix_len"], inp["prefix_offset"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_full_size_decode_step_causal_sampled_sequence():
    w = workloads.WORKLOADS[1]
    inp = workloads.attention_inputs(w, device=DEV)
    o, lse = _attn(inp)
    b = 5
    one = {k: inp[k][b:b + 1] for k in ("q", "k_blk", "v_blk")}
    off = int(inp["prefix_offset_host"][b])
    L = int(inp["prefix_len_host"][b])
    ro, rl = causal_block_attention(one["q"], inp["k_prefix"][off:off + L], inp["v_prefix"][off:off + L],
                                    one["k_blk"], one["v_blk"], [L], [0])
    err, raw = attn_err(to_np(o[b:b + 1]), ro)
    assert err <= ATTN_TOL[torch.bfloat16], (err, raw)


def _drafts(tokens_ref, S, rng, p_wrong):
    d = tokens_ref.copy()
    wrong = rng.random(d.size) < p_wrong
    d[wrong] = (d[wrong] + 1 + rng.integers(0, 5, wrong.sum())) % 1_000_000
    return d


@pytest.mark.parametrize("rows,V,S,p_wrong", [
    (128, 131072, 16, 0.1),
    (64, 4096, 8, 0.3),
    (40, 1000, 1, 0.5),
    (256, 20000, 64, 0.02),
])
def test_verify_commit_matches_oracle(rows, V, S, p_wrong):
    w = workloads.WORKLOADS[1].with_(V=V)
    logits = workloads.logits(w, device=DEV, rows=rows)
    x = logits.cpu().numpy()
    ar = np.argmax(x, axis=1)
    rng = np.random.default_rng(rows + S)
    draft = _drafts(ar, S, rng, p_wrong)
    res = api.spec_verify(logits, torch.tensor(draft, dtype=torch.int32, device=DEV), S)
    torch.cuda.synchronize()
    assert api.get_device_status() == 0
    ref = verify_commit(x, draft, S)
    gap = top2_gap(x)
    ok_blocks = [b for b in range(rows // S) if (gap[b * S:(b + 1) * S] > 1e-6).all()]
    assert len(ok_blocks) >= (rows // S) * 0.95
    n = res["n_accept"].cpu().numpy()
    com = res["commit"].cpu().numpy().astype(bool)
    tok = res["tokens"].cpu().numpy()
    for b in ok_blocks:
        sl = slice(b * S, (b + 1) * S)
        assert n[b] == ref["n_accept"][b]
        assert (com[sl] == ref["commit"][sl]).all()
        assert (tok[sl] == ref["tokens"][sl]).all()


def test_verify_all_accepted_and_none_accepted():
    w = workloads.WORKLOADS[1].with_(V=2048)
    logits = workloads.logits(w, device=DEV, rows=32)
    ar = np.argmax(logits.cpu().numpy(), axis=1)
    draft = ar.copy()
    draft[16:] = (ar[16:] + 1) % 2048      # block 0 all right, block 1 all wrong
    res = api.spec_verify(logits, torch.tensor(draft, dtype=torch.int32, device=DEV), 16)
    torch.cuda.synchronize()
    assert res["n_accept"].cpu().tolist() == [16, 0]
    com = res["commit"].cpu().numpy().astype(bool)
    assert com[:16].all() and com[16] and not com[17:].any()
