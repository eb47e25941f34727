"""GPU parity of bd_kv_append (committing a block into the prefix cache)
against the oracle: a byte copy, so the cache and the lengths must match bit
for bit. Also: a refused sequence leaves everything of it untouched, and the
next block's attention over the appended cache matches the oracle over the
concatenated layout."""

import numpy as np
import pytest
import torch

from block_diffusion_lm_bd_b200 import api, workloads
from oracle.attention import block_attention
from oracle.kv_cache import kv_append as kv_append_ref
from _util import ATTN_TOL, LSE_TOL, attn_err, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _bits(t):
    t = t.detach().cpu()
    return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.numpy()


def _setup(B, S, H_kv, d, dtype, lens, cap, seed=0):
    g = torch.Generator(device=DEV).manual_seed(seed)
    rows = B * cap
    kp = torch.randn(rows, H_kv, d, device=DEV, generator=g).to(dtype)
    vp = torch.randn(rows, H_kv, d, device=DEV, generator=g).to(dtype)
    kn = torch.randn(B, S, H_kv, d, device=DEV, generator=g).to(dtype)
    vn = torch.randn(B, S, H_kv, d, device=DEV, generator=g).to(dtype)
    L = torch.tensor(lens, dtype=torch.int32, device=DEV)
    off = torch.arange(B, dtype=torch.int64, device=DEV) * cap
    capa = torch.full((B,), cap, dtype=torch.int64, device=DEV)
    return kp, vp, kn, vn, L, off, capa


def _check(kp, vp, kn, vn, L, off, capa, mask=None, expect_status=0):
    ref = kv_append_ref(kp, vp, kn, vn, L, off, capa, seq_mask=mask)
    api.kv_append(kp, vp, kn, vn, L, off, capa, seq_mask=mask)
    assert api.get_device_status() == expect_status
    assert np.array_equal(_bits(kp), ref[0])
    assert np.array_equal(_bits(vp), ref[1])
    assert L.cpu().numpy().tolist() == ref[2].tolist()
    return ref[3]


@pytest.mark.parametrize("dtype,B,S,H_kv,d,lens,cap", [
    (torch.bfloat16, 5, 16, 8, 128, [0, 7, 100, 33, 1], 128),
    (torch.bfloat16, 3, 1, 1, 64, [0, 5, 9], 12),
    (torch.float32, 4, 32, 2, 64, [31, 0, 64, 2], 96),
    (torch.float32, 2, 64, 4, 128, [0, 64], 128),
    (torch.bfloat16, 300, 16, 2, 64, list(range(0, 300)), 320),
])
def test_append_matches_oracle_bit_for_bit(dtype, B, S, H_kv, d, lens, cap):
    args = _setup(B, S, H_kv, d, dtype, lens, cap)
    assert _check(*args) == []


def test_seq_mask_selects_sequences():
    args = _setup(6, 16, 8, 128, torch.bfloat16, [3, 4, 5, 6, 7, 8], 64, seed=1)
    mask = torch.tensor([1, 0, 0, 1, 1, 0], dtype=torch.uint8, device=DEV)
    assert _check(*args, mask=mask) == []


def test_overflowing_sequence_is_skipped_and_reported():
    # sequence 1 would spill into sequence 2's rows; sequence 3 would leave the array
    kp, vp, kn, vn, L, off, capa = _setup(4, 16, 2, 64, torch.bfloat16, [10, 20, 0, 30], 32, seed=2)
    before = (_bits(kp).copy(), L.cpu().clone())
    skipped = _check(kp, vp, kn, vn, L, off, capa, expect_status=5)
    assert skipped == [1, 3]
    assert L.cpu().tolist() == [26, 20, 16, 30]
    assert np.array_equal(_bits(kp)[32:64], before[0][32:64])  # sequence 1 untouched


def test_repeated_appends_grow_the_prefix_block_by_block():
    kp, vp, kn, vn, L, off, capa = _setup(3, 16, 8, 128, torch.bfloat16, [0, 5, 40], 96, seed=3)
    for step in range(3):
        g = torch.Generator(device=DEV).manual_seed(100 + step)
        kn = torch.randn(kn.shape, device=DEV, generator=g).to(kn.dtype)
        vn = torch.randn(vn.shape, device=DEV, generator=g).to(vn.dtype)
        assert _check(kp, vp, kn, vn, L, off, capa) == []
    assert L.cpu().tolist() == [48, 53, 88]


def test_next_block_attention_over_appended_cache():
    """Algorithm 1: after the commit, the next block attends to old prefix ++
    committed block. GPU append then GPU attention, against the oracle on the
    concatenated layout."""
    w = workloads.WORKLOADS[1].with_(B=4)
    S = w.S
    inp = workloads.attention_inputs(w, device=DEV, lens=[100, 0, 1000, 257], pad_rows=S)
    lens = inp["prefix_len_host"].tolist()
    off = inp["prefix_offset"][:4].contiguous()
    cap = (inp["prefix_offset"][1:] - inp["prefix_offset"][:-1]).contiguous()
    g = torch.Generator(device=DEV).manual_seed(9)
    kc = torch.randn(4, S, w.H_kv, w.d, device=DEV, generator=g).to(torch.bfloat16)
    vc = torch.randn(4, S, w.H_kv, w.d, device=DEV, generator=g).to(torch.bfloat16)
    old_k, old_v = inp["k_prefix"].clone(), inp["v_prefix"].clone()
    api.kv_append(inp["k_prefix"], inp["v_prefix"], kc, vc, inp["prefix_len"], off, cap)
    assert api.get_device_status() == 0
    nxt = workloads.attention_inputs(w, device=DEV, step=1, block_only=True)
    o, lse = api.attn_step(nxt["q"], inp["k_prefix"], inp["v_prefix"], nxt["k_blk"], nxt["v_blk"],
                           inp["prefix_len"], off)
    torch.cuda.synchronize()
    ks, vs, offs = [], [], [0]
    for b in range(4):
        o0 = int(inp["prefix_offset_host"][b])
        ks.append(torch.cat([old_k[o0:o0 + lens[b]], kc[b]]).cpu())
        vs.append(torch.cat([old_v[o0:o0 + lens[b]], vc[b]]).cpu())
        offs.append(offs[-1] + lens[b] + S)
    ro, rl = block_attention(nxt["q"], torch.cat(ks), torch.cat(vs), nxt["k_blk"], nxt["v_blk"],
                             [x + S for x in lens], offs[:-1])
    err, raw = attn_err(to_np(o), ro)
    assert err <= ATTN_TOL[torch.bfloat16], (err, raw)
    assert float(np.abs(to_np(lse) - rl).max()) <= LSE_TOL[torch.bfloat16]
