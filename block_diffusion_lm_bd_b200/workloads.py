"""Seeded synthetic inputs for the denoise step.

This module only draws random numbers and lays them out; it holds none of the
step's arithmetic. Both the CUDA path and the float64 oracle consume what it
returns (the oracle gets host copies of the very same tensors).

The five workloads stand in for the sizes the source pages talk about: block
sizes S = 16 and 32 ("Technical summary: Nemotron-TwoTower", §Training and
conditioning, curriculum bullet and §Main results, block-size sensitivity;
"Nemotron-Labs Diffusion", 32-token FastDiffuser blocks), contexts up to 262k
tokens ("Training Hybrid Block Diffusion Language Models with Partial
Bidirectionality", §Results, 65K and 262K-token throughput) and a 131072-token
vocabulary. No dataset, prompt or model weight is used.

Value recipes (read from the workload list; "N(0,2)" is read as variance 2):
  0 tiny fp32      q,k,v ~ N(0,1) fp32; logits N(0,1) + spike U(0,12)
  1 bf16 decode    q,k,v ~ N(0,1)/sqrt(2) -> bf16; logits N(0,2) + spike U(0,16)
  2 ragged S=32    as 1; L_b ~ U{1024..32768}; masked fraction ~ U(0.2,1.0)
  3 long context   q,k,v ~ N(0,1) -> bf16; one sequence, L = 262144
  4 block loop     as 1, B = 64, L = 8192; q/k_blk/v_blk/logits redrawn per step
bf16 tensors are drawn in fp32 and rounded to nearest-even bf16.
Seeds: 20261202 + 1000 * workload index (+ step for the loop).
"""

import math
from dataclasses import dataclass, field, replace

import torch

SEED_BASE = 20261202


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    H_q: int
    H_kv: int
    d: int
    S: int
    V: int
    gamma: float
    dtype: torch.dtype
    qkv_std: float
    logit_std: float
    spike_max: float
    prefix_len: int = 0            # fixed prefix length (if lens is None)
    prefix_range: tuple = None     # (lo, hi) inclusive, drawn per sequence
    masked: str = "all"            # "all", "count:<n>", "fraction:<lo>,<hi>"
    steps: int = 1                 # > 1: the block refinement loop
    commit_at_least_one: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def g(self):
        return self.H_q // self.H_kv

    def seed(self, step=0):
        return SEED_BASE + 1000 * self.index + step

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    0: Workload(0, "tiny fp32", B=1, H_q=8, H_kv=2, d=64, S=16, V=1024, gamma=0.9,
                dtype=torch.float32, qkv_std=1.0, logit_std=1.0, spike_max=12.0,
                prefix_len=256, masked="count:8"),
    1: Workload(1, "bf16 decode step", B=8, H_q=32, H_kv=8, d=128, S=16, V=131072,
                gamma=0.9, dtype=torch.bfloat16, qkv_std=1 / math.sqrt(2),
                logit_std=math.sqrt(2), spike_max=16.0, prefix_len=4096, masked="all"),
    2: Workload(2, "bf16 ragged prefixes S=32", B=32, H_q=32, H_kv=8, d=128, S=32,
                V=131072, gamma=0.95, dtype=torch.bfloat16, qkv_std=1 / math.sqrt(2),
                logit_std=math.sqrt(2), spike_max=16.0, prefix_range=(1024, 32768),
                masked="fraction:0.2,1.0"),
    3: Workload(3, "long-context single sequence", B=1, H_q=32, H_kv=8, d=128, S=16,
                V=131072, gamma=0.9, dtype=torch.bfloat16, qkv_std=1.0,
                logit_std=math.sqrt(2), spike_max=16.0, prefix_len=262144, masked="all"),
    4: Workload(4, "full block loop", B=64, H_q=32, H_kv=8, d=128, S=16, V=131072,
                gamma=0.9, dtype=torch.bfloat16, qkv_std=1 / math.sqrt(2),
                logit_std=math.sqrt(2), spike_max=16.0, prefix_len=8192, masked="all",
                steps=16, commit_at_least_one=True),
    # LM head fused with unmasking at the decode step: the 128 masked rows of
    # the decode-step workload, hidden size D, its vocabulary and logit law
    5: Workload(5, "LM head + unmask, decode step", B=8, H_q=32, H_kv=8, d=128, S=16,
                V=131072, gamma=0.9, dtype=torch.bfloat16, qkv_std=1 / math.sqrt(2),
                logit_std=math.sqrt(2), spike_max=16.0, prefix_len=4096, masked="all",
                extra={"D": 4096}),
    # one Mamba-2 layer's block-local bidirectional scan for the loop
    # workload's 64 sequences (B=64, S=16): 64 heads of 64 channels, state 128,
    # 8 B/C groups
    6: Workload(6, "block-local bidirectional Mamba scan", B=64, H_q=32, H_kv=8, d=128, S=16,
                V=131072, gamma=0.9, dtype=torch.float32, qkv_std=1.0,
                logit_std=math.sqrt(2), spike_max=16.0, prefix_len=8192, masked="all",
                extra={"H": 64, "P": 64, "N": 128, "G": 8}),
}


def _cpu_gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _dev_gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def prefix_lengths(w: Workload, seed=None):
    """Per-sequence prefix lengths (CPU int64 tensor [B])."""
    if w.prefix_range is None:
        return torch.full((w.B,), w.prefix_len, dtype=torch.int64)
    lo, hi = w.prefix_range
    g = _cpu_gen(w.seed() if seed is None else seed)
    return torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64)


def _normal(shape, std, dtype, gen, device):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def attention_inputs(w: Workload, device="cpu", step=0, lens=None, pad_rows=0,
                     block_only=False):
    """Inputs of one attention step.

    Returns a dict with q [B,S,H_q,d], k_prefix/v_prefix [R,H_kv,d] (packed
    rows, sequence b at rows prefix_offset[b] .. + prefix_len[b]),
    k_blk/v_blk [B,S,H_kv,d], prefix_len int32 [B], prefix_offset int64 [B+1]
    and the host copies of the lengths. pad_rows > 0 leaves that many unused
    (random) rows after each sequence's prefix, which a correct kernel never
    reads. block_only=True redraws only q, k_blk, v_blk (a loop step).
    """
    if lens is None:
        lens = prefix_lengths(w)
    lens = torch.as_tensor(lens, dtype=torch.int64).cpu()
    B = lens.numel()
    span = lens + pad_rows
    offset = torch.zeros(B + 1, dtype=torch.int64)
    offset[1:] = torch.cumsum(span, 0)
    R = int(offset[-1])
    gen = _dev_gen(device, w.seed(step) + 500)
    out = {}
    out["q"] = _normal((B, w.S, w.H_q, w.d), w.qkv_std, w.dtype, gen, device)
    out["k_blk"] = _normal((B, w.S, w.H_kv, w.d), w.qkv_std, w.dtype, gen, device)
    out["v_blk"] = _normal((B, w.S, w.H_kv, w.d), w.qkv_std, w.dtype, gen, device)
    if not block_only:
        pgen = _dev_gen(device, w.seed() + 700)
        out["k_prefix"] = _normal((max(R, 1), w.H_kv, w.d), w.qkv_std, w.dtype, pgen, device)
        out["v_prefix"] = _normal((max(R, 1), w.H_kv, w.d), w.qkv_std, w.dtype, pgen, device)
        out["prefix_len"] = lens.to(torch.int32).to(device)
        out["prefix_offset"] = offset.to(device)
        out["prefix_len_host"] = lens.clone()
        out["prefix_offset_host"] = offset.clone()
        out["total_rows"] = max(R, 1)
    return out


def lmhead_inputs(w: Workload, device="cpu", step=0, rows=None, D=None, V=None):
    """Hidden states bf16 [rows, D] ~ N(0, 1) and an LM head bf16 [V, D] whose
    logits follow the unmask workloads' law: W ~ N(0, logit_std^2 / D) gives
    logits ~ N(0, logit_std^2), and every row r gets one spike U(0, spike_max)
    at a uniformly drawn token t_r by adding (s_r / |h_r|^2) h_r to W[t_r]
    (rows drawing the same token share its row)."""
    rows = w.B * w.S if rows is None else rows
    D = w.extra.get("D", 4096) if D is None else D
    V = w.V if V is None else V
    gen = _dev_gen(device, w.seed(step) + 1100)
    h = torch.randn((rows, D), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    W = torch.randn((V, D), generator=gen, device=device, dtype=torch.float32)
    W.mul_(w.logit_std / math.sqrt(D))
    cg = _cpu_gen(w.seed(step) + 1300)
    pos = torch.randint(0, V, (rows,), generator=cg)
    amp = torch.rand(rows, generator=cg, dtype=torch.float32) * w.spike_max
    hf = h.float()
    coef = (amp.to(device) / (hf * hf).sum(1)).unsqueeze(1)
    W.index_add_(0, pos.to(device), coef * hf)
    return h, W.to(torch.bfloat16)


def mamba_inputs(w: Workload, device="cpu", step=0, B=None, S=None, H=None, P=None, N=None,
                 G=None):
    """Inputs of one Mamba-2 layer's block scan, float32: x, B, C ~ N(0, 1);
    step sizes log-uniform in [0.001, 0.1] (after the softplus); decays
    A = -U(1, 16); skip D ~ U(0.5, 1.5); boundary state h0 ~ N(0, 1)."""
    e = w.extra
    B = w.B if B is None else B
    S = w.S if S is None else S
    H = e.get("H", 64) if H is None else H
    P = e.get("P", 64) if P is None else P
    N = e.get("N", 128) if N is None else N
    G = e.get("G", 8) if G is None else G
    gen = _dev_gen(device, w.seed(step) + 1500)

    def normal(*shape):
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)

    def uniform(lo, hi, *shape):
        return lo + (hi - lo) * torch.rand(shape, generator=gen, device=device, dtype=torch.float32)

    out = {"x": normal(B, S, H, P),
           "dt": torch.exp(uniform(math.log(1e-3), math.log(1e-1), B, S, H)),
           "B_fwd": normal(B, S, G, N), "C_fwd": normal(B, S, G, N),
           "dt_rev": torch.exp(uniform(math.log(1e-3), math.log(1e-1), B, S, H)),
           "B_rev": normal(B, S, G, N), "C_rev": normal(B, S, G, N),
           "A_fwd": -uniform(1.0, 16.0, H), "A_rev": -uniform(1.0, 16.0, H),
           "D_skip": uniform(0.5, 1.5, H), "h0": normal(B, H, P, N)}
    return out


MAMBA_ARGS = ("x", "dt", "B_fwd", "C_fwd", "dt_rev", "B_rev", "C_rev", "A_fwd", "A_rev", "D_skip",
              "h0")


def initial_mask(w: Workload, rows=None, seed=None):
    """Mask of still-[MASK] block positions (CPU uint8 [B*S])."""
    B, S = w.B, w.S
    g = _cpu_gen((w.seed() if seed is None else seed) + 100)
    m = torch.zeros(B, S, dtype=torch.uint8)
    if w.masked == "all":
        m[:] = 1
    elif w.masked.startswith("count:"):
        n = int(w.masked.split(":")[1])
        for b in range(B):
            m[b, torch.randperm(S, generator=g)[:n]] = 1
    elif w.masked.startswith("fraction:"):
        lo, hi = (float(t) for t in w.masked.split(":")[1].split(","))
        f = lo + (hi - lo) * torch.rand(B, generator=g, dtype=torch.float64)
        for b in range(B):
            n = max(1, int(round(float(f[b]) * S)))
            m[b, torch.randperm(S, generator=g)[:n]] = 1
    else:
        raise ValueError(w.masked)
    return m.reshape(-1)


def logits(w: Workload, device="cpu", step=0, rows=None):
    """Full-vocabulary logits [rows, V] fp32: N(0, logit_std^2) plus one spike
    U(0, spike_max) added at a uniformly drawn token of every row."""
    rows = w.B * w.S if rows is None else rows
    gen = _dev_gen(device, w.seed(step) + 900)
    x = torch.randn((rows, w.V), generator=gen, device=device, dtype=torch.float32)
    x.mul_(w.logit_std)
    cg = _cpu_gen(w.seed(step) + 300)
    pos = torch.randint(0, w.V, (rows,), generator=cg)
    amp = torch.rand(rows, generator=cg, dtype=torch.float32) * w.spike_max
    x[torch.arange(rows, device=device), pos.to(device)] += amp.to(device)
    return x
