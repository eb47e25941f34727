"""Planted mistakes in the oracle must be caught by its pins.

Each mutant is a one-line change to a copy of the oracle's source, made here
on the CPU (the oracle on disk is untouched). The pin tests of
test_oracle_attention.py / test_oracle_unmask.py are then run against the
mutated copy; at least one of them has to fail, or the pins would not protect
against that kind of mistake (a dropped term, a wrong sign or index, a wrong
operand, an off-by-one).
"""

import importlib.util
import inspect
import os

import pytest

import test_oracle_attention as TA
import test_oracle_kv_cache as TK
import test_oracle_lmhead as TL
import test_oracle_mamba as TM
import test_oracle_spec as TS
import test_oracle_unmask as TU

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_mutant(relpath, old, new, name):
    src = open(os.path.join(ROOT, relpath)).read()
    assert src.count(old) >= 1, f"mutation site not found: {old!r}"
    src = src.replace(old, new)
    spec = importlib.util.spec_from_loader(name, loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


def _collect(module):
    """All pin tests of a module as (callable, list-of-arg-dicts)."""
    out = []
    for nm, fn in inspect.getmembers(module, inspect.isfunction):
        if not nm.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if params:
            argnames = params[0].args[0]
            values = params[0].args[1]
            names = [a.strip() for a in argnames.split(",")]
            calls = []
            for v in values:
                v = v if len(names) > 1 else (v,)
                calls.append(dict(zip(names, v)))
            out.append((fn, calls))
        else:
            out.append((fn, [{}]))
    return out


def _some_pin_fails(module, patches, monkeypatch):
    for attr, val in patches.items():
        monkeypatch.setattr(module, attr, val)
    for fn, calls in _collect(module):
        for kw in calls:
            try:
                fn(**kw)
            except Exception:
                return True
    return False


ATTN_MUTANTS = [
    ("scale 1/d", "scale = 1.0 / np.sqrt(d)", "scale = 1.0 / d"),
    ("interleaved GQA", "    return h // g\n", "    return h % H_kv\n"),
    ("block keys causal", "k_blk[b, :, kv, :]], axis=0)", "k_blk[b, :1, kv, :]], axis=0)"),
    ("drop prefix", "[k_prefix[off:off + L, kv, :], k_blk", "[k_prefix[off:off, kv, :], k_blk"),
    ("prefix off by one", "k_prefix[off:off + L, kv, :], k_blk[b, :, kv, :]",
     "k_prefix[off + 1:off + L + 1, kv, :], k_blk[b, :, kv, :]"),
    ("no normalisation", "o = (p @ V) / l", "o = (p @ V)"),
    ("lse without max", "lse = mx[:, 0] + np.log(l[:, 0])", "lse = np.log(l[:, 0])"),
    ("combine weights sign", "w = np.exp(lse_parts - M[None, :])", "w = np.exp(M[None, :] - lse_parts)"),
]


@pytest.mark.parametrize("mut", ATTN_MUTANTS, ids=[m[0] for m in ATTN_MUTANTS])
def test_attention_mutant_is_caught(mut, monkeypatch):
    name, old, new = mut
    mod = _load_mutant("oracle/attention.py", old, new, "mut_attn")
    patches = {"block_attention": mod.block_attention, "attend": mod.attend,
               "lse_combine": mod.lse_combine, "block_attention_rows": mod.block_attention_rows}
    assert _some_pin_fails(TA, patches, monkeypatch), f"no pin caught mutant {name!r}"


UNMASK_MUTANTS = [
    ("ties to highest id", "tok = int(np.flatnonzero(row == mx)[0])", "tok = int(np.flatnonzero(row == mx)[-1])"),
    (">= instead of >", "commit[r] = conf[r] > thr", "commit[r] = conf[r] >= thr"),
    ("no max shift in Z", "z = np.exp(row - mx).sum()", "z = np.exp(row).sum()"),
    ("fallback ties to last", "best = masked[int(np.flatnonzero(c == c.max())[0])]",
     "best = masked[int(np.flatnonzero(c == c.max())[-1])]"),
    ("fallback picks min", "c == c.max()", "c == c.min()"),
    ("mask not updated", '"mask_out": m & ~commit', '"mask_out": m'),
    ("unmasked rows scored", "        if not m[r]:\n            continue\n", ""),
]


@pytest.mark.parametrize("mut", UNMASK_MUTANTS, ids=[m[0] for m in UNMASK_MUTANTS])
def test_unmask_mutant_is_caught(mut, monkeypatch):
    name, old, new = mut
    mod = _load_mutant("oracle/unmask.py", old, new, "mut_unmask")
    patches = {"confidence_unmask": mod.confidence_unmask, "top2_gap": mod.top2_gap}
    assert _some_pin_fails(TU, patches, monkeypatch), f"no pin caught mutant {name!r}"


KV_MUTANTS = [
    ("append one row late", "lo = off[b] + L[b]\n", "lo = off[b] + L[b] + 1\n"),
    ("length not advanced", "        L[b] += S\n", ""),
    ("capacity not checked", "L[b] + S <= cap[b]", "True"),
    ("mask ignored", "        if not sel[b]:\n            continue\n", ""),
    ("K and V swapped", "        v[lo:lo + S] = vn[b]\n", "        v[lo:lo + S] = kn[b]\n"),
]


@pytest.mark.parametrize("mut", KV_MUTANTS, ids=[m[0] for m in KV_MUTANTS])
def test_kv_append_mutant_is_caught(mut, monkeypatch):
    name, old, new = mut
    mod = _load_mutant("oracle/kv_cache.py", old, new, "mut_kv")
    assert _some_pin_fails(TK, {"kv_append": mod.kv_append}, monkeypatch), \
        f"no pin caught mutant {name!r}"


LMHEAD_MUTANTS = [
    ("head not transposed", "return h @ _f64(w_vocab).T", "return h @ _f64(w_vocab)"),
    ("row list ignored", "        h = h[np.asarray(rows, dtype=np.int64)]\n", "        pass\n"),
    ("hidden scaled by 1/sqrt(D)", "return h @ _f64(w_vocab).T", "return (h @ _f64(w_vocab).T) / np.sqrt(h.shape[1])"),
    ("unmasked rows predicted", "    idx = np.flatnonzero(m)\n", "    idx = np.arange(m.shape[0])\n"),
]


@pytest.mark.parametrize("mut", LMHEAD_MUTANTS, ids=[m[0] for m in LMHEAD_MUTANTS])
def test_lmhead_mutant_is_caught(mut, monkeypatch):
    name, old, new = mut
    src = open(os.path.join(ROOT, "oracle/lmhead.py")).read()
    assert src.count(old) >= 1, old
    # the module imports confidence_unmask relatively: load it inside the package
    import oracle
    spec = importlib.util.spec_from_loader("oracle._mut_lmhead", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), "<mutant lmhead>", "exec"), mod.__dict__)
    patches = {"lmhead_logits": mod.lmhead_logits, "lmhead_unmask": mod.lmhead_unmask}
    assert _some_pin_fails(TL, patches, monkeypatch), f"no pin caught mutant {name!r}"


MAMBA_MUTANTS = [
    ("interleaved groups", "        g = h // hpg\n", "        g = h % G\n"),
    ("reverse scan starts from the boundary state", "        state = np.zeros_like(h0[h])\n", "        state = h0[h].copy()\n"),
    ("skip term dropped", " + Dskip[h] * x[t, h]", ""),
    ("decay after the input", "state = np.exp(dt[t, h] * A[h]) * state + dt[t, h] * np.outer(x[t, h], Bm[t, g])",
     "state = np.exp(dt[t, h] * A[h]) * (state + dt[t, h] * np.outer(x[t, h], Bm[t, g]))"),
    ("reverse uses forward step sizes", "np.exp(dt_r[t, h] * A_r[h])", "np.exp(dt[t, h] * A_r[h])"),
    ("reverse reads C instead of C_r", "y[t, h] += state @ C_r[t, g]", "y[t, h] += state @ Cm[t, g]"),
]


@pytest.mark.parametrize("mut", MAMBA_MUTANTS, ids=[m[0] for m in MAMBA_MUTANTS])
def test_mamba_mutant_is_caught(mut, monkeypatch):
    name, old, new = mut
    mod = _load_mutant("oracle/mamba.py", old, new, "mut_mamba")
    patches = {"block_scan": mod.block_scan, "batch_block_scan": mod.batch_block_scan}
    assert _some_pin_fails(TM, patches, monkeypatch), f"no pin caught mutant {name!r}"


SPEC_MUTANTS = [
    ("block keys not causal", "k_blk[b, :i + 1, kv]], axis=0)\n                V = np.concatenate([v_prefix[off:off + L, kv], v_blk[b, :i + 1, kv]]",
     "k_blk[b, :, kv]], axis=0)\n                V = np.concatenate([v_prefix[off:off + L, kv], v_blk[b, :, kv]]"),
    ("causal excludes the diagonal", "k_blk[b, :i + 1, kv]], axis=0)\n                V = np.concatenate([v_prefix[off:off + L, kv], v_blk[b, :i + 1, kv]]",
     "k_blk[b, :max(i, 1), kv]], axis=0)\n                V = np.concatenate([v_prefix[off:off + L, kv], v_blk[b, :max(i, 1), kv]]"),
    ("no correction token", "            commit[b * S + n] = True  # the autoregressive token at the first mismatch\n",
     "            pass\n"),
    ("ties to the highest id", "tokens[r] = int(np.flatnonzero(x[r] == x[r].max())[0])",
     "tokens[r] = int(np.flatnonzero(x[r] == x[r].max())[-1])"),
    ("accepts past a mismatch", "        commit[b * S:b * S + n] = True\n", "        commit[b * S:b * S + S] = True\n"),
]


@pytest.mark.parametrize("mut", SPEC_MUTANTS, ids=[m[0] for m in SPEC_MUTANTS])
def test_spec_mutant_is_caught(mut, monkeypatch):
    name, old, new = mut
    src = open(os.path.join(ROOT, "oracle/spec.py")).read()
    assert src.count(old) >= 1, old
    spec = importlib.util.spec_from_loader("oracle._mut_spec", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), "<mutant spec>", "exec"), mod.__dict__)
    patches = {"causal_block_attention": mod.causal_block_attention,
               "verify_commit": mod.verify_commit}
    assert _some_pin_fails(TS, patches, monkeypatch), f"no pin caught mutant {name!r}"


def test_unmutated_copy_passes_every_pin(monkeypatch):
    """Control: the loader itself does not make pins fail."""
    mod = _load_mutant("oracle/attention.py", "import numpy as np", "import numpy as np", "same_attn")
    patches = {"block_attention": mod.block_attention, "attend": mod.attend,
               "lse_combine": mod.lse_combine, "block_attention_rows": mod.block_attention_rows}
    assert not _some_pin_fails(TA, patches, monkeypatch)
    mod = _load_mutant("oracle/unmask.py", "import numpy as np", "import numpy as np", "same_unmask")
    assert not _some_pin_fails(TU, {"confidence_unmask": mod.confidence_unmask,
                                    "top2_gap": mod.top2_gap}, monkeypatch)
    mod = _load_mutant("oracle/kv_cache.py", "import numpy as np", "import numpy as np", "same_kv")
    assert not _some_pin_fails(TK, {"kv_append": mod.kv_append}, monkeypatch)
    mod = _load_mutant("oracle/mamba.py", "import numpy as np", "import numpy as np", "same_mamba")
    assert not _some_pin_fails(TM, {"block_scan": mod.block_scan,
                                    "batch_block_scan": mod.batch_block_scan}, monkeypatch)
