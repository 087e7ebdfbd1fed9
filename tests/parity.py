"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle,
compare with the tolerances of the spec.

Tolerances (bf16 inputs, fp32 accumulation, bf16 output):
  * O: max-abs <= 1e-2 AND relative Frobenius <= 5e-3 against the fp64 oracle;
  * lse: max-abs <= 2e-3 on rows with a finite lse; -inf rows must be -inf.
Where the oracle computes only sampled rows (full-size workloads), the same
bounds apply to those rows.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200.synth import Inputs

O_MAX_ABS = 1e-2
O_REL_FRO = 5e-3
LSE_MAX_ABS = 2e-3


def to_device(inp: Inputs, dev="cuda"):
    return dict(q=inp.q.to(dev), k=inp.k.to(dev), v=inp.v.to(dev),
                kv_lens=None if inp.kv_lens is None else inp.kv_lens.to(dev),
                sink=None if inp.sink is None else inp.sink.to(dev))


def run_gpu(inp: Inputs):
    t = to_device(inp)
    out, lse = binding.gqa_attention_fwd(t["q"], t["k"], t["v"], t["kv_lens"], t["sink"], scale=inp.scale,
                                         causal=inp.causal)
    err = binding.gqa_get_device_error()
    assert err == 0, "device error %d (%s)" % (err, binding.STATUS.get(err))
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def run_oracle(inp: Inputs):
    return oracle.attention(inp.q, inp.k, inp.v, inp.kv_lens, inp.sink, scale=inp.scale, causal=inp.causal)


def compare(o_gpu, l_gpu, o_ref, l_ref, what=""):
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    assert o_gpu.shape == o_ref.shape
    assert np.all(np.isfinite(o_gpu)), "%s: non-finite output" % what
    diff = np.abs(o_gpu - o_ref)
    max_abs = float(diff.max()) if diff.size else 0.0
    den = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o_gpu - o_ref)) / den if den > 0 else float(np.linalg.norm(o_gpu))
    assert max_abs <= O_MAX_ABS, "%s: O max-abs %.3g > %.1g" % (what, max_abs, O_MAX_ABS)
    assert rel <= O_REL_FRO, "%s: O rel-Frobenius %.3g > %.1g" % (what, rel, O_REL_FRO)
    if l_gpu is not None:
        l_gpu = np.asarray(l_gpu, np.float64)
        l_ref = np.asarray(l_ref, np.float64)
        fin = np.isfinite(l_ref)
        assert np.array_equal(np.isneginf(l_gpu), np.isneginf(l_ref)), "%s: -inf lse rows differ" % what
        if fin.any():
            lm = float(np.abs(l_gpu[fin] - l_ref[fin]).max())
            assert lm <= LSE_MAX_ABS, "%s: lse max-abs %.3g > %.1g" % (what, lm, LSE_MAX_ABS)
    return max_abs, rel


def sample_rows(B, Hq, Tq, n, seed=0):
    """Flat rows (b*Hq + h)*Tq + i: the first and last row of every head group
    plus a seeded random sample."""
    total = B * Hq * Tq
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(total, size=min(n, total), replace=False).tolist())
    for b in range(B):
        for h in (0, Hq - 1):
            rows.add((b * Hq + h) * Tq)
            rows.add((b * Hq + h) * Tq + Tq - 1)
    return np.array(sorted(rows), np.int64)
