"""A NaN inside the visible keys of a row makes that row NaN, as IEEE arithmetic
on the definition does, and leaves every other row untouched.

Padding past a sequence's length is masked and must never leak (the parity
tests fill it with NaN); a NaN in a key or value a row does see is a different
case: softmax(s) has a NaN score, or P V a NaN term, and the row's output and
its log-sum-exp are NaN.  The oracle computes the same thing in fp64.  Each
kernel family computes its row maxima and exponentials its own way (the
two-lane kernel with a NaN-propagating three-input max, the decode kernel's
transposed tiles, the wide kernel's 128-key tiles), so each is covered: the
set of NaN rows must equal the oracle's, and the other rows must agree within
the parity tolerances.

A NaN (or inf) in a V row inside the valid length reaches, besides the rows
that see the key, the rows of the same 128-key tile that mask it by causality
(their P is 0 there, and 0 * NaN is NaN), so the V cases use no causal mask.
"""
import numpy as np
import pytest
import torch

from gqa_attention_forward_flash_b200.synth import Workload, make_inputs

from parity import compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

CASES = {
    # two-lane kernel, dual-Q lanes (prefill): rows at or after the poisoned key
    "prefill_k": (Workload("nan_prefill", B=1, Hq=8, Hkv=2, Tq=300, Tkv=300, d=128, causal=True, seed=31),
                  "k", (0, 1, 77, 5)),
    # (non-causal: a V row that a causal row masks still meets it in the P V
    # product of the shared 128-key tile, as 0 * NaN)
    "prefill_v": (Workload("nan_prefill", B=1, Hq=8, Hkv=2, Tq=300, Tkv=300, d=128, seed=32),
                  "v", (0, 0, 200, 64)),
    # two-lane kernel, split-key lanes (short queries over a long cache)
    "short_q_k": (Workload("nan_short_q", B=2, Hq=32, Hkv=4, Tq=16, Tkv=2000, d=128, causal=True, seed=33),
                  "k", (1, 3, 1500, 0)),
    # swap-AB decode kernel
    "decode_k": (Workload("nan_decode", B=3, Hq=32, Hkv=4, Tq=1, Tkv=1500, d=128, seed=34), "k", (2, 1, 901, 100)),
    "decode_v": (Workload("nan_decode", B=3, Hq=32, Hkv=4, Tq=1, Tkv=1500, d=128, seed=35), "v", (0, 3, 12, 7)),
    # wide kernel (head dim 256)
    "d256_k": (Workload("nan_d256", B=2, Hq=16, Hkv=2, Tq=3, Tkv=1200, d=256, sigma=0.5, causal=True, seed=36),
               "k", (1, 0, 640, 200)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_nan_in_visible_key_or_value_poisons_exactly_the_rows_that_see_it(name):
    w, which, idx = CASES[name]
    inp = make_inputs(w)
    getattr(inp, which)[idx] = float("nan")
    o, l = run_gpu(inp)
    o_ref, l_ref = run_oracle(inp)
    nan_ref = np.isnan(o_ref).any(axis=-1)
    nan_gpu = np.isnan(o).any(axis=-1)
    assert nan_ref.any() and not nan_ref.all(), "the case must poison some rows but not all"
    assert np.array_equal(nan_gpu, nan_ref), "%s: NaN rows differ (%d vs %d)" % (name, nan_gpu.sum(), nan_ref.sum())
    assert np.array_equal(np.isnan(l), np.isnan(l_ref)), "%s: NaN lse rows differ" % name
    keep = ~nan_ref
    compare(o[keep], l[keep], o_ref[keep], l_ref[keep], name)


@pytest.mark.parametrize("which", ["k8", "v8"])
def test_nan_in_visible_fp8_byte_poisons_exactly_the_rows_that_see_it(which):
    """E4M3 K/V (the decode kernel's FP8 variant, whose softmax warps run the
    segment epilogues themselves): the NaN code 0x7F inside a row's visible
    keys makes exactly the rows that see it NaN, as in the oracle's decode."""
    import oracle
    from gqa_attention_forward_flash_b200 import binding

    w = Workload("nan_fp8", B=3, Hq=32, Hkv=4, Tq=1, Tkv=1500, d=128, kv_fp8=True, seed=37)
    inp = make_inputs(w)
    getattr(inp, which).view(torch.uint8)[1, 2, 700, 5] = 0x7F  # the E4M3 NaN code
    dev = "cuda"
    out, lse = binding.gqa_attention_fwd_fp8kv(inp.q.to(dev), inp.k8.to(dev), inp.v8.to(dev), inp.k_scale,
                                               inp.v_scale, None, None, scale=inp.scale, causal=inp.causal)
    assert binding.gqa_get_device_error() == 0
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    ro, rl = oracle.attention_fp8kv(inp.q, inp.k8, inp.v8, inp.k_scale, inp.v_scale, None, None,
                                    scale=inp.scale, causal=inp.causal)
    nan_ref = np.isnan(ro).any(axis=-1)
    assert nan_ref.any() and not nan_ref.all()
    assert np.array_equal(np.isnan(o).any(axis=-1), nan_ref)
    assert np.array_equal(np.isnan(l), np.isnan(rl))
    keep = ~nan_ref
    compare(o[keep], l[keep], ro[keep], rl[keep], "fp8 " + which)
