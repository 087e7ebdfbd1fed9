"""The paged-K/V forward (gqa_attention_fwd_paged) on the GPU.

Paging is a storage layout: the same logical keys and values, stored in pages
at shuffled physical positions among NaN-filled spare pages, with page-table
entries past each sequence's pages set to -1.  The paged call must give the
contiguous call's output bit for bit (the kernels walk the same tiles in the
same order) and match the fp64 oracle on the contiguous tensors.
"""
import numpy as np
import pytest
import torch

import oracle
from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200.synth import WORKLOADS, Workload, make_inputs, paginate, shrink

from parity import compare, run_oracle, sample_rows

pytestmark = pytest.mark.gpu

CASES = {
    "decode_ragged_nan": shrink(WORKLOADS["batched_decode"], B=4, Tkv=1000),
    "short_q_causal": shrink(WORKLOADS["short_q_long_kv"], B=2, Tkv=1500),
    "d64_causal_sink": Workload("d64", B=2, Hq=8, Hkv=2, Tq=37, Tkv=900, d=64, causal=True, ragged=True, nan_pad=True,
                                sink=True, seed=21),
    "zero_lengths": Workload("zero", B=3, Hq=8, Hkv=2, Tq=4, Tkv=300, d=128, causal=True, ragged=True, sink=True,
                             seed=13),
}


def _lens(inp):
    if inp.kv_lens is not None:
        return inp.kv_lens.clone()
    return torch.full((inp.q.shape[0],), inp.k.shape[2], dtype=torch.int32)


def _run_both(inp, page_size, seed=5):
    lens = _lens(inp)
    kc, vc, table = paginate(inp.k, inp.v, lens, page_size, seed=seed)
    dev = "cuda"
    q = inp.q.to(dev)
    sink = None if inp.sink is None else inp.sink.to(dev)
    o_p, l_p = binding.gqa_attention_fwd_paged(q, kc.to(dev), vc.to(dev), table.to(dev), lens.to(dev), sink,
                                               scale=inp.scale, causal=inp.causal)
    assert binding.gqa_get_device_error() == 0
    o_c, l_c = binding.gqa_attention_fwd(q, inp.k.to(dev), inp.v.to(dev), lens.to(dev), sink, scale=inp.scale,
                                         causal=inp.causal)
    assert binding.gqa_get_device_error() == 0
    return o_p, l_p, o_c, l_c


@pytest.mark.parametrize("page_size", [16, 64, 128, 256])
@pytest.mark.parametrize("name", sorted(CASES))
def test_paged_equals_contiguous_and_matches_the_oracle(name, page_size):
    w = CASES[name]
    inp = make_inputs(w)
    if name == "zero_lengths":
        inp.kv_lens[0] = 0
        inp.kv_lens[1] = 1
    o_p, l_p, o_c, l_c = _run_both(inp, page_size)
    assert torch.equal(o_p, o_c), "paged output differs from the contiguous one"
    assert torch.equal(l_p, l_c)
    inp.kv_lens = _lens(inp)
    o_ref, l_ref = run_oracle(inp)
    compare(o_p.float().cpu().numpy(), l_p.cpu().numpy(), o_ref, l_ref, "%s, page %d" % (name, page_size))


def test_paged_full_size_decode_sampled():
    w = WORKLOADS["batched_decode"]
    inp = make_inputs(w)
    o_p, l_p, o_c, l_c = _run_both(inp, 64)
    assert torch.equal(o_p, o_c)
    rows = sample_rows(w.B, w.Hq, w.Tq, 96, seed=3)
    o_ref, l_ref = oracle.attention_rows(inp.q, inp.k, inp.v, inp.kv_lens, inp.sink, inp.scale, inp.causal, rows)
    o = o_p.float().cpu().numpy().reshape(-1, w.d)[rows]
    l = l_p.cpu().numpy().reshape(-1)[rows]
    compare(o, l, o_ref, l_ref, "batched decode, paged")


def test_out_of_range_page_id_is_reported_not_read():
    w = CASES["decode_ragged_nan"]
    inp = make_inputs(w)
    lens = _lens(inp)
    kc, vc, table = paginate(inp.k, inp.v, lens, 64, seed=9)
    table[0, 0] = kc.shape[0] + 5  # past the last page
    dev = "cuda"
    binding.gqa_attention_fwd_paged(inp.q.to(dev), kc.to(dev), vc.to(dev), table.to(dev), lens.to(dev), None,
                                    scale=inp.scale, causal=inp.causal)
    assert binding.gqa_get_device_error() == -10  # GQA_ERR_PAGE, then cleared
    assert binding.gqa_get_device_error() == 0
