"""The swap-AB decode kernel (head dim 128, at most 16 packed query rows per
(batch, KV head)) against the fp64 oracle.

Calls with G*Tq <= 16 at d = 128 take this kernel; the cases span both row
counts it reads (8 and 16), a single row (MHA decode), causal rows with Tq > 1,
the sink, logical lengths of 0, 1 and around the 128-key tile edge, NaN-filled
padding, rows long enough to be split over several CTAs and merged, and logits
peaked enough to move the running maximum late in a row (the lazy rescale).
"""
import numpy as np
import pytest
import torch

from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200.synth import Workload, make_inputs, paginate

from parity import compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def _set_lengths(inp, lens):
    """Logical lengths, with every K/V row at or past its length NaN (the inputs
    must be drawn without padding, so that every row below a length is finite)."""
    inp.kv_lens = torch.tensor(lens, dtype=torch.int32)
    for b, n in enumerate(lens):
        inp.k[b, :, n:] = float("nan")
        inp.v[b, :, n:] = float("nan")

CASES = {
    # name: (Hq, Hkv, Tq, causal, sink)
    "g8_decode": (32, 4, 1, False, False),
    "g8_decode_sink": (16, 2, 1, True, True),
    "mha_one_row": (4, 4, 1, False, True),
    "g16_decode": (32, 2, 1, False, False),
    "g4_tq2_causal": (8, 2, 2, True, False),
    "g5_tq3_causal_sink": (10, 2, 3, True, True),
    "g3_tq3": (6, 2, 3, False, False),
    "g2_tq8_causal": (4, 2, 8, True, True),
}


@pytest.mark.parametrize("Tkv", [300, 5000])
@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_kernel_matches_the_oracle(name, Tkv):
    Hq, Hkv, Tq, causal, sink = CASES[name]
    w = Workload(name, B=3, Hq=Hq, Hkv=Hkv, Tq=Tq, Tkv=Tkv, d=128, causal=causal, ragged=True, sink=sink,
                 seed=40 + Tkv % 7)
    inp = make_inputs(w)
    # lengths at the tile edges and the degenerate ones, then one drawn at random
    edge = [0, 1, 127, 128, 129, 256, Tkv]
    _set_lengths(inp, [edge[(Hq + Tq) % len(edge)], Tkv, int(inp.kv_lens[2])])
    o, l = run_gpu(inp)
    o_ref, l_ref = run_oracle(inp)
    compare(o, l, o_ref, l_ref, "%s Tkv=%d lens=%s" % (name, Tkv, inp.kv_lens.tolist()))


@pytest.mark.parametrize("Tq", [1, 2])
def test_decode_kernel_every_length_near_the_tile_edges(Tq):
    # one batch row per length: 1..3, 126..130, 254..258 keys
    lens = [1, 2, 3, 126, 127, 128, 129, 130, 254, 255, 256, 257, 258]
    w = Workload("edges", B=len(lens), Hq=8, Hkv=1, Tq=Tq, Tkv=260, d=128, causal=True, sink=True, seed=61)
    inp = make_inputs(w)
    _set_lengths(inp, lens)
    o, l = run_gpu(inp)
    o_ref, l_ref = run_oracle(inp)
    compare(o, l, o_ref, l_ref, "edges Tq=%d" % Tq)


def test_decode_kernel_late_maximum_rescale():
    # logits that keep growing along the row: the running max moves many times,
    # in pieces split over several CTAs
    w = Workload("ramp", B=2, Hq=16, Hkv=2, Tq=1, Tkv=6000, d=128, seed=62)
    inp = make_inputs(w)
    ramp = torch.linspace(0.0, 24.0, w.Tkv).to(torch.float32)
    inp.k = (inp.k.float() * 0.2 + ramp[None, None, :, None] * inp.q.float().mean(dim=(1, 2), keepdim=True)).to(torch.bfloat16)
    o, l = run_gpu(inp)
    o_ref, l_ref = run_oracle(inp)
    compare(o, l, o_ref, l_ref, "late maximum")


def test_decode_kernel_constant_values():
    # every visible V row equal -> O equals that row whatever the weights (|O| ~ 1)
    w = Workload("const", B=2, Hq=16, Hkv=2, Tq=1, Tkv=3000, d=128, ragged=True, nan_pad=True, seed=63)
    inp = make_inputs(w)
    row = torch.randn(w.d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    for b in range(w.B):
        n = int(inp.kv_lens[b])
        inp.v[b, :, :n] = row
    o, l = run_gpu(inp)
    expect = np.broadcast_to(row.float().numpy().astype(np.float64), o.shape)
    live = (inp.kv_lens > 0).numpy()
    assert np.max(np.abs(o[live] - expect[live])) <= 1e-2


def test_decode_kernel_paged_equals_contiguous():
    w = Workload("pg", B=4, Hq=32, Hkv=4, Tq=1, Tkv=2000, d=128, ragged=True, sink=True, seed=64)
    inp = make_inputs(w)
    _set_lengths(inp, [0] + inp.kv_lens.tolist()[1:])
    dev = "cuda"
    kc, vc, table = paginate(inp.k, inp.v, inp.kv_lens, 16, seed=7)
    q, sink, lens = inp.q.to(dev), inp.sink.to(dev), inp.kv_lens.to(dev)
    o_p, l_p = binding.gqa_attention_fwd_paged(q, kc.to(dev), vc.to(dev), table.to(dev), lens, sink,
                                               scale=inp.scale, causal=inp.causal)
    assert binding.gqa_get_device_error() == 0
    o_c, l_c = binding.gqa_attention_fwd(q, inp.k.to(dev), inp.v.to(dev), lens, sink, scale=inp.scale,
                                         causal=inp.causal)
    assert binding.gqa_get_device_error() == 0
    assert torch.equal(o_p, o_c) and torch.equal(l_p, l_c)
    o_ref, l_ref = run_oracle(inp)
    compare(o_p.float().cpu().numpy(), l_p.cpu().numpy(), o_ref, l_ref, "paged decode kernel")


def test_decode_kernel_agrees_with_the_split_path():
    # the uniform-split path (two-lane kernel + combine) on the same inputs
    w = Workload("cmp", B=3, Hq=16, Hkv=2, Tq=1, Tkv=4000, d=128, ragged=True, nan_pad=True, sink=True, seed=65)
    inp = make_inputs(w)
    o, l = run_gpu(inp)
    dev = "cuda"
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    lens, sink = inp.kv_lens.to(dev), inp.sink.to(dev)
    o_part, l_part = binding.gqa_attention_fwd_partial(q, k, v, lens, scale=inp.scale, causal=inp.causal,
                                                       num_splits=4)
    o2, l2 = binding.gqa_splitkv_combine(o_part, l_part, sink)
    assert binding.gqa_get_device_error() == 0
    o2 = o2.float().cpu().numpy()
    assert np.max(np.abs(o - o2)) <= 1e-2
    fin = np.isfinite(l)
    assert np.max(np.abs(l[fin] - l2.cpu().numpy()[fin])) <= 2e-3
