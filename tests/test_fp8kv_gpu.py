"""GPU parity of the FP8 (E4M3) K/V entry point against the fp64 oracle, which
decodes the same bytes and multiplies by the same per-tensor scales.

The kernel reads each K/V tile as bytes, widens it exactly to f16 in shared
memory (zeroing V rows past the logical length), takes Q to f16 and keeps P in
f16; the tolerance is that of the bf16 path.  Cases: ragged lengths with NaN
padding (the NaN bytes must never reach the output), 8 and 16 packed rows, a
causal decode step with Tq > 1 and a sink, zero lengths and lengths at tile
edges, scales far from 1, and the full-size batched decode on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200.synth import WORKLOADS, Workload, make_inputs, shrink, to_e4m3

from parity import compare, sample_rows

pytestmark = pytest.mark.gpu

W = WORKLOADS["batched_decode_fp8kv"]
CASES = {
    "decode_ragged_nan": shrink(W, B=4, Tkv=3000),
    "g4_eight_rows": Workload("g4", B=3, Hq=8, Hkv=2, Tq=1, Tkv=1000, d=128, ragged=True, nan_pad=True,
                              kv_fp8=True, seed=41),
    "g8_tq2_causal_sink": Workload("g8t2", B=3, Hq=16, Hkv=2, Tq=2, Tkv=777, d=128, causal=True, sink=True,
                                   ragged=True, nan_pad=True, kv_fp8=True, seed=42),
    "mha": Workload("mha", B=2, Hq=4, Hkv=4, Tq=1, Tkv=515, d=128, kv_fp8=True, seed=43),
}


def run(inp):
    dev = "cuda"
    kv = None if inp.kv_lens is None else inp.kv_lens.to(dev)
    sink = None if inp.sink is None else inp.sink.to(dev)
    out, lse = binding.gqa_attention_fwd_fp8kv(inp.q.to(dev), inp.k8.to(dev), inp.v8.to(dev), inp.k_scale,
                                               inp.v_scale, kv, sink, scale=inp.scale, causal=inp.causal)
    err = binding.gqa_get_device_error()
    assert err == 0, binding.STATUS.get(err, err)
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def ref(inp):
    return oracle.attention_fp8kv(inp.q, inp.k8, inp.v8, inp.k_scale, inp.v_scale, inp.kv_lens, inp.sink,
                                  scale=inp.scale, causal=inp.causal)


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8kv_parity_small(name):
    inp = make_inputs(CASES[name])
    o, l = run(inp)
    ro, rl = ref(inp)
    compare(o, l, ro, rl, name)


def test_fp8kv_zero_and_edge_lengths():
    # drawn without padding, then padded with NaN past the chosen lengths
    w = Workload("edges", B=5, Hq=16, Hkv=2, Tq=1, Tkv=640, d=128, sink=True, kv_fp8=True, seed=44)
    inp = make_inputs(w)
    inp.kv_lens = torch.tensor([0, 128, 129, 640, 1], dtype=torch.int32)
    k, v = inp.k.clone(), inp.v.clone()
    for b, n in enumerate(inp.kv_lens.tolist()):
        k[b, :, n:] = float("nan")
        v[b, :, n:] = float("nan")
    inp.k8, inp.k_scale = to_e4m3(k)
    inp.v8, inp.v_scale = to_e4m3(v)
    o, l = run(inp)
    ro, rl = ref(inp)
    compare(o, l, ro, rl, "edge lengths")
    assert np.all(o[0] == 0)  # no key: O = 0, lse = sink
    np.testing.assert_allclose(l[0, :, 0], inp.sink.numpy(), atol=1e-6)


def test_fp8kv_scales_far_from_one():
    inp = make_inputs(CASES["g4_eight_rows"])
    # the same bytes with scales scaled by 2^-7 and 2^9 and the logit scale compensating
    inp.k_scale *= 2.0 ** -7
    inp.scale *= 2.0 ** 7
    inp.v_scale *= 2.0 ** 9
    o, l = run(inp)
    ro, rl = ref(inp)
    compare(o / 2.0 ** 9, l, ro / 2.0 ** 9, rl, "scaled")
    assert np.abs(ro).max() > 1.0


def test_fp8kv_full_size_sampled():
    inp = make_inputs(W)
    o, l = run(inp)
    assert np.all(np.isfinite(o))
    rows = sample_rows(W.B, W.Hq, W.Tq, 384, seed=3)
    ro, rl = oracle.attention_rows_fp8kv(inp.q, inp.k8, inp.v8, inp.k_scale, inp.v_scale, inp.kv_lens, inp.sink,
                                         inp.scale, inp.causal, rows)
    compare(o.reshape(-1, W.d)[rows], l.reshape(-1)[rows], ro, rl, "batched_decode_fp8kv")


def test_fp8kv_deterministic_and_graph_capturable():
    inp = make_inputs(CASES["decode_ragged_nan"])
    dev = "cuda"
    q, k8, v8, kv = inp.q.to(dev), inp.k8.to(dev), inp.v8.to(dev), inp.kv_lens.to(dev)
    a, la = binding.gqa_attention_fwd_fp8kv(q, k8, v8, inp.k_scale, inp.v_scale, kv, scale=inp.scale)
    out, lse = torch.empty_like(a), torch.empty_like(la)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            binding.gqa_attention_fwd_fp8kv(q, k8, v8, inp.k_scale, inp.v_scale, kv, None, out, lse,
                                            scale=inp.scale, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, a) and torch.equal(lse, la)
    assert binding.gqa_get_device_error() == 0


def test_fp8kv_unsupported_shapes_are_refused():
    dev = "cuda"
    q = torch.zeros((1, 32, 1, 64), dtype=torch.bfloat16, device=dev)
    k8 = torch.zeros((1, 1, 100, 64), dtype=torch.uint8, device=dev)
    with pytest.raises(binding.GQAError) as e:
        binding.gqa_attention_fwd_fp8kv(q, k8, k8, 1.0, 1.0)
    assert e.value.status == -7  # head dim 64
    q = torch.zeros((1, 32, 1, 128), dtype=torch.bfloat16, device=dev)
    k8 = torch.zeros((1, 1, 100, 128), dtype=torch.uint8, device=dev)
    with pytest.raises(binding.GQAError) as e:
        binding.gqa_attention_fwd_fp8kv(q, k8, k8, 1.0, 1.0)
    assert e.value.status == -7  # 32 packed rows
