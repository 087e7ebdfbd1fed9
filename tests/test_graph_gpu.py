"""CUDA graphs: calls into the library captured in a graph and replayed give the
eager results bit for bit (the kernels are deterministic and take every size
through kernel parameters), for the swap-AB decode kernel, the two-lane kernel
and the wide kernel (cooperative launch, in-kernel merge); a captured call that would
need more scratch than is in place is refused, not allocated."""
import pytest
import torch

from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200.synth import Workload, WORKLOADS, make_inputs, shrink

pytestmark = pytest.mark.gpu

CASES = {
    "decode_swap_ab": shrink(WORKLOADS["batched_decode"], B=4, Tkv=3000),
    "prefill_two_lane": Workload("gp", B=1, Hq=8, Hkv=2, Tq=300, Tkv=700, d=128, causal=True, sink=True, seed=91),
    "wide_head_d512": shrink(WORKLOADS["wide_head_sink_decode"], B=2, Tkv=1500, kv_len=1403),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_graph_replay_equals_eager(name):
    inp = make_inputs(CASES[name])
    dev = "cuda"
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    kv = None if inp.kv_lens is None else inp.kv_lens.to(dev)
    sink = None if inp.sink is None else inp.sink.to(dev)
    o_e, l_e = binding.gqa_attention_fwd(q, k, v, kv, sink, scale=inp.scale, causal=inp.causal)
    torch.cuda.synchronize()
    out = torch.empty_like(o_e)
    lse = torch.empty_like(l_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(3):  # back to back, the way a layer loop would
                binding.gqa_attention_fwd(q, k, v, kv, sink, out, lse, scale=inp.scale, causal=inp.causal, stream=s)
    for _ in range(4):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert binding.gqa_get_device_error() == 0
        assert torch.equal(out, o_e) and torch.equal(lse, l_e)


def test_capture_refuses_to_grow_scratch():
    # more row-blocks (8192 merge tickets) than any call before in this process has
    # needed: the ticket array would have to grow, and a capture must not allocate
    w = Workload("big", B=1024, Hq=8, Hkv=8, Tq=1, Tkv=16, d=64, seed=92)
    inp = make_inputs(w)
    dev = "cuda"
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Tq), dtype=torch.float32, device=dev)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with pytest.raises(binding.GQAError) as e:
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                binding.gqa_attention_fwd(q, k, v, None, None, out, lse, stream=s)
    assert e.value.status == -9
