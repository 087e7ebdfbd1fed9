"""The allocation-free entry point, checked against the fp64 oracle and against
gqa_attention_fwd.

Some callers cannot let a library allocate device memory while they run:
engines that divide all of HBM among their own pools at start-up, code running
where an allocation (which may synchronise the device) is not allowed, hosts
without a device allocator.  gqa_attention_fwd_noalloc serves them from a
fixed array inside the library.  Called twice in a row through the C ABI, it
must match the oracle within the parity tolerances and reproduce
gqa_attention_fwd within the same tolerances; the error word it leaves in its
array must read back as zero through gqa_get_device_error.

The cases cover the three kernel families: the swap-AB decode kernel (head
dim 128, few packed rows), the two-lane kernel (head dims 64 and 128, split-key
and dual-Q lanes) and the wide kernel (head dims 256 and 512), whose merge
counters also live in the fixed array.

This file is named so that pytest collects it last: a run that stops at the
first failure has then already run every other test.
"""
import ctypes

import pytest
import torch

from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200 import build as build_mod
from gqa_attention_forward_flash_b200.synth import WORKLOADS, Workload, make_inputs, shrink

from parity import compare, run_oracle

pytestmark = pytest.mark.gpu

CASES = {
    "decode_ragged_nan": shrink(WORKLOADS["batched_decode"], B=4, Tkv=3000),
    "short_q_long_kv": shrink(WORKLOADS["short_q_long_kv"], B=2, Tkv=2500),
    "causal_prefill": shrink(WORKLOADS["full_causal_prefill"], B=1, Hq=8, Hkv=2, Tq=1100, Tkv=1100),
    "d64_causal_sink": Workload("d64", B=2, Hq=8, Hkv=2, Tq=37, Tkv=900, d=64, causal=True, ragged=True,
                                nan_pad=True, sink=True, seed=21),
    # head dims 256 and 512: the wide kernel's split row-blocks are merged in the
    # kernel, with their counters in the array
    "d256_sink_nan_split": Workload("d256", B=2, Hq=16, Hkv=2, Tq=3, Tkv=6000, d=256, sigma=0.5, causal=True,
                                    sink=True, kv_len=5555, nan_pad=True, seed=22),
    "d512_sink_nan_split": shrink(WORKLOADS["wide_head_sink_decode"], B=2, Tkv=3000, kv_len=2903),
}


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return binding.load()


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_oracle_and_fwd_on_two_calls(lib, name):
    w = CASES[name]
    inp = make_inputs(w)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    kv = None if inp.kv_lens is None else inp.kv_lens.cuda()
    sink = None if inp.sink is None else inp.sink.cuda()
    oracle_o, oracle_l = run_oracle(inp)
    fwd_o, fwd_l = binding.gqa_attention_fwd(q, k, v, kv, sink, scale=inp.scale, causal=inp.causal)
    assert binding.gqa_get_device_error() == 0
    fwd_o = fwd_o.float().cpu().numpy()
    fwd_l = fwd_l.cpu().numpy()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((w.B, w.Hq, w.Tq), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.gqa_attention_fwd_noalloc(_p(q), _p(k), _p(v), _p(kv), _p(sink), _p(out), _p(lse),
                                           w.B, w.Hq, w.Hkv, w.Tq, w.Tkv, w.d, inp.scale, int(inp.causal), stream)
        assert rc == 0, binding.STATUS.get(rc, rc)
        # waits for the stream; reads (and clears) the array's error word too
        assert lib.gqa_get_device_error(stream) == 0
        o = out.float().cpu().numpy()
        l = lse.cpu().numpy()
        compare(o, l, oracle_o, oracle_l, "%s, call %d, against the oracle" % (name, call))
        compare(o, l, fwd_o, fwd_l, "%s, call %d, against gqa_attention_fwd" % (name, call))


def test_noalloc_rejects_problems_beyond_its_array(lib):
    # 70000 row-blocks exceed the array's 65536 merge tickets
    B = 70000
    q = torch.zeros((B, 1, 1, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, 1, 1, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    rc = lib.gqa_attention_fwd_noalloc(_p(q), _p(k), _p(k), None, None, _p(out), None, B, 1, 1, 1, 1, 64, 0.125, 0,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -9  # GQA_ERR_SCRATCH
