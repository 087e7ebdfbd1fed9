"""Sequence parallelism over key shards, on one GPU with the library's kernels.

The ranks are emulated one after another on the same device: shard r's keys
go through gqa_shard_lengths and the stream-K forward (no sink), the shards'
(out, lse) are stacked as an all-gather would stack them, and
gqa_combine_shards merges them; the result must match the fp64 oracle on the
unsharded K/V within the usual tolerance (the shards' outputs are rounded to
bf16 once more than the single-GPU path's).  The whole module path, NCCL
all-gather included, runs as a one-rank process group in a child process.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gqa_attention_forward_flash_b200 import binding, seqpar
from gqa_attention_forward_flash_b200.synth import WORKLOADS, Workload, make_inputs

from parity import compare, run_oracle

pytestmark = pytest.mark.gpu


def _sharded(inp, W, sink=True):
    B, Hq, Tq, d = inp.q.shape
    cap = (inp.k.shape[2] + W - 1) // W
    dev = "cuda"
    q = inp.q.to(dev)
    lens = inp.kv_lens.to(dev)
    o_all = torch.empty((W, B, Hq, Tq, d), dtype=torch.bfloat16, device=dev)
    l_all = torch.empty((W, B, Hq, Tq), dtype=torch.float32, device=dev)
    for r in range(W):
        k = torch.zeros((B, inp.k.shape[1], cap, d), dtype=torch.bfloat16)
        v = torch.zeros_like(k)
        hi = min((r + 1) * cap, inp.k.shape[2])
        k[:, :, : hi - r * cap] = inp.k[:, :, r * cap: hi]
        v[:, :, : hi - r * cap] = inp.v[:, :, r * cap: hi]
        ln = binding.gqa_shard_lengths(lens, r * cap, hi - r * cap)
        binding.gqa_attention_fwd(q, k.to(dev), v.to(dev), ln, None, o_all[r], l_all[r], scale=inp.scale,
                                  causal=False)
    s = inp.sink.to(dev) if (sink and inp.sink is not None) else None
    out, lse = binding.gqa_combine_shards(o_all, l_all, s)
    assert binding.gqa_get_device_error() == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


CASES = {
    "decode_g8_d128": Workload("sp1", B=4, Hq=32, Hkv=4, Tq=1, Tkv=3000, d=128, causal=True, ragged=True,
                               sink=True, seed=81),
    "decode_g4_d64": Workload("sp2", B=3, Hq=8, Hkv=2, Tq=1, Tkv=1000, d=64, ragged=True, sink=True, seed=82),
    "tq5_noncausal": Workload("sp3", B=2, Hq=16, Hkv=2, Tq=5, Tkv=900, d=128, ragged=True, seed=83),
    "decode_d256": Workload("sp4", B=2, Hq=16, Hkv=2, Tq=1, Tkv=700, d=256, ragged=True, sink=True, seed=84),
}


@pytest.mark.parametrize("W", [2, 3, 4])
@pytest.mark.parametrize("name", sorted(CASES))
def test_key_shards_merge_to_the_unsharded_result(name, W):
    w = CASES[name]
    inp = make_inputs(w)
    cap = (w.Tkv + W - 1) // W
    # lengths ending exactly on, just past and before a shard boundary, and zero
    lens = inp.kv_lens.clone()
    lens[0] = cap
    lens[-1] = min(cap + 1, w.Tkv)
    if w.B > 2:
        lens[1] = 0
    inp.kv_lens = lens
    o, l = _sharded(inp, W)
    o_ref, l_ref = run_oracle(inp)
    compare(o, l, o_ref, l_ref, "%s W=%d" % (name, W))


def test_full_size_decode_over_four_shards_sampled():
    import oracle
    w = WORKLOADS["batched_decode"]
    inp = make_inputs(w)
    o, l = _sharded(inp, 4)
    rows = np.random.default_rng(5).choice(w.B * w.Hq * w.Tq, 48, replace=False)
    ro, rl = oracle.attention_rows(inp.q, inp.k, inp.v, inp.kv_lens, inp.sink, inp.scale, w.causal, rows)
    o2 = o.reshape(-1, w.d)[rows]
    l2 = l.reshape(-1)[rows]
    assert np.max(np.abs(o2 - ro)) <= 1e-2
    assert np.linalg.norm(o2 - ro) / np.linalg.norm(ro) <= 5e-3
    assert np.max(np.abs(l2 - rl)) <= 2e-3


def _one_rank(port, q_out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        w = CASES["decode_g8_d128"]
        inp = make_inputs(w)
        dev = "cuda"
        out, lse = seqpar.gqa_attention_fwd_seqpar(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.kv_lens.to(dev),
                                                   inp.sink.to(dev), scale=inp.scale, causal=True)
        torch.cuda.synchronize()
        q_out.put((out.float().cpu().numpy(), lse.cpu().numpy(), binding.gqa_get_device_error()))
    finally:
        dist.destroy_process_group()


def test_module_path_with_a_process_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_one_rank, args=(port, q))
    p.start()
    o, l, err = q.get(timeout=300)
    p.join(timeout=120)
    assert p.exitcode == 0 and err == 0
    w = CASES["decode_g8_d128"]
    inp = make_inputs(w)
    o_ref, l_ref = run_oracle(inp)
    compare(o, l, o_ref, l_ref, "one-rank module path")
