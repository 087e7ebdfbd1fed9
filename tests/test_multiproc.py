"""Multi-process host logic on CPU (gloo, world size 2): the sequence-parallel
forward's process-group plumbing (shard lengths, packed buffers, all-gather,
combine from the gathered buffer) and the bench's barrier / max-over-ranks.

The device operations of the sequence-parallel call are replaced here by
oracle-based stand-ins (the oracle is test infrastructure); what runs for real
is the module's own code and the collectives.  The CUDA kernels behind the same
calls are checked on the GPU in test_seqpar_gpu.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from gqa_attention_forward_flash_b200 import seqpar
from gqa_attention_forward_flash_b200.synth import Workload, make_inputs


class OracleOps:
    """CPU stand-ins with the kernels' contracts (outputs bf16, lse fp32, -inf for no key)."""

    @staticmethod
    def shard_lengths(kv_lens, key_offset, capacity):
        return (kv_lens.to(torch.int64) - key_offset).clamp(0, capacity).to(torch.int32)

    @staticmethod
    def forward(q, k, v, lens, sink, out, lse, scale=None, causal=False):
        assert sink is None
        o, l = oracle.attention(q, k, v, lens, None, scale=scale, causal=causal)
        out.copy_(torch.from_numpy(o).to(torch.bfloat16))
        lse.copy_(torch.from_numpy(l).to(torch.float32))

    @staticmethod
    def combine(o_all, l_all, sink, out, lse):
        o = o_all.float().permute(1, 2, 3, 0, 4).contiguous().numpy()
        l = l_all.permute(1, 2, 3, 0).contiguous().numpy()
        ro, rl = oracle.combine(o, l, None if sink is None else sink.numpy())
        return torch.from_numpy(ro), torch.from_numpy(rl)


CASES = {
    # name: (Workload, lengths or None)
    "decode_causal_sink": (Workload("d", B=4, Hq=8, Hkv=2, Tq=1, Tkv=600, d=64, causal=True, sink=True, seed=71),
                           [0, 1, 299, 600]),
    "tq3_noncausal": (Workload("n", B=3, Hq=4, Hkv=1, Tq=3, Tkv=520, d=64, seed=72), [300, 260, 17]),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, case, q_out):
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        if case == "bench":
            bench.barrier(world)
            q_out.put((rank, bench.all_max(world, float(rank + 1) * 1.5)))
            return
        w, lens = CASES[case]
        inp = make_inputs(w)
        inp.kv_lens = torch.tensor(lens, dtype=torch.int32)
        cap = w.Tkv // world
        sl = slice(rank * cap, (rank + 1) * cap)
        out, lse = seqpar.gqa_attention_fwd_seqpar(inp.q, inp.k[:, :, sl].contiguous(), inp.v[:, :, sl].contiguous(),
                                                   inp.kv_lens, inp.sink, scale=inp.scale, causal=w.causal,
                                                   ops=OracleOps)
        q_out.put((rank, (out.numpy(), lse.numpy())))
    finally:
        dist.destroy_process_group()


def _run(case, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_packed_layout_is_aligned():
    for B, Hq, Tq, d in [(1, 1, 1, 64), (3, 5, 7, 128), (16, 32, 1, 512)]:
        off, total = seqpar.packed_layout(B, Hq, Tq, d)
        assert off % 16 == 0 and total % 16 == 0
        assert off >= B * Hq * Tq * d * 2 and total >= off + B * Hq * Tq * 4


def test_causal_rows_beyond_one_need_global_alignment():
    w = Workload("c", B=1, Hq=2, Hkv=1, Tq=2, Tkv=8, d=64, causal=True)
    inp = make_inputs(w)
    with pytest.raises(NotImplementedError):
        seqpar.gqa_attention_fwd_seqpar(inp.q, inp.k, inp.v, torch.tensor([8], dtype=torch.int32), causal=True,
                                        ops=OracleOps)


@pytest.mark.parametrize("case", sorted(CASES))
def test_seqpar_two_ranks_match_the_unsharded_oracle(case):
    res = _run(case)
    w, lens = CASES[case]
    inp = make_inputs(w)
    kv = torch.tensor(lens, dtype=torch.int32)
    ro, rl = oracle.attention(inp.q, inp.k, inp.v, kv, inp.sink, scale=inp.scale, causal=w.causal)
    for r in (0, 1):
        o, l = res[r]
        assert np.max(np.abs(o - ro)) <= 1e-2
        rel = np.linalg.norm(o - ro) / max(np.linalg.norm(ro), 1e-30)
        assert rel <= 5e-3
        fin = np.isfinite(rl)
        assert np.array_equal(np.isneginf(l), np.isneginf(rl))
        assert np.max(np.abs(l[fin] - rl[fin])) <= 2e-3
    # both ranks hold the same result
    assert np.array_equal(res[0][0], res[1][0])


def test_bench_max_over_ranks():
    res = _run("bench")
    assert res[0] == res[1] == 3.0
