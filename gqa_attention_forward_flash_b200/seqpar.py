"""Sequence parallelism over a key-sharded K/V cache.

The kernbench2 benches commit log (long-context decode commit) spreads every
sequence's keys over several devices: each device computes the softmax state of
its slice, and the states are merged (there, a chain reduce to a root).  Here,
for one process per GPU:

1. rank r holds keys [key_offset, key_offset + capacity) of every sequence
   (k_shard, v_shard: bf16 [B, Hkv, capacity, d]); ``gqa_shard_lengths`` turns
   the global lengths into the shard's;
2. the stream-K forward runs on the shard (no sink), writing its output (bf16,
   normalised over the shard's keys) and lse straight into one packed buffer;
3. one all-gather moves every rank's packed buffer to every rank (over NVLink /
   NVSwitch with NCCL: a single collective per call, the buffers are small);
4. ``gqa_combine_shards`` merges the ranks' results (the sink enters once), on
   every rank, reading the gathered buffer in place.

Every rank ends with the whole output, which is what a replicated next layer
needs; with NVSwitch every rank reaches every peer at full bandwidth, so the
all-gather costs one collective's latency instead of a chain's W - 1 steps.

Supported: any Tq without the causal mask, and causal calls with Tq = 1 (one
query row per head sees every key below its length, so the shards need no
global alignment).  Causal calls with Tq > 1 would need the band's global key
positions inside the kernels and raise NotImplementedError.

The device steps are the library's kernels (``binding``); ``ops`` exists so
that the process-group plumbing can be exercised where no GPU is present.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


class DeviceOps:
    """The library's kernels: the operations a sequence-parallel call performs."""

    shard_lengths = staticmethod(binding.gqa_shard_lengths)
    forward = staticmethod(binding.gqa_attention_fwd)
    combine = staticmethod(binding.gqa_combine_shards)


def packed_layout(B: int, Hq: int, Tq: int, d: int):
    """Byte layout of one rank's packed (out, lse) buffer: out bf16 [B,Hq,Tq,d]
    at 0, lse fp32 [B,Hq,Tq] at ``lse_offset``, the whole rounded up to 16 bytes.
    Returns (lse_offset, total_bytes)."""
    rows = B * Hq * Tq
    lse_offset = (rows * d * 2 + 15) // 16 * 16
    total = (lse_offset + rows * 4 + 15) // 16 * 16
    return lse_offset, total


def _all_gather_bytes(send: torch.Tensor, world: int, group) -> torch.Tensor:
    recv = torch.empty(world * send.numel(), dtype=send.dtype, device=send.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(recv, send, group=group)
    else:
        dist.all_gather(list(recv.chunk(world)), send, group=group)
    return recv


def gqa_attention_fwd_seqpar(q, k_shard, v_shard, kv_lens, sink=None, scale=None, causal=False, key_offset=None,
                             group=None, out=None, lse=None, ops=DeviceOps):
    """The forward over K/V whose keys are split across the ranks of ``group``.

    q: bf16 [B, Hq, Tq, d], the same on every rank; k_shard, v_shard: bf16
    [B, Hkv, capacity, d], this rank's keys; kv_lens: int32 [B], the global
    logical lengths (required); sink: fp32 [Hq] or None; key_offset: global
    position of this rank's first key (default rank * capacity, i.e. equal
    contiguous shards).  Returns (out bf16 [B,Hq,Tq,d], lse fp32 [B,Hq,Tq]) on
    every rank.  Every rank must call it with the same shapes (a collective)."""
    B, Hq, Tq, d = q.shape
    capacity = k_shard.shape[2]
    if causal and Tq > 1:
        raise NotImplementedError("causal sequence parallelism needs Tq == 1")
    if kv_lens is None:
        raise ValueError("sequence parallelism needs the global kv_lens")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if key_offset is None:
        key_offset = rank * capacity
    rows = B * Hq * Tq
    lse_offset, nbytes = packed_layout(B, Hq, Tq, d)

    lens = ops.shard_lengths(kv_lens, key_offset, capacity)
    send = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    o_loc = send[: rows * d * 2].view(torch.bfloat16).view(B, Hq, Tq, d)
    l_loc = send[lse_offset: lse_offset + rows * 4].view(torch.float32).view(B, Hq, Tq)
    # one query row per head: causal and non-causal coincide on every shard
    ops.forward(q, k_shard, v_shard, lens, None, o_loc, l_loc, scale=scale, causal=False)

    recv = _all_gather_bytes(send, world, group).view(world, nbytes)
    o_all = recv[:, : rows * d * 2].view(torch.bfloat16).view(world, B, Hq, Tq, d)
    l_all = recv[:, lse_offset: lse_offset + rows * 4].view(torch.float32).view(world, B, Hq, Tq)
    return ops.combine(o_all, l_all, sink, out, lse)
