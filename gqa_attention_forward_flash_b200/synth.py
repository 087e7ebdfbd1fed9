"""Seeded synthetic inputs for the GQA attention forward.

This module holds no attention arithmetic: it only draws the tensors that both
the CUDA path and the fp64 oracle are fed, so that the two sides see the same
bits.  Everything is drawn on the CPU from ``torch.Generator`` seeded per
workload, so a given (workload, seed) gives identical tensors on every machine
with the same torch build.

Recipe (per workload below):
  * Q, K, V: ``randn`` in float32 times ``sigma``, rounded to bf16
    (round-to-nearest-even, torch's cast);
  * kv_len: all equal to the workload's length, or, for the batched decode,
    ``randint`` uniform in [1, Tkv];
  * K and V rows at positions >= kv_len (the padded capacity) are overwritten
    with NaN where the workload asks for NaN padding, so that any read of a
    padded row shows up in the output;
  * sink: ``randn`` float32 per query head (already in the scaled-logit domain);
  * FP8 K/V (workloads with ``kv_fp8``): K and V drawn as above, then stored as
    OCP FP8 E4M3 with one scale per tensor, the AstrAI fp8 quantize recipe:
    scale = amax / 448 over the tensor's finite values, bytes = (x / scale)
    rounded to E4M3 by torch's cast (the NaN padding stays NaN).

The five named workloads are the shapes the pages measure or describe: the
tiny prefill, the batched decode with ragged lengths, the short-query/long-KV
prefill (AstrAI commit log, head-packing commit: G=8, B=16, q=16, kv=16k), the
full causal prefill, and the wide-head decode with a sink and a length that is
not a multiple of 128 (nvfp4-megamoe-kernel dsv4/kernels/attention commit log:
head dims up to 512, sink logit, logical vs padded length).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Tq: int
    Tkv: int            # buffer capacity of K/V
    d: int
    sigma: float = 1.0  # std of Q, K, V
    causal: bool = False
    sink: bool = False
    kv_len: int | None = None   # fixed logical length (None: = Tkv)
    ragged: bool = False        # kv_len ~ U[1, Tkv] per batch
    nan_pad: bool = False       # K/V rows >= kv_len are NaN
    seed: int = 0
    kv_fp8: bool = False        # K/V stored as E4M3 bytes with per-tensor scales

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


WORKLOADS = {
    "tiny_prefill": Workload("tiny_prefill", B=1, Hq=4, Hkv=1, Tq=16, Tkv=128, d=64,
                             seed=1001),
    "batched_decode": Workload("batched_decode", B=16, Hq=32, Hkv=4, Tq=1, Tkv=16384, d=128,
                               ragged=True, nan_pad=True, seed=1002),
    "short_q_long_kv": Workload("short_q_long_kv", B=16, Hq=32, Hkv=4, Tq=16, Tkv=16384, d=128,
                                causal=True, seed=1003),
    "full_causal_prefill": Workload("full_causal_prefill", B=4, Hq=32, Hkv=8, Tq=4096, Tkv=4096,
                                    d=128, causal=True, seed=1004),
    "wide_head_sink_decode": Workload("wide_head_sink_decode", B=8, Hq=32, Hkv=1, Tq=4, Tkv=8192,
                                      d=512, sigma=0.5, causal=True, sink=True, kv_len=8131,
                                      nan_pad=True, seed=1005),
    # the batched decode with its K/V cache in FP8 (E4M3, per-tensor scales)
    "batched_decode_fp8kv": Workload("batched_decode_fp8kv", B=16, Hq=32, Hkv=4, Tq=1, Tkv=16384, d=128,
                                     ragged=True, nan_pad=True, seed=1006, kv_fp8=True),
}


def shrink(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    return replace(w, **kw)


@dataclass
class Inputs:
    q: torch.Tensor            # bf16 [B, Hq, Tq, d]
    k: torch.Tensor            # bf16 [B, Hkv, Tkv, d]
    v: torch.Tensor            # bf16 [B, Hkv, Tkv, d]
    kv_lens: torch.Tensor | None   # int32 [B]
    sink: torch.Tensor | None      # float32 [Hq]
    scale: float
    causal: bool
    k8: torch.Tensor | None = None   # E4M3 [B, Hkv, Tkv, d] (kv_fp8 workloads)
    v8: torch.Tensor | None = None
    k_scale: float = 1.0
    v_scale: float = 1.0


def make_inputs(w: Workload, seed: int | None = None) -> Inputs:
    """Draw the workload's tensors on the CPU."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)

    def normal(shape):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if w.sigma != 1.0:
            x.mul_(w.sigma)
        return x.to(torch.bfloat16)

    q = normal((w.B, w.Hq, w.Tq, w.d))
    k = normal((w.B, w.Hkv, w.Tkv, w.d))
    v = normal((w.B, w.Hkv, w.Tkv, w.d))
    if w.ragged:
        kv_lens = torch.randint(1, w.Tkv + 1, (w.B,), generator=g, dtype=torch.int32)
    elif w.kv_len is not None:
        kv_lens = torch.full((w.B,), w.kv_len, dtype=torch.int32)
    else:
        kv_lens = None
    if w.nan_pad and kv_lens is not None:
        for b in range(w.B):
            n = int(kv_lens[b])
            if n < w.Tkv:
                k[b, :, n:, :] = float("nan")
                v[b, :, n:, :] = float("nan")
    sink = torch.randn((w.Hq,), generator=g, dtype=torch.float32) if w.sink else None
    inp = Inputs(q=q, k=k, v=v, kv_lens=kv_lens, sink=sink, scale=w.scale, causal=w.causal)
    if w.kv_fp8:
        inp.k8, inp.k_scale = to_e4m3(k)
        inp.v8, inp.v_scale = to_e4m3(v)
    return inp


E4M3_MAX = 448.0


def to_e4m3(x: torch.Tensor):
    """One tensor as E4M3 bytes and its scale: scale = amax / 448 over the finite
    values, bytes = x / scale rounded by torch's cast (NaN stays NaN)."""
    xf = x.float()
    fin = torch.isfinite(xf)
    amax = float(xf[fin].abs().max()) if bool(fin.any()) else 1.0
    scale = amax / E4M3_MAX if amax > 0 else 1.0
    return (xf / scale).to(torch.float8_e4m3fn), scale



def paginate(k, v, kv_lens, page_size: int, seed: int, spare_pages: int = 3):
    """Store contiguous K/V [B, Hkv, Tkv, d] as a paged cache: pages of page_size
    tokens laid out [num_pages, Hkv, page_size, d], each sequence's pages at
    shuffled physical positions among spare NaN-filled pages, and a page table
    int32 [B, max_pages] whose entries past a sequence's pages are -1 (never read).
    Storage layout only: the keys and values of every logical position are those
    of the contiguous tensors.  Returns (k_cache, v_cache, page_table)."""
    B, Hkv, Tkv, d = k.shape
    max_pages = (Tkv + page_size - 1) // page_size
    lens = [int(x) for x in kv_lens.tolist()]
    used = [(len_ + page_size - 1) // page_size for len_ in lens]
    num_pages = sum(used) + spare_pages
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    order = torch.randperm(num_pages, generator=g).tolist()
    k_cache = torch.full((num_pages, Hkv, page_size, d), float("nan"), dtype=k.dtype)
    v_cache = torch.full((num_pages, Hkv, page_size, d), float("nan"), dtype=v.dtype)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        for j in range(used[b]):
            phys = order[nxt]
            nxt += 1
            table[b, j] = phys
            lo, hi = j * page_size, min((j + 1) * page_size, Tkv)
            k_cache[phys, :, : hi - lo] = k[b, :, lo:hi, :]
            v_cache[phys, :, : hi - lo] = v[b, :, lo:hi, :]
    return k_cache, v_cache, table
