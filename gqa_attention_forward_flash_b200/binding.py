"""Thin Python binding of the C ABI (include/gqa_attn.h), same names.

Argument marshalling only: shapes come from the tensors, pointers from
``data_ptr()``, the stream from torch's current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback.  If the
library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgqa_attn.so")

STATUS = {
    0: "GQA_OK", -1: "GQA_ERR_NULL", -2: "GQA_ERR_SHAPE", -3: "GQA_ERR_ALIGN", -4: "GQA_ERR_SPLITS",
    -5: "GQA_ERR_CUDA", -6: "GQA_ERR_TIMEOUT", -7: "GQA_ERR_UNSUPPORTED", -8: "GQA_ERR_KVLEN",
    -9: "GQA_ERR_SCRATCH", -10: "GQA_ERR_PAGE", -11: "GQA_ERR_SMEM_ALIGN",
}
MAX_SPLITS = 256

# exported names and their C signatures (restype, argtypes)
_P, _I, _F, _L = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
SIGNATURES = {
    "gqa_attention_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "gqa_attention_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "gqa_attention_fwd_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "gqa_attention_fwd_fp8kv": (_I, [_P, _P, _P, _F, _F, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "gqa_attention_fwd_partial": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _P, _P]),
    "gqa_splitkv_combine": (_I, [_P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P]),
    "gqa_shard_lengths": (_I, [_P, _I, _I, _I, _P, _P]),
    "gqa_combine_shards": (_I, [_P, _L, _P, _L, _I, _P, _P, _P, _I, _I, _I, _I, _P]),
    "gqa_get_device_error": (_I, [_P]),
    "gqa_profile_begin": (_I, []),
    "gqa_profile_take": (_I, [_P, _I, _P]),
    "gqa_status_string": (ctypes.c_char_p, [_I]),
    "gqa_version": (_I, []),
}

_lib = None


class GQAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (fn, STATUS.get(status, "?"), status))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError("libgqa_attn.so is not built; run `python -m gqa_attention_forward_flash_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise GQAError(fn, rc)


def _need(t, dtype, name, ndim):
    if t.dtype != dtype or t.dim() != ndim or not t.is_contiguous() or not t.is_cuda:
        raise ValueError("%s must be a contiguous CUDA %s tensor with %d dims" % (name, dtype, ndim))


def gqa_attention_fwd(q, k, v, kv_lens=None, sink=None, out=None, lse=None, scale=None, causal=False,
                      stream=None):
    """O (and lse) of the GQA forward.  q [B,Hq,Tq,d], k/v [B,Hkv,Tkv,d] bf16;
    kv_lens int32 [B] or None; sink fp32 [Hq] or None.  Returns (out, lse)."""
    _need(q, torch.bfloat16, "q", 4)
    _need(k, torch.bfloat16, "k", 4)
    _need(v, torch.bfloat16, "v", 4)
    B, Hq, Tq, d = q.shape
    _, Hkv, Tkv, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device)
    if kv_lens is not None:
        _need(kv_lens, torch.int32, "kv_lens", 1)
    if sink is not None:
        _need(sink, torch.float32, "sink", 1)
    if scale is None:
        scale = d ** -0.5
    rc = load().gqa_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), _ptr(sink), _ptr(out), _ptr(lse),
                                  B, Hq, Hkv, Tq, Tkv, d, float(scale), int(bool(causal)), _stream(stream))
    _check("gqa_attention_fwd", rc)
    return out, lse


def gqa_attention_fwd_paged(q, k_cache, v_cache, page_table, kv_lens, sink=None, out=None, lse=None, scale=None,
                            causal=False, stream=None):
    """The forward over a paged K/V cache.  q [B,Hq,Tq,d] bf16; k_cache/v_cache
    [num_pages, Hkv, page_size, d] bf16; page_table int32 [B, max_pages];
    kv_lens int32 [B] (required); sink fp32 [Hq] or None.  Returns (out, lse)."""
    _need(q, torch.bfloat16, "q", 4)
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    _need(page_table, torch.int32, "page_table", 2)
    _need(kv_lens, torch.int32, "kv_lens", 1)
    B, Hq, Tq, d = q.shape
    num_pages, Hkv, page_size, _ = k_cache.shape
    max_pages = page_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device)
    if sink is not None:
        _need(sink, torch.float32, "sink", 1)
    if scale is None:
        scale = d ** -0.5
    rc = load().gqa_attention_fwd_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table), _ptr(kv_lens),
                                        _ptr(sink), _ptr(out), _ptr(lse), B, Hq, Hkv, Tq, num_pages, page_size,
                                        max_pages, d, float(scale), int(bool(causal)), _stream(stream))
    _check("gqa_attention_fwd_paged", rc)
    return out, lse


def _need_e4m3(t, name, ndim):
    if t.dtype not in (torch.float8_e4m3fn, torch.uint8) or t.dim() != ndim or not t.is_contiguous() or not t.is_cuda:
        raise ValueError("%s must be a contiguous CUDA float8_e4m3fn (or uint8) tensor with %d dims" % (name, ndim))


def gqa_attention_fwd_fp8kv(q, k8, v8, k_scale, v_scale, kv_lens=None, sink=None, out=None, lse=None, scale=None,
                            causal=False, stream=None):
    """The forward on an FP8 K/V cache: K = k8 * k_scale, V = v8 * v_scale with
    k8/v8 E4M3 [B,Hkv,Tkv,d] (float8_e4m3fn or their uint8 bytes) and per-tensor
    scales.  q [B,Hq,Tq,d] bf16.  Returns (out, lse)."""
    _need(q, torch.bfloat16, "q", 4)
    _need_e4m3(k8, "k8", 4)
    _need_e4m3(v8, "v8", 4)
    B, Hq, Tq, d = q.shape
    _, Hkv, Tkv, _ = k8.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device)
    if kv_lens is not None:
        _need(kv_lens, torch.int32, "kv_lens", 1)
    if sink is not None:
        _need(sink, torch.float32, "sink", 1)
    if scale is None:
        scale = d ** -0.5
    rc = load().gqa_attention_fwd_fp8kv(_ptr(q), _ptr(k8), _ptr(v8), float(k_scale), float(v_scale), _ptr(kv_lens),
                                        _ptr(sink), _ptr(out), _ptr(lse), B, Hq, Hkv, Tq, Tkv, d, float(scale),
                                        int(bool(causal)), _stream(stream))
    _check("gqa_attention_fwd_fp8kv", rc)
    return out, lse


def gqa_attention_fwd_noalloc(q, k, v, kv_lens=None, sink=None, out=None, lse=None, scale=None, causal=False,
                              stream=None):
    """gqa_attention_fwd without device allocation inside the library (its split
    scratch is a fixed array in the library; see include/gqa_attn.h)."""
    _need(q, torch.bfloat16, "q", 4)
    _need(k, torch.bfloat16, "k", 4)
    _need(v, torch.bfloat16, "v", 4)
    B, Hq, Tq, d = q.shape
    _, Hkv, Tkv, _ = k.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device)
    if kv_lens is not None:
        _need(kv_lens, torch.int32, "kv_lens", 1)
    if sink is not None:
        _need(sink, torch.float32, "sink", 1)
    if scale is None:
        scale = d ** -0.5
    rc = load().gqa_attention_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), _ptr(sink), _ptr(out),
                                          _ptr(lse), B, Hq, Hkv, Tq, Tkv, d, float(scale), int(bool(causal)),
                                          _stream(stream))
    _check("gqa_attention_fwd_noalloc", rc)
    return out, lse


def gqa_attention_fwd_partial(q, k, v, kv_lens=None, scale=None, causal=False, num_splits=2, o_part=None,
                              lse_part=None, stream=None):
    """Split partials (no combine, no sink): o_part fp32 [B,Hq,Tq,S,d], lse_part fp32 [B,Hq,Tq,S]."""
    _need(q, torch.bfloat16, "q", 4)
    _need(k, torch.bfloat16, "k", 4)
    _need(v, torch.bfloat16, "v", 4)
    if kv_lens is not None:
        _need(kv_lens, torch.int32, "kv_lens", 1)
    B, Hq, Tq, d = q.shape
    _, Hkv, Tkv, _ = k.shape
    if o_part is None:
        o_part = torch.empty((B, Hq, Tq, num_splits, d), dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty((B, Hq, Tq, num_splits), dtype=torch.float32, device=q.device)
    _need(o_part, torch.float32, "o_part", 5)
    _need(lse_part, torch.float32, "lse_part", 4)
    if tuple(o_part.shape) != (B, Hq, Tq, num_splits, d) or tuple(lse_part.shape) != (B, Hq, Tq, num_splits):
        raise ValueError("o_part must be [B, Hq, Tq, num_splits, d] and lse_part [B, Hq, Tq, num_splits]")
    if scale is None:
        scale = d ** -0.5
    rc = load().gqa_attention_fwd_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), B, Hq, Hkv, Tq, Tkv, d,
                                          float(scale), int(bool(causal)), int(num_splits), _ptr(o_part),
                                          _ptr(lse_part), _stream(stream))
    _check("gqa_attention_fwd_partial", rc)
    return o_part, lse_part


def gqa_splitkv_combine(o_part, lse_part, sink=None, out=None, lse=None, stream=None):
    """LSE combine of [B,Hq,Tq,S,d] partials into bf16 out [B,Hq,Tq,d] and lse."""
    _need(o_part, torch.float32, "o_part", 5)
    _need(lse_part, torch.float32, "lse_part", 4)
    B, Hq, Tq, S, d = o_part.shape
    if tuple(lse_part.shape) != (B, Hq, Tq, S):
        raise ValueError("lse_part must be [B, Hq, Tq, S] for o_part [B, Hq, Tq, S, d]")
    if sink is not None:
        _need(sink, torch.float32, "sink", 1)
    if out is None:
        out = torch.empty((B, Hq, Tq, d), dtype=torch.bfloat16, device=o_part.device)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=o_part.device)
    _need(out, torch.bfloat16, "out", 4)
    _need(lse, torch.float32, "lse", 3)
    rc = load().gqa_splitkv_combine(_ptr(o_part), _ptr(lse_part), S, _ptr(sink), _ptr(out), _ptr(lse),
                                    B, Hq, Tq, d, _stream(stream))
    _check("gqa_splitkv_combine", rc)
    return out, lse


def gqa_shard_lengths(kv_lens, key_offset, shard_capacity, out=None, stream=None):
    """clamp(kv_lens - key_offset, 0, shard_capacity): int32 [B] on the device."""
    _need(kv_lens, torch.int32, "kv_lens", 1)
    if out is None:
        out = torch.empty_like(kv_lens)
    _need(out, torch.int32, "out", 1)
    rc = load().gqa_shard_lengths(_ptr(kv_lens), kv_lens.shape[0], int(key_offset), int(shard_capacity), _ptr(out),
                                  _stream(stream))
    _check("gqa_shard_lengths", rc)
    return out


def gqa_combine_shards(o_shards, lse_shards, sink=None, out=None, lse=None, stream=None):
    """LSE merge of per-shard results: o_shards bf16 [S, B, Hq, Tq, d] (any shard
    stride, rows contiguous), lse_shards fp32 [S, B, Hq, Tq].  Returns (out, lse)."""
    if o_shards.dim() != 5 or o_shards.dtype != torch.bfloat16 or not o_shards.is_cuda or not o_shards[0].is_contiguous():
        raise ValueError("o_shards must be a CUDA bf16 [S, B, Hq, Tq, d] tensor with contiguous shards")
    S, B, Hq, Tq, d = o_shards.shape
    if (lse_shards.dtype != torch.float32 or not lse_shards.is_cuda or tuple(lse_shards.shape) != (S, B, Hq, Tq)
            or not lse_shards[0].is_contiguous()):
        raise ValueError("lse_shards must be a CUDA fp32 [S, B, Hq, Tq] tensor with contiguous shards")
    if sink is not None:
        _need(sink, torch.float32, "sink", 1)
    if out is None:
        out = torch.empty((B, Hq, Tq, d), dtype=torch.bfloat16, device=o_shards.device)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=o_shards.device)
    _need(out, torch.bfloat16, "out", 4)
    _need(lse, torch.float32, "lse", 3)
    rc = load().gqa_combine_shards(_ptr(o_shards), o_shards.stride(0), _ptr(lse_shards), lse_shards.stride(0), S,
                                   _ptr(sink), _ptr(out), _ptr(lse), B, Hq, Tq, d, _stream(stream))
    _check("gqa_combine_shards", rc)
    return out, lse


def gqa_get_device_error(stream=None) -> int:
    return load().gqa_get_device_error(_stream(stream))


def gqa_profile_begin() -> None:
    _check("gqa_profile_begin", load().gqa_profile_begin())


def gqa_profile_take(max_calls: int = 4096):
    """Per-call kernel durations (ms) since gqa_profile_begin."""
    ms = (ctypes.c_float * max_calls)()
    n = ctypes.c_int(0)
    _check("gqa_profile_take", load().gqa_profile_take(ms, max_calls, ctypes.byref(n)))
    return list(ms[:n.value])


def gqa_status_string(status: int) -> str:
    return load().gqa_status_string(int(status)).decode()


def gqa_version() -> int:
    return load().gqa_version()
