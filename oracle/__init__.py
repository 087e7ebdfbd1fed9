"""fp64 CPU oracle for the grouped-query-attention forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The product path never
does, and it shares no code with the CUDA library.

The arithmetic lives in ``gqa_oracle.c`` (plain C, double precision, OpenMP over
output rows); this module only compiles it with gcc and marshals numpy arrays.
bf16 tensors are passed as their uint16 bit patterns.

Functions (each restates the definition written in the C file's header):

* :func:`attention` -- the full forward, O and lse for every row.
* :func:`attention_window` -- the same restricted to keys in [kv_begin, kv_end):
  the partial a split of the keys produces.
* :func:`attention_rows` -- the full forward for a list of flat rows
  ``(b*Hq + h)*Tq + i`` only (for sampled checks at full size).
* :func:`combine` -- the LSE merge of per-split partials.
* :func:`attention_fp8kv`, :func:`attention_rows_fp8kv` -- the forward with K and
  V stored as OCP FP8 E4M3 bytes and one scale per tensor (K = value(k) * k_scale,
  V = value(v) * v_scale), computed in double.
* :func:`e4m3_decode` -- the E4M3 byte decoder those use.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_LIB = os.path.join(_HERE, "_gqa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, IEEE semantics kept)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_long
        D = ctypes.c_double
        lib.oracle_attention_window.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, D, I, L, L, I]
        lib.oracle_attention_window.restype = I
        lib.oracle_attention_rows.argtypes = [P, P, P, P, P, P, L, P, P, I, I, I, I, I, I, D, I, I]
        lib.oracle_attention_rows.restype = I
        lib.oracle_attention_window_fp8kv.argtypes = [P, P, P, D, D, P, P, P, P, I, I, I, I, I, I, D, I, L, L, I]
        lib.oracle_attention_window_fp8kv.restype = I
        lib.oracle_attention_rows_fp8kv.argtypes = [P, P, P, D, D, P, P, P, L, P, P, I, I, I, I, I, I, D, I, I]
        lib.oracle_attention_rows_fp8kv.restype = I
        lib.oracle_e4m3_decode.argtypes = [P, P, L]
        lib.oracle_e4m3_decode.restype = None
        lib.oracle_combine.argtypes = [P, P, I, P, P, P, I, I, I, I]
        lib.oracle_combine.restype = I
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def _bits(x) -> np.ndarray:
    """bf16 tensor/array -> contiguous uint16 bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(x)
    assert a.dtype == np.uint16
    return np.ascontiguousarray(a)


def _opt(x, dtype):
    if x is None:
        return None, None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(np.asarray(x, dtype=dtype))
    return a, a.ctypes.data_as(ctypes.c_void_p)


def attention_window(q, k, v, kv_lens, sink, scale, causal, kv_begin, kv_end, threads=0):
    """Partial attention over keys [kv_begin, kv_end) ∩ visible set.

    q: bf16 [B, Hq, Tq, d]; k, v: bf16 [B, Hkv, Tkv, d]; kv_lens: int32 [B] or
    None (all Tkv); sink: float32 [Hq] or None.  Returns (out fp64 [B,Hq,Tq,d],
    lse fp64 [B,Hq,Tq])."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, Tq, d = qb.shape
    _, Hkv, Tkv, _ = kb.shape
    kl, klp = _opt(kv_lens, np.int32)
    sk, skp = _opt(sink, np.float32)
    out = np.zeros((B, Hq, Tq, d), np.float64)
    lse = np.zeros((B, Hq, Tq), np.float64)
    rc = _load().oracle_attention_window(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, klp, skp,
        out.ctypes.data, lse.ctypes.data, B, Hq, Hkv, Tq, Tkv, d, float(scale), int(bool(causal)),
        int(kv_begin), int(kv_end), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_window failed: %d" % rc)
    del kl, sk
    return out, lse


def attention(q, k, v, kv_lens=None, sink=None, scale=None, causal=False, threads=0):
    """The full forward (see the module docstring)."""
    d = _bits(q).shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    Tkv = _bits(k).shape[2]
    return attention_window(q, k, v, kv_lens, sink, scale, causal, 0, Tkv, threads)


def attention_rows(q, k, v, kv_lens, sink, scale, causal, rows, threads=0):
    """The full forward at flat rows ``(b*Hq + h)*Tq + i`` only.

    Returns (out fp64 [n, d], lse fp64 [n])."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, Tq, d = qb.shape
    _, Hkv, Tkv, _ = kb.shape
    kl, klp = _opt(kv_lens, np.int32)
    sk, skp = _opt(sink, np.float32)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((r.size, d), np.float64)
    lse = np.zeros((r.size,), np.float64)
    rc = _load().oracle_attention_rows(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, klp, skp, r.ctypes.data, r.size,
        out.ctypes.data, lse.ctypes.data, B, Hq, Hkv, Tq, Tkv, d, float(scale),
        int(bool(causal)), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_rows failed: %d" % rc)
    del kl, sk
    return out, lse


def combine(o_part, lse_part, sink=None):
    """LSE merge.  o_part: float32 [B, Hq, Tq, S, d]; lse_part: float32
    [B, Hq, Tq, S]; sink: float32 [Hq] or None.  Returns (out fp64 [B,Hq,Tq,d],
    lse fp64 [B,Hq,Tq])."""
    o, _ = _opt(o_part, np.float32)
    l, _ = _opt(lse_part, np.float32)
    B, Hq, Tq, S, d = o.shape
    assert l.shape == (B, Hq, Tq, S)
    sk, skp = _opt(sink, np.float32)
    out = np.zeros((B, Hq, Tq, d), np.float64)
    lse = np.zeros((B, Hq, Tq), np.float64)
    rc = _load().oracle_combine(o.ctypes.data, l.ctypes.data, S, skp, out.ctypes.data,
                                lse.ctypes.data, B, Hq, Tq, d)
    if rc != 0:
        raise ValueError("oracle_combine failed: %d" % rc)
    del sk
    return out, lse


def _bytes(x) -> np.ndarray:
    """E4M3 tensor/array (torch.float8_e4m3fn or uint8) -> contiguous uint8 bytes."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype != torch.uint8:
                assert x.dtype == torch.float8_e4m3fn
                x = x.view(torch.uint8)
            return np.ascontiguousarray(x.numpy())
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(x)
    assert a.dtype == np.uint8
    return np.ascontiguousarray(a)


def e4m3_decode(x) -> np.ndarray:
    """Values (fp64) of E4M3 bytes."""
    b = _bytes(x)
    out = np.zeros(b.shape, np.float64)
    _load().oracle_e4m3_decode(b.ctypes.data, out.ctypes.data, b.size)
    return out


def attention_fp8kv(q, k8, v8, k_scale, v_scale, kv_lens=None, sink=None, scale=None, causal=False, threads=0):
    """The full forward on K = value(k8) * k_scale, V = value(v8) * v_scale.

    q: bf16 [B, Hq, Tq, d]; k8, v8: E4M3 [B, Hkv, Tkv, d].  Returns (out fp64
    [B,Hq,Tq,d], lse fp64 [B,Hq,Tq])."""
    qb, kb, vb = _bits(q), _bytes(k8), _bytes(v8)
    B, Hq, Tq, d = qb.shape
    _, Hkv, Tkv, _ = kb.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    kl, klp = _opt(kv_lens, np.int32)
    sk, skp = _opt(sink, np.float32)
    out = np.zeros((B, Hq, Tq, d), np.float64)
    lse = np.zeros((B, Hq, Tq), np.float64)
    rc = _load().oracle_attention_window_fp8kv(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, float(k_scale), float(v_scale), klp, skp,
        out.ctypes.data, lse.ctypes.data, B, Hq, Hkv, Tq, Tkv, d, float(scale), int(bool(causal)),
        0, int(Tkv), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_window_fp8kv failed: %d" % rc)
    del kl, sk
    return out, lse


def attention_rows_fp8kv(q, k8, v8, k_scale, v_scale, kv_lens, sink, scale, causal, rows, threads=0):
    """attention_fp8kv at flat rows ``(b*Hq + h)*Tq + i`` only: (out fp64 [n, d], lse fp64 [n])."""
    qb, kb, vb = _bits(q), _bytes(k8), _bytes(v8)
    B, Hq, Tq, d = qb.shape
    _, Hkv, Tkv, _ = kb.shape
    kl, klp = _opt(kv_lens, np.int32)
    sk, skp = _opt(sink, np.float32)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((r.size, d), np.float64)
    lse = np.zeros((r.size,), np.float64)
    rc = _load().oracle_attention_rows_fp8kv(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, float(k_scale), float(v_scale), klp, skp,
        r.ctypes.data, r.size, out.ctypes.data, lse.ctypes.data, B, Hq, Hkv, Tq, Tkv, d, float(scale),
        int(bool(causal)), int(threads))
    if rc != 0:
        raise ValueError("oracle_attention_rows_fp8kv failed: %d" % rc)
    del kl, sk
    return out, lse
