"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_attn.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return binding.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gqa_attention_fwd", "gqa_splitkv_combine", "gqa_attention_fwd_partial"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in binding.SIGNATURES, name


def test_exported_symbols_are_c_linkage():
    out = os.popen("nm -D --defined-only %s" % binding.LIB_PATH).read()
    for name in declared_functions():
        assert re.search(r"\bT %s$" % name, out, flags=re.M), name


def test_version_and_status_strings(lib):
    assert lib.gqa_version() >= 100
    for code in binding.STATUS:
        assert lib.gqa_status_string(code)


P = ctypes.c_void_p


def fwd(lib, q=16, k=16, v=16, kv=None, sink=None, out=16, lse=16, B=1, Hq=4, Hkv=1, Tq=4, Tkv=8, d=64,
        scale=0.125, causal=0):
    return lib.gqa_attention_fwd(P(q), P(k), P(v), P(kv), P(sink), P(out), P(lse), B, Hq, Hkv, Tq, Tkv, d,
                                 scale, causal, None)


def test_shape_errors(lib):
    assert fwd(lib, Hq=6, Hkv=4) == -2          # Hq % Hkv
    assert fwd(lib, Tkv=0) == -2                # no key buffer
    assert fwd(lib, B=-1) == -2
    assert fwd(lib, Hkv=0) == -2
    assert fwd(lib, d=96) == -7                 # unsupported head dim
    assert fwd(lib, scale=0.0) == -2            # the scale must be positive and finite
    assert fwd(lib, scale=-1.0) == -2
    assert fwd(lib, scale=float("inf")) == -2
    assert fwd(lib, B=1 << 20, Hq=1 << 10, Hkv=1 << 10, Tkv=1 << 12) == -2  # index overflow


def test_null_and_alignment_errors(lib):
    assert fwd(lib, q=0) == -1
    assert fwd(lib, out=0) == -1
    assert fwd(lib, k=24) == -3
    assert fwd(lib, out=8) == -3


def test_empty_problem_is_a_no_op(lib):
    assert fwd(lib, B=0, q=0, k=0, v=0, out=0) == 0
    assert fwd(lib, Tq=0, q=0, k=0, v=0, out=0) == 0


def test_partial_and_combine_argument_errors(lib):
    f = lib.gqa_attention_fwd_partial
    assert f(P(16), P(16), P(16), None, 1, 4, 1, 4, 8, 64, 0.1, 0, 0, P(16), P(16), None) == -4
    assert f(P(16), P(16), P(16), None, 1, 4, 1, 4, 8, 64, 0.1, 0, 257, P(16), P(16), None) == -4
    assert f(P(16), P(16), P(16), None, 1, 4, 1, 4, 8, 64, 0.1, 0, 2, None, P(16), None) == -1
    c = lib.gqa_splitkv_combine
    assert c(P(16), P(16), 0, None, P(16), P(16), 1, 4, 4, 64, None) == -4
    assert c(P(16), P(16), 2, None, P(16), P(16), 1, 4, 4, 66, None) == -2
    assert c(None, P(16), 2, None, P(16), P(16), 1, 4, 4, 64, None) == -1
    assert c(P(16), P(16), 2, None, P(24), P(16), 1, 4, 4, 64, None) == -3


def test_valid_call_without_a_gpu_fails_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert fwd(lib) == -5  # GQA_ERR_CUDA: no silent CPU path


def paged(lib, page_size=64, d=64, table=16, lens=16, num_pages=8, max_pages=4):
    return lib.gqa_attention_fwd_paged(P(16), P(16), P(16), P(table), P(lens), None, P(16), P(16), 1, 4, 1, 4,
                                       num_pages, page_size, max_pages, d, 0.125, 0, None)


def test_paged_entry_rejects_bad_arguments_on_the_host(lib):
    assert paged(lib, page_size=48) == -2      # not a power of two
    assert paged(lib, page_size=4) == -2       # below 8
    assert paged(lib, page_size=2048) == -2    # above 1024
    assert paged(lib, num_pages=0) == -2
    assert paged(lib, max_pages=0) == -2
    assert paged(lib, d=256) == -7             # only head dims 64 and 128
    assert paged(lib, table=None) == -1        # page table required
    assert paged(lib, lens=None) == -1         # kv_lens required


def test_shard_entry_points_reject_bad_arguments_on_the_host(lib):
    s = lib.gqa_shard_lengths
    assert s(P(16), -1, 0, 8, P(16), None) == -2          # negative batch
    assert s(P(16), 2, -3, 8, P(16), None) == -2          # negative offset
    assert s(P(16), 2, 0, -1, P(16), None) == -2          # negative capacity
    assert s(None, 2, 0, 8, P(16), None) == -1
    assert s(P(16), 0, 0, 8, None, None) == 0             # nothing to do
    c = lib.gqa_combine_shards
    rows_d = 1 * 4 * 2 * 64
    assert c(P(16), rows_d, P(16), 8, 0, None, P(16), P(16), 1, 4, 2, 64, None) == -4      # no shard
    assert c(P(16), rows_d, P(16), 8, 257, None, P(16), P(16), 1, 4, 2, 64, None) == -4    # too many
    assert c(P(16), rows_d, P(16), 8, 2, None, P(16), P(16), 1, 4, 2, 66, None) == -2      # d % 4
    assert c(P(16), rows_d - 4, P(16), 8, 2, None, P(16), P(16), 1, 4, 2, 64, None) == -2  # shards overlap
    assert c(P(16), rows_d, P(16), 7, 2, None, P(16), P(16), 1, 4, 2, 64, None) == -2      # lse shards overlap
    assert c(P(16), rows_d + 2, P(16), 8, 2, None, P(16), P(16), 1, 4, 2, 64, None) == -3  # stride not 8-byte
    assert c(P(24), rows_d, P(16), 8, 2, None, P(16), P(16), 1, 4, 2, 64, None) == -3      # base misaligned
    assert c(None, rows_d, P(16), 8, 2, None, P(16), P(16), 1, 4, 2, 64, None) == -1


def test_binding_wrappers_validate_before_calling(lib):
    """Every wrapper checks dtype, rank, contiguity and device before the C call
    (a wrong tensor never reaches a kernel); CPU tensors are refused here."""
    import torch
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    q = torch.zeros((1, 4, 2, 64), dtype=bf)
    k = torch.zeros((1, 1, 8, 64), dtype=bf)
    op = torch.zeros((1, 4, 2, 3, 64), dtype=f32)
    lp = torch.zeros((1, 4, 2, 3), dtype=f32)
    with pytest.raises(ValueError):
        binding.gqa_attention_fwd_partial(q, k, k, num_splits=3)
    with pytest.raises(ValueError):
        binding.gqa_attention_fwd_partial(q.float(), k, k, num_splits=3)
    with pytest.raises(ValueError):
        binding.gqa_splitkv_combine(op, lp)
    with pytest.raises(ValueError):
        binding.gqa_splitkv_combine(op.double(), lp)
    with pytest.raises(ValueError):
        binding.gqa_splitkv_combine(op.transpose(3, 4), lp)
    with pytest.raises(ValueError):
        binding.gqa_attention_fwd_noalloc(q, k, k)
    with pytest.raises(ValueError):
        binding.gqa_attention_fwd(q, k, k, kv_lens=torch.zeros(1, dtype=i32))


def test_fp8kv_entry_rejects_bad_arguments_on_the_host(lib):
    f = lib.gqa_attention_fwd_fp8kv
    args = lambda ks=1.0, vs=1.0, d=128, Hq=8, Tq=1: (P(16), P(16), P(16), ks, vs, None, None, P(16), P(16), 1, Hq, 1,
                                                      Tq, 8, d, 0.125, 0, None)
    assert f(*args(ks=0.0)) == -2
    assert f(*args(vs=-1.0)) == -2
    assert f(*args(ks=float("inf"))) == -2
    assert f(*args(d=64)) == -7
    assert f(*args(Hq=32)) == -7      # 32 packed rows: not a decode shape
    assert f(*args(Tq=3)) == -7       # 8 heads x 3 rows = 24 packed rows
