"""The paged-cache input recipe (host side, no GPU): the pages, read back through
the page table, hold exactly the contiguous K/V of every logical position; table
entries past a sequence's pages are -1; spare pages are NaN and never referenced;
no physical page serves two (sequence, logical page) slots."""
import pytest
import torch

from gqa_attention_forward_flash_b200.synth import Workload, make_inputs, paginate


@pytest.mark.parametrize("page_size", [8, 16, 64, 128])
def test_pages_read_back_as_the_contiguous_cache(page_size):
    w = Workload("p", B=3, Hq=8, Hkv=2, Tq=1, Tkv=300, d=64, ragged=True, seed=31)
    inp = make_inputs(w)
    lens = inp.kv_lens.clone()
    lens[0] = 0
    lens[1] = w.Tkv
    kc, vc, table = paginate(inp.k, inp.v, lens, page_size, seed=4)
    num_pages, Hkv, ps, d = kc.shape
    assert (Hkv, ps, d) == (w.Hkv, page_size, w.d)
    assert table.dtype == torch.int32 and table.shape == (w.B, (w.Tkv + page_size - 1) // page_size)
    used = set()
    for b in range(w.B):
        n = int(lens[b])
        npg = (n + page_size - 1) // page_size
        assert torch.all(table[b, npg:] == -1)
        for j in range(npg):
            phys = int(table[b, j])
            assert 0 <= phys < num_pages and phys not in used
            used.add(phys)
            lo, hi = j * page_size, min((j + 1) * page_size, n)
            assert torch.equal(kc[phys, :, : hi - lo], inp.k[b, :, lo:hi])
            assert torch.equal(vc[phys, :, : hi - lo], inp.v[b, :, lo:hi])
    spare = [p for p in range(num_pages) if p not in used]
    assert len(spare) >= 1
    for p in spare:
        assert torch.isnan(kc[p].float()).all() and torch.isnan(vc[p].float()).all()


def test_fp8_input_recipe():
    """FP8 K/V inputs: E4M3 bytes with one scale per tensor, amax / 448 over the
    finite values; dequantised they stay within half an E4M3 step of the drawn
    bf16 values, and the NaN padding stays NaN."""
    import math

    import torch

    from gqa_attention_forward_flash_b200.synth import WORKLOADS, make_inputs, shrink
    w = shrink(WORKLOADS["batched_decode_fp8kv"], B=3, Tkv=257)
    inp = make_inputs(w)
    assert inp.k8.dtype == torch.float8_e4m3fn and inp.v8.dtype == torch.float8_e4m3fn
    for x, x8, sc in ((inp.k, inp.k8, inp.k_scale), (inp.v, inp.v8, inp.v_scale)):
        xf = x.float()
        fin = torch.isfinite(xf)
        assert math.isclose(sc, float(xf[fin].abs().max()) / 448.0, rel_tol=1e-7)
        deq = x8.float() * sc
        assert torch.equal(torch.isnan(deq), ~fin)
        # E4M3 keeps 3 mantissa bits: relative error at most 2^-4 for normal values
        err = (deq[fin] - xf[fin]).abs()
        assert bool((err <= xf[fin].abs() * 2.0 ** -4 + sc * 2.0 ** -10).all())
