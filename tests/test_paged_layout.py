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
