"""Failure detection on the GPU without a fault: every wait inside the kernels is
bounded, and an expired wait records GQA_ERR_TIMEOUT, makes every role of the CTA
leave (in-flight copies drained, TMEM freed) and ends the launch; the host reads
the status and the next call works.

The wait that runs out here is a legitimate one: with one row-block split over
every CTA, each CTA's ticket warp waits for its own split piece for the whole
span (about a millisecond at this size), and the wait limit is set to 1 ms for
that call (GQA_WAIT_TIMEOUT_MS)."""
import pytest
import torch

from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200.synth import WORKLOADS, make_inputs, shrink

from parity import compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def test_an_expired_wait_is_reported_and_the_next_call_works(monkeypatch):
    dev = "cuda"
    B, Hq, Hkv, Tq, d = 1, 8, 1, 1, 128
    Tkv = 148 * 900 * 128  # 900 key tiles per CTA
    q = torch.zeros((B, Hq, Tq, d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((B, Hkv, Tkv, d), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    k.zero_()
    v.zero_()
    monkeypatch.setenv("GQA_WAIT_TIMEOUT_MS", "1")
    binding.gqa_attention_fwd(q, k, v, None, None)
    err = binding.gqa_get_device_error()
    monkeypatch.delenv("GQA_WAIT_TIMEOUT_MS")
    del k, v
    torch.cuda.empty_cache()
    assert err == -6, "expected GQA_ERR_TIMEOUT, got %d" % err
    # the error word and the merge tickets were reset by the read: a normal call is exact again
    assert binding.gqa_get_device_error() == 0
    inp = make_inputs(shrink(WORKLOADS["batched_decode"], B=3, Tkv=2000))
    o, l = run_gpu(inp)
    o_ref, l_ref = run_oracle(inp)
    compare(o, l, o_ref, l_ref, "after a timeout")
