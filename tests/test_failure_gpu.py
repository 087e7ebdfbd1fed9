"""Failure detection on the GPU without a fault: every wait inside the kernels is
bounded, and an expired wait records GQA_ERR_TIMEOUT, makes every role of the CTA
leave (in-flight copies drained, TMEM freed) and ends the launch; the host reads
the status and the next call works.

The wait that runs out here is a legitimate one: with one row-block split over
every CTA (one per SM), each CTA's ticket warp waits for its own split piece for
its whole span of 250 key tiles (a few hundred microseconds), and the wait limit
is set to 40 microseconds for that call (GQA_WAIT_TIMEOUT_US).  The limit is
counted in cycles of the nominal SM clock, so at a lower real clock it lasts
longer in wall time; the span is several times longer than the limit even at
half the clock."""
import pytest
import torch

from gqa_attention_forward_flash_b200 import binding
from gqa_attention_forward_flash_b200.synth import WORKLOADS, make_inputs, shrink

from parity import compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

TILES_PER_CTA = 250
LIMIT_US = 40


def test_an_expired_wait_is_reported_and_the_next_call_works(monkeypatch):
    dev = "cuda"
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, Hq, Hkv, Tq, d = 1, 8, 1, 1, 128
    Tkv = sms * TILES_PER_CTA * 128
    q = torch.zeros((B, Hq, Tq, d), dtype=torch.bfloat16, device=dev)
    k = torch.zeros((B, Hkv, Tkv, d), dtype=torch.bfloat16, device=dev)
    v = torch.zeros_like(k)
    monkeypatch.setenv("GQA_WAIT_TIMEOUT_US", str(LIMIT_US))
    binding.gqa_attention_fwd(q, k, v, None, None)
    err = binding.gqa_get_device_error()
    monkeypatch.delenv("GQA_WAIT_TIMEOUT_US")
    del k, v
    torch.cuda.empty_cache()
    assert err == -6, "expected GQA_ERR_TIMEOUT, got %d" % err
    # the error word and the merge tickets were reset by the read: a normal call is exact again
    assert binding.gqa_get_device_error() == 0
    inp = make_inputs(shrink(WORKLOADS["batched_decode"], B=3, Tkv=2000))
    o, l = run_gpu(inp)
    o_ref, l_ref = run_oracle(inp)
    compare(o, l, o_ref, l_ref, "after a timeout")
