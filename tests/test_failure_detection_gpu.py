"""Failure detection on the GPU without a fault: every wait in the kernel is
bounded, and a wait that runs out is reported as FA_ERR_TIMEOUT while the CUDA
context stays usable.

fa_selftest_wait_timeout launches the kernel with its loads withheld (nothing
is in flight, so the CTAs drain at once) and a 20 ms wait limit; the
consumers' waits for Q and K / V run out.
"""
import math

import pytest
import torch

import attention_forward_19_b200 as fa
from fa_inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("dtype,layout,D,causal", [("bf16", "BHSD", 128, True), ("fp16", "BSND", 64, False)])
def test_bounded_waits_time_out_and_context_survives(dtype, layout, D, causal):
    _need_gpu()
    w = Workload("selftest", dtype, layout, 1, 3, 1000, 1000, D, causal, 1 / math.sqrt(D), seed=11)
    q, k, v = (t.cuda() for t in make_qkv(w))
    stream = torch.cuda.current_stream()
    o1, lse1 = fa.flash_attention_forward(q, k, v, layout=layout, causal=causal, scale=w.scale)
    fa.check_device_status()

    o_s = torch.full_like(o1, 7.0)
    lse_s = torch.full_like(lse1, 7.0)
    lay = fa.FA_BHSD if layout == "BHSD" else fa.FA_BSND
    dt = fa.FA_BF16 if dtype == "bf16" else fa.FA_FP16
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    st = fa.fa_selftest_wait_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_s.data_ptr(), lse_s.data_ptr(),
                                     w.B, w.H, w.Sq, w.Sk, w.D, lay, causal, w.scale, dt, 20000,
                                     stream.cuda_stream)
    e1.record(stream)
    assert st == fa.FA_OK
    assert fa.fa_device_status(stream.cuda_stream) == fa.FA_ERR_TIMEOUT
    # the kernel returned after about one wait limit, not hung
    assert e0.elapsed_time(e1) < 2000.0
    # nothing was written
    assert bool((o_s == 7.0).all()) and bool((lse_s == 7.0).all())
    # the error word was cleared, and the context still computes the same result
    assert fa.fa_device_status(stream.cuda_stream) == fa.FA_OK
    o2, lse2 = fa.flash_attention_forward(q, k, v, layout=layout, causal=causal, scale=w.scale)
    fa.check_device_status()
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)
