"""The entry point that allocates nothing (fa_fwd_noalloc).

Some callers of this library cannot allocate device memory: a plugin whose
host framework owns every device allocation and passes only input and output
buffers, or a latency-bound path that must not call the CUDA allocator.
fa_fwd_noalloc serves them by keeping the dynamic schedule's scratch in a
fixed array inside the library.  This test calls it through the C ABI, twice
in a row (the second call must not be disturbed by what the first left in the
shared scratch), and checks each result against fa_fwd_ws with a
caller-provided workspace, within the tolerances of the parity tests.

The file is named so that pytest collects it last.
"""
import math

import pytest
import torch

import attention_forward_19_b200 as fa
from fa_inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu

O_TOL = {"fp16": 1e-2, "bf16": 2e-2}
LSE_TOL = 1e-3

CASES = [
    Workload("noalloc_bf16_bhsd_causal", "bf16", "BHSD", 2, 8, 3000, 3000, 128, True, 1 / math.sqrt(128), seed=11),
    Workload("noalloc_fp16_bsnd", "fp16", "BSND", 1, 6, 777, 1301, 64, False, 0.125, seed=12),
]


def _raw_call(entry, w, q, k, v, o, lse, stream, ws=None):
    lay = fa.LAYOUTS[w.layout]
    dt = fa.FA_BF16 if w.dtype == "bf16" else fa.FA_FP16
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
            w.B, w.H, w.Sq, w.Sk, w.D, lay, int(w.causal), w.scale, dt)
    if ws is None:
        return entry(*args, stream)
    return entry(*args, ws.data_ptr(), ws.numel(), stream)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_no_alloc_entry_matches_workspace_entry(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    q, k, v = make_qkv(w, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    o_ref, l_ref = torch.empty_like(q), torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_fwd_workspace_size(), dtype=torch.uint8, device="cuda")
    assert _raw_call(fa.fa_fwd_ws, w, q, k, v, o_ref, l_ref, stream, ws) == fa.FA_OK
    outs = []
    for _ in range(2):
        o, lse = torch.full_like(q, float("nan")), torch.full((w.B, w.H, w.Sq), float("nan"), device="cuda")
        assert _raw_call(fa.fa_fwd_noalloc, w, q, k, v, o, lse, stream) == fa.FA_OK
        outs.append((o, lse))
    assert fa.fa_device_status(stream) == fa.FA_OK
    for o, lse in outs:
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert (o.float() - o_ref.float()).abs().max().item() <= O_TOL[w.dtype]
        assert (lse - l_ref).abs().max().item() <= LSE_TOL
