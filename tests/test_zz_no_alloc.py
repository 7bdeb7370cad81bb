"""The entry point that allocates nothing (fa_fwd_noalloc).

Some callers of this library cannot allocate device memory: a plugin whose
host framework owns every device allocation and passes only input and output
buffers, or a latency-bound path that must not call the CUDA allocator.
fa_fwd_noalloc serves them by keeping the dynamic schedule's scratch in a
fixed array inside the library.  This test calls it through the C ABI, twice
in a row (the second call must not be disturbed by what the first left in the
shared scratch), and checks each result against fa_fwd_ws with a
caller-provided workspace.  Both run the same kernel with the same work
units, and a unit's result does not depend on which CTA computes it, so the
outputs must be bit-identical; the tolerances of the parity tests, and one
direct comparison with the fp64 oracle, are checked as well.

The file is named so that pytest collects it last.
"""
import math

import numpy as np
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
        # the same kernel and the same units: the same bits
        assert torch.equal(o, o_ref)
        assert torch.equal(lse, l_ref)


def test_no_alloc_entry_against_oracle():
    """One element-by-element comparison of fa_fwd_noalloc's output with the fp64 oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from oracle import attn
    w = Workload("noalloc_bf16_bsnd_causal_small", "bf16", "BSND", 1, 3, 700, 700, 128, True,
                 1 / math.sqrt(128), seed=13)
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = torch.empty_like(qd), torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert _raw_call(fa.fa_fwd_noalloc, w, qd, kd, vd, o, lse, stream) == fa.FA_OK
    assert fa.fa_device_status(stream) == fa.FA_OK
    o_ref, lse_ref = attn.default().fwd(q, k, v, layout=w.layout, causal=w.causal, scale=float(np.float32(w.scale)))
    o_gpu = o.cpu().permute(0, 2, 1, 3).to(torch.float64).numpy()
    assert np.max(np.abs(o_gpu - o_ref)) <= O_TOL[w.dtype]
    assert np.max(np.abs(lse.cpu().to(torch.float64).numpy() - lse_ref)) <= LSE_TOL
