"""GPU parity of the split-KV forward (fa_fwd_splitkv): the key range of every
query row split across CTAs and the partial results merged by a second kernel.

Against the fp64 oracle on the same inputs, with the forward's bounds (max
|O - O_oracle| <= 1e-2 fp16 / 2e-2 bf16, max |LSE - LSE_oracle| <= 1e-3):
the c1 workload (fp16 BSND 1x512x2x64) at several split counts, a
decoding-like shape (one query row against 16,001 keys), splits that end
inside a key tile and key ranges shorter than the requested split count.
Against fa_fwd on the same inputs: the same bounds (the partials are fp32,
so the two differ by rounding only).
"""
import math

import numpy as np
import pytest
import torch

import attention_forward_19_b200 as fa
from fa_inputs import WORKLOADS, Workload, make_qkv

pytestmark = pytest.mark.gpu

O_TOL = {"fp16": 1e-2, "bf16": 2e-2}
LSE_TOL = 1e-3


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _bhsd(x, layout):
    return x.permute(0, 2, 1, 3) if layout == "BSND" else x


CASES = [
    # name, workload, nsplit
    ("c1_n1", WORKLOADS["fp16_bsnd_b1_h2_s512_d64"], 1),
    ("c1_n2", WORKLOADS["fp16_bsnd_b1_h2_s512_d64"], 2),
    ("c1_n4", WORKLOADS["fp16_bsnd_b1_h2_s512_d64"], 4),
    ("ragged_bf16", Workload("bf16_bhsd_b2_h3_q300_k5000", "bf16", "BHSD", 2, 3, 300, 5000, 128, False,
                             1.0 / math.sqrt(128)), 8),
    ("decode_fp16", Workload("fp16_bsnd_b1_h4_q1_k16001_d64", "fp16", "BSND", 1, 4, 1, 16001, 64, False, 0.125), 16),
    ("many_splits", Workload("bf16_bsnd_b1_h8_q129_k4096", "bf16", "BSND", 1, 8, 129, 4096, 128, False,
                             1.0 / math.sqrt(128)), 64),
    ("fewer_tiles_than_splits", Workload("fp16_bhsd_b1_h2_q200_k100", "fp16", "BHSD", 1, 2, 200, 100, 128, False,
                                         1.0 / math.sqrt(128)), 8),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_splitkv_matches_oracle_and_fa_fwd(orc, case):
    _need_gpu()
    name, w, nsplit = case
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = fa.flash_attention_forward_splitkv(qd, kd, vd, layout=w.layout, scale=w.scale, nsplit=nsplit)
    fa.check_device_status()
    o_ref, lse_ref = orc.fwd(q, k, v, layout=w.layout, causal=False, scale=float(np.float32(w.scale)))
    o_gpu = _bhsd(o.cpu(), w.layout).double().numpy()
    lse_gpu = lse.cpu().double().numpy()
    eo = float(np.max(np.abs(o_gpu - o_ref)))
    el = float(np.max(np.abs(lse_gpu - lse_ref)))
    print(f"PARITY splitkv {name} (nsplit {nsplit}): max|dO| {eo:.3e} max|dLSE| {el:.3e}")
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(lse_gpu))
    assert eo <= O_TOL[w.dtype] and el <= LSE_TOL
    # against the one-pass kernel on the same inputs
    o1, l1 = fa.flash_attention_forward(qd, kd, vd, layout=w.layout, causal=False, scale=w.scale)
    fa.check_device_status()
    assert float((o1.double() - o.double()).abs().max()) <= O_TOL[w.dtype]
    assert float((l1.double() - lse.double()).abs().max()) <= LSE_TOL


def test_splitkv_reuses_a_larger_workspace_and_overwrites_outputs():
    _need_gpu()
    w = WORKLOADS["fp16_bsnd_b1_h2_s512_d64"]
    q, k, v = (t.cuda() for t in make_qkv(w))
    ws = torch.empty(fa.fa_fwd_splitkv_workspace_size(w.B, w.H, w.Sq, w.D, 8) + 4096, dtype=torch.uint8,
                     device="cuda")
    ref_o, ref_l = fa.flash_attention_forward_splitkv(q, k, v, layout=w.layout, scale=w.scale, nsplit=4)
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.H, w.Sq), float("nan"), device="cuda")
    for n in (4, 4, 8):
        fa.flash_attention_forward_splitkv(q, k, v, layout=w.layout, scale=w.scale, nsplit=n, out=out, lse=lse,
                                           workspace=ws)
        fa.check_device_status()
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        if n == 4:   # the same split count, the same kernels: the same bits
            assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
