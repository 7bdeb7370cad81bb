"""fa_fwd_heads on the GPU: the head ranges of several ranks, emulated one
after another on one GPU (independent launches; no launch waits on another).

Each range's launch must write exactly its own heads' rows of O and LSE and
leave every other element untouched, and the ranges together must give the
single-call result bit for bit (a head's result does not depend on the launch
that computes it).  One case is also compared with the fp64 oracle.
"""
import math

import numpy as np
import pytest
import torch

import attention_forward_19_b200 as fa
from attention_forward_19_b200 import shard
from fa_inputs import WORKLOADS, Workload, make_qkv

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


CASES = [
    (Workload("heads_bf16_bhsd_c", "bf16", "BHSD", 2, 5, 700, 700, 128, True, 1 / math.sqrt(128), seed=61), 3),
    (Workload("heads_fp16_bsnd_n", "fp16", "BSND", 3, 3, 333, 901, 64, False, 0.125, seed=62), 2),
    (Workload("heads_bf16_bsnd_c", "bf16", "BSND", 2, 3, 1000, 1000, 128, True, 1 / math.sqrt(128), seed=63), 4),
    (Workload("heads_fp16_bhsd_c_d64", "fp16", "BHSD", 1, 7, 257, 513, 64, True, 0.125, seed=64), 8),
    (WORKLOADS["bf16_bhsd_b2_h40_s8192_d128_causal"], 8),
]


def _nan_like(q, w):
    return torch.full_like(q, float("nan")), torch.full((w.B, w.H, w.Sq), float("nan"), device=q.device)


@pytest.mark.parametrize("w,world", CASES, ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_head_ranges_write_only_their_rows_and_assemble_bitwise(w, world):
    _need_gpu()
    q, k, v = make_qkv(w, device="cuda")
    o_ref, l_ref = fa.flash_attention_forward(q, k, v, layout=w.layout, causal=w.causal, scale=w.scale)
    ranges = shard.head_ranges(w.B, w.H, w.Sq, w.Sk, w.causal, world)
    o, lse = _nan_like(q, w)
    for r, (begin, count) in enumerate(ranges):
        sched = "dynamic" if r % 2 == 0 else "static"
        fa.flash_attention_forward(q, k, v, layout=w.layout, causal=w.causal, scale=w.scale, out=o, lse=lse,
                                   schedule=sched, heads=(begin, count))
        fa.check_device_status()
        if r == 0:
            # only rank 0's rows are written so far, and they are the single call's bits
            done_o = torch.zeros_like(o, dtype=torch.bool)
            done_l = torch.zeros_like(lse, dtype=torch.bool)
            for t, d in ((o, done_o), (lse, done_l)):
                for view in shard.head_rows(d, begin, count, w.layout, w.H):
                    view.fill_(True)
            assert torch.equal(o[done_o], o_ref[done_o]) and torch.equal(lse[done_l], l_ref[done_l])
            assert bool(torch.isnan(o[~done_o].float()).all()) and bool(torch.isnan(lse[~done_l]).all())
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_head_range_against_oracle(orc):
    _need_gpu()
    w = Workload("heads_oracle", "bf16", "BSND", 2, 3, 400, 400, 128, True, 1 / math.sqrt(128), seed=65)
    q, k, v = make_qkv(w)
    o, lse = _nan_like(q.cuda(), w)
    begin, count = 2, 3                                    # heads (0,2), (1,0), (1,1): crosses a batch
    fa.flash_attention_forward(q.cuda(), k.cuda(), v.cuda(), layout=w.layout, causal=True, scale=w.scale, out=o,
                               lse=lse, heads=(begin, count))
    fa.check_device_status()
    rows = np.arange(begin * w.Sq, (begin + count) * w.Sq, dtype=np.int64)
    o_ref, l_ref = orc.fwd(q, k, v, layout=w.layout, causal=True, scale=float(np.float32(w.scale)), rows=rows)
    ob = o.cpu().permute(0, 2, 1, 3).reshape(w.B * w.H * w.Sq, w.D)[rows].to(torch.float64).numpy()
    lb = lse.cpu().reshape(-1)[rows].to(torch.float64).numpy()
    assert np.max(np.abs(ob - o_ref)) <= 2e-2 and np.max(np.abs(lb - l_ref)) <= 1e-3


def test_empty_and_invalid_ranges():
    _need_gpu()
    w = Workload("heads_err", "fp16", "BHSD", 1, 2, 128, 128, 64, False, 0.125, seed=66)
    q, k, v = make_qkv(w, device="cuda")
    o, lse = _nan_like(q, w)
    fa.flash_attention_forward(q, k, v, layout="BHSD", scale=w.scale, out=o, lse=lse, heads=(1, 0))
    fa.check_device_status()
    assert bool(torch.isnan(o.float()).all())
    for bad in ((-1, 1), (0, 3), (2, 1), (1, -1)):
        with pytest.raises(fa.FaError) as e:
            fa.flash_attention_forward(q, k, v, layout="BHSD", scale=w.scale, out=o, lse=lse, heads=bad)
        assert e.value.status == fa.FA_ERR_INVALID_ARG
