"""GPU parity of the packed variable-length entry (fa_fwd_varlen) against the
fp64 oracle, per sequence, through the C ABI.

Bounds as for the dense path: max |O_gpu - O_oracle| <= 1e-2 (fp16) / 2e-2
(bf16), max |LSE_gpu - LSE_oracle| <= 1e-3.  Length mixes cover empty query
sequences, one-row sequences, tiles that end one row before / after a tile
boundary, and Sq != Sk within a sequence.  Also: a packed batch of equal
lengths is bit-identical to the dense BSND run of the same memory, the static
and dynamic schedules agree bitwise, and invalid offsets are reported without
touching the other sequences.
"""
import math

import numpy as np
import pytest
import torch

import attention_forward_19_b200 as fa
from fa_inputs import VARLEN_WORKLOADS, VarlenWorkload, Workload, make_qkv, make_varlen_qkv

pytestmark = pytest.mark.gpu

O_TOL = {"fp16": 1e-2, "bf16": 2e-2}
LSE_TOL = 1e-3


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def V(dtype, D, causal, lengths, H=2, qk_std=1.0, seed=5):
    name = f"{dtype}_d{D}_{'c' if causal else 'n'}_{len(lengths)}seq"
    return VarlenWorkload(name, dtype, H, D, causal, 1.0 / math.sqrt(D), lengths=tuple(lengths),
                          qk_std=qk_std, seed=seed)


CASES = [
    V("bf16", 128, True, [(1000, 1000), (1, 1), (257, 257), (0, 5), (128, 128), (3000, 3000), (129, 129)]),
    V("bf16", 128, False, [(300, 1000), (1000, 300), (7, 2), (256, 4096), (255, 1)]),
    V("bf16", 128, True, [(300, 1000), (1000, 300), (513, 511)], H=3),
    V("fp16", 64, True, [(513, 257), (255, 255), (1, 700), (384, 384)]),
    V("fp16", 128, False, [(127, 127), (128, 128), (129, 129), (0, 0), (2, 2000)]),
    V("bf16", 128, False, [(700, 700), (1500, 1500)], H=4, qk_std=3.0),
]


def run_varlen(w, q, k, v, cu_q, cu_k, schedule="dynamic"):
    o, lse = fa.flash_attention_varlen_forward(q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(),
                                               causal=w.causal, scale=w.scale, schedule=schedule)
    fa.check_device_status()
    return o, lse


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_varlen_matches_oracle(orc, w):
    _need_gpu()
    q, k, v, cu_q, cu_k = make_varlen_qkv(w)
    o, lse = run_varlen(w, q, k, v, cu_q, cu_k)
    o_ref, lse_ref = orc.fwd_varlen(q, k, v, cu_q.tolist(), cu_k.tolist(), causal=w.causal,
                                    scale=float(np.float32(w.scale)))
    og = o.cpu().to(torch.float64).numpy()
    lg = lse.cpu().to(torch.float64).numpy()
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(lg))
    eo = np.max(np.abs(og - o_ref))
    el = np.max(np.abs(lg - lse_ref))
    print(f"PARITY varlen {w.name}: max|dO| {eo:.3e} max|dLSE| {el:.3e}")
    assert eo <= O_TOL[w.dtype] and el <= LSE_TOL


def test_varlen_workload_sampled_rows(orc):
    """The 16-sequence packed workload (55k rows, 32 heads), on the first and last
    16 rows and every 211th row of every sequence."""
    _need_gpu()
    w = VARLEN_WORKLOADS["bf16_varlen_n16_h32_d128_causal"]
    q, k, v, cu_q, cu_k = make_varlen_qkv(w)
    o, lse = run_varlen(w, q, k, v, cu_q, cu_k)
    cq = cu_q.tolist()
    rows = set()
    for b in range(len(cq) - 1):
        rows.update(range(cq[b], min(cq[b] + 16, cq[b + 1])))
        rows.update(range(cq[b], cq[b + 1], 211))
        rows.update(range(max(cq[b], cq[b + 1] - 16), cq[b + 1]))
    rows = np.array(sorted(rows), dtype=np.int64)
    o_ref, lse_ref = orc.fwd_varlen(q, k, v, cq, cu_k.tolist(), causal=w.causal, scale=float(np.float32(w.scale)),
                                    rows=rows)
    idx = torch.from_numpy(rows).cuda()
    og = o.index_select(0, idx).cpu().to(torch.float64).numpy()
    lg = lse.index_select(1, idx).cpu().to(torch.float64).numpy()
    eo = np.max(np.abs(og - o_ref))
    el = np.max(np.abs(lg - lse_ref))
    print(f"PARITY varlen {w.name}: max|dO| {eo:.3e} max|dLSE| {el:.3e} ({len(rows)} rows)")
    assert eo <= O_TOL[w.dtype] and el <= LSE_TOL


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_match_dense_bitwise(causal):
    """Packed sequences of one length are the dense BSND batch of the same memory."""
    _need_gpu()
    w = Workload("eq", "bf16", "BSND", 3, 4, 700, 700, 128, causal, 1 / math.sqrt(128), seed=9)
    q, k, v = (t.cuda() for t in make_qkv(w))
    o_d, lse_d = fa.flash_attention_forward(q, k, v, layout="BSND", causal=causal, scale=w.scale)
    cu = torch.arange(0, 4 * 700, 700, dtype=torch.int32, device="cuda")
    o_v, lse_v = fa.flash_attention_varlen_forward(q.reshape(-1, 4, 128), k.reshape(-1, 4, 128),
                                                   v.reshape(-1, 4, 128), cu, cu, causal=causal, scale=w.scale)
    fa.check_device_status()
    assert torch.equal(o_v.reshape(o_d.shape), o_d)
    # dense lse [B, H, S]; packed lse [H, B*S]
    assert torch.equal(lse_v.reshape(4, 3, 700).permute(1, 0, 2), lse_d)


def test_static_and_dynamic_schedules_agree_bitwise():
    _need_gpu()
    w = CASES[0]
    q, k, v, cu_q, cu_k = make_varlen_qkv(w)
    o1, l1 = run_varlen(w, q, k, v, cu_q, cu_k, schedule="static")
    o2, l2 = run_varlen(w, q, k, v, cu_q, cu_k, schedule="dynamic")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_invalid_offsets_reported_and_isolated(orc):
    """A sequence whose offsets decrease, or that is longer than max_seqlen, is skipped
    (its rows untouched) and reported as FA_ERR_INVALID_ARG; the others are computed."""
    _need_gpu()
    w = V("bf16", 128, True, [(300, 300), (200, 200), (400, 400)])
    q, k, v, cu_q, cu_k = make_varlen_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o_ref, l_ref = orc.fwd_varlen(q, k, v, cu_q.tolist(), cu_k.tolist(), causal=True,
                                  scale=float(np.float32(w.scale)))
    bad_k = cu_k.clone()
    bad_k[2] = bad_k[1] - 1              # sequence 1: keys [300, 299) decrease
    out = torch.full_like(qd, 5.0)
    lse = torch.full((w.H, qd.shape[0]), 5.0, device="cuda")
    fa.flash_attention_varlen_forward(qd, kd, vd, cu_q.cuda(), bad_k.cuda(), max_seqlen_q=400, max_seqlen_k=400,
                                      causal=True, scale=w.scale, out=out, lse=lse)
    assert fa.fa_device_status(torch.cuda.current_stream().cuda_stream) == fa.FA_ERR_INVALID_ARG
    assert bool((out[300:500] == 5.0).all()) and bool((lse[:, 300:500] == 5.0).all())
    # sequence 2 still reads its own keys [299, 699): compare it on its own rows
    keep = np.r_[0:300]
    og = out.cpu().to(torch.float64).numpy()
    assert np.max(np.abs(og[keep] - o_ref[keep])) <= O_TOL["bf16"]
    # a length beyond max_seqlen_q is reported too
    out2 = torch.empty_like(qd)
    lse2 = torch.empty((w.H, qd.shape[0]), device="cuda")
    fa.flash_attention_varlen_forward(qd, kd, vd, cu_q.cuda(), cu_k.cuda(), max_seqlen_q=300, max_seqlen_k=400,
                                      causal=True, scale=w.scale, out=out2, lse=lse2)
    assert fa.fa_device_status(torch.cuda.current_stream().cuda_stream) == fa.FA_ERR_INVALID_ARG
    assert np.max(np.abs(out2[:500].cpu().to(torch.float64).numpy() - o_ref[:500])) <= O_TOL["bf16"]
    # and the next valid call is clean
    run_varlen(w, q, k, v, cu_q, cu_k)


def test_host_arguments_checked():
    _need_gpu()
    q = torch.zeros(10, 2, 128, dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, 10], dtype=torch.int32, device="cuda")
    with pytest.raises(fa.FaError):
        fa.flash_attention_varlen_forward(q, q, q, cu, cu, max_seqlen_q=11, max_seqlen_k=10)
    with pytest.raises(fa.FaError):
        fa.flash_attention_varlen_forward(q, q.cpu(), q, cu, cu, max_seqlen_q=10, max_seqlen_k=10)
