"""GPU parity of ring (context-parallel) attention and of its merge kernel.

* fa_lse_merge against the oracle's merge (oracle/merge.py) on the same
  inputs, for every flag combination, both layouts, D = 64 and 128 and ragged
  row counts, including rows whose LSE is -inf.  The kernel works in fp32:
  bound 1e-5 relative for the running result and the LSE, and, for the 16-bit
  output, one unit in the last place of the output type.
* fa_fwd_ring_step (a ring step's blocks attended and merged in one launch)
  against the same step composed of oracle blocks and oracle merges in fp64
  (ring.BlockwiseStep), over several steps: causal masks offset by whole
  chunks, a segment starting at a later key chunk, first / last flags, the
  running result (fp32 O and LSE) after a step and the final output, ragged
  chunk sizes, D = 64 and 128, both dtypes and layouts.
* The ring schedule of W ranks emulated on one GPU (the same fa_fwd_ring_step
  launches as the distributed run; only the transfers are replaced by
  lookups) against whole-sequence attention from the fp64 oracle, with the
  forward's bounds: max |O - O_oracle| <= 2e-2 (bf16) / 1e-2 (fp16), max
  |LSE - LSE_oracle| <= 1e-3.  Chunk sizes include ragged ones (not multiples
  of 128 rows), and the 64K-row, 8-head causal workload split over 8 ranks is
  checked on sampled rows.
"""
import math

import numpy as np
import pytest
import torch

import attention_forward_19_b200 as fa
from attention_forward_19_b200 import ring
from oracle.merge import merge_partials
from ring_oracle_ops import OracleOps

pytestmark = pytest.mark.gpu

O_TOL = {torch.float16: 1e-2, torch.bfloat16: 2e-2}
LSE_TOL = 1e-3
ULP = {torch.float16: 2.0 ** -10, torch.bfloat16: 2.0 ** -7}


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _head_major(t, layout):
    t = t.double().cpu()
    return (t.permute(0, 2, 1, 3) if layout == "BSND" else t).numpy()


def _partials(layout, dtype, B, H, S, D, seed):
    g = torch.Generator().manual_seed(seed)
    shape = (B, S, H, D) if layout == "BSND" else (B, H, S, D)
    o_part = (torch.randn(shape, generator=g) * 2).to(dtype)
    o_acc = torch.randn(shape, generator=g) * 2
    lse_part = torch.randn((B, H, S), generator=g) * 6
    lse_acc = torch.randn((B, H, S), generator=g) * 6
    lse_part[0, 0, :3] = -math.inf           # rows with an empty block
    lse_acc[0, -1, -2:] = -math.inf
    if S > 5:
        lse_part[0, 0, 5] = lse_acc[0, 0, 5] = -math.inf
    return o_part, lse_part, o_acc, lse_acc


@pytest.mark.parametrize("layout", ["BSND", "BHSD"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D,S", [(128, 1000), (64, 129), (128, 1)])
@pytest.mark.parametrize("accumulate,final", [(False, False), (True, False), (True, True), (False, True)])
def test_merge_kernel_matches_oracle_merge(layout, dtype, D, S, accumulate, final):
    _need_gpu()
    B, H = 2, 3
    o_part, lse_part, o_acc, lse_acc = _partials(layout, dtype, B, H, S, D, seed=S + D)
    acc_d, lacc_d = o_acc.cuda(), lse_acc.cuda()
    res_o, res_l = fa.lse_merge(o_part.cuda(), lse_part.cuda(), acc_d, lacc_d, layout=layout,
                                accumulate=accumulate, final=final)
    torch.cuda.synchronize()
    parts = [_head_major(o_part, layout)]
    lses = [lse_part.double().numpy()]
    if accumulate:
        parts.insert(0, _head_major(o_acc, layout))
        lses.insert(0, lse_acc.double().numpy())
    o_ref, l_ref = merge_partials(parts, lses)
    got_o = _head_major(res_o, layout)
    got_l = res_l.double().cpu().numpy()
    if final:
        assert res_o.dtype == dtype
        bound = ULP[dtype] * np.abs(o_ref) + 1e-6
    else:
        assert res_o.dtype == torch.float32 and res_o.data_ptr() == acc_d.data_ptr()
        bound = 1e-5 * np.abs(o_ref) + 1e-6
    assert np.all(np.abs(got_o - o_ref) <= bound), float(np.max(np.abs(got_o - o_ref) - bound))
    fin = np.isfinite(l_ref)
    assert np.array_equal(fin, np.isfinite(got_l)) and np.all(got_l[~fin] == -np.inf)
    assert np.max(np.abs(got_l[fin] - l_ref[fin]) / np.maximum(1.0, np.abs(l_ref[fin]))) <= 1e-5
    if not accumulate:                       # only the partial's own empty rows are empty
        assert np.all(got_o[~fin] == 0)


def _qkv(layout, dtype, B, H, S, D, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    shape = (B, S, H, D) if layout == "BSND" else (B, H, S, D)
    return [(torch.randn(shape, generator=g) * (std if i < 2 else 1.0)).to(dtype) for i in range(3)]


STEP_CASES = [
    # layout, dtype, B, H, Sc (rows per chunk), D
    ("BHSD", torch.bfloat16, 1, 2, 200, 128),
    ("BSND", torch.float16, 2, 2, 129, 64),
    ("BSND", torch.bfloat16, 1, 3, 256, 128),
    ("BHSD", torch.float16, 1, 1, 40, 128),
]

# three steps over two local query chunks (segments: query chunk, key chunks [lo, hi), diagonal last
# chunk, first, last): diagonal blocks with causal offsets 0 and Sc; a full two-chunk segment merged
# into a running result; a segment from the second key chunk with its diagonal; the final merges
STEPS = [
    [(0, 0, 1, True, True, False), (1, 0, 2, True, True, False)],
    [(1, 0, 2, False, False, False), (0, 1, 2, True, False, True)],
    [(1, 0, 1, False, False, True)],
]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: f"{c[0]}_{str(c[1])[6:]}_B{c[2]}H{c[3]}_Sc{c[4]}_D{c[5]}")
def test_ring_step_matches_oracle_blocks_and_merges(case):
    _need_gpu()
    layout, dtype, B, H, Sc, D = case
    scale = 1.0 / math.sqrt(D)
    g = torch.Generator().manual_seed(Sc * 7 + D)
    shape = (B, 2 * Sc, H, D) if layout == "BSND" else (B, H, 2 * Sc, D)
    q = torch.randn(shape, generator=g).to(dtype)
    kvs = [[torch.randn(shape, generator=g).to(dtype) for _ in range(2)] for _ in STEPS]
    ref = ring.BlockwiseStep(OracleOps(layout, scale))
    r_out, r_lse, r_acc = (torch.zeros(shape, dtype=torch.float64), torch.zeros((B, H, 2 * Sc), dtype=torch.float64),
                           torch.zeros(shape, dtype=torch.float64))
    ops = ring.CudaStepOps(layout, scale)
    qd = q.cuda()
    out = torch.full(shape, float("nan"), dtype=dtype, device="cuda")
    lse = torch.full((B, H, 2 * Sc), float("nan"), device="cuda")
    acc = torch.full(shape, float("nan"), device="cuda")
    seq = 1 if layout == "BSND" else 2
    for n, (segs, (k, v)) in enumerate(zip(STEPS, kvs)):
        ops.step(qd, k.cuda(), v.cuda(), segs, Sc, out, lse, acc)
        ref.step(q.double(), k.double(), v.double(), segs, Sc, r_out, r_lse, r_acc)
        fa.check_device_status()
        if n == 0:
            # after the first step both chunks hold running results: fp32 O in acc, LSE in lse
            err_o = float((acc.double().cpu() - r_acc).abs().max())
            err_l = float((lse.double().cpu() - r_lse).abs().max())
            assert err_o <= O_TOL[dtype] and err_l <= LSE_TOL, (err_o, err_l)
            assert torch.isnan(out).all()          # nothing final yet
    err_o = float((out.double().cpu() - r_out).abs().max())
    err_l = float((lse.double().cpu() - r_lse).abs().max())
    print(f"PARITY ring step {layout} {dtype} B{B} H{H} Sc{Sc} D{D}: max|dO| {err_o:.3e} max|dLSE| {err_l:.3e}")
    assert err_o <= O_TOL[dtype] and err_l <= LSE_TOL
    assert ops.launches == len(STEPS)


def test_ring_step_rejects_bad_segments():
    _need_gpu()
    shape = (1, 256, 2, 128)
    q, k, v, out = (torch.zeros(shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    lse = torch.zeros((1, 2, 256), device="cuda")
    acc = torch.zeros(shape, device="cuda")
    bad = [
        [(0, 0, 128, -1, 1, 1), (64, 0, 128, -1, 1, 1)],     # overlapping rows
        [(200, 0, 128, -1, 1, 1)],                           # rows past the tensor
        [(0, 200, 100, -1, 1, 1)],                           # keys past the tensor
        [(0, 0, 0, -1, 1, 1)],                               # no keys
        [(0, 0, 128, -1, 2, 1)],                             # a flag other than 0 / 1
        [],                                                  # no segment
        [(0, 0, 128, -1, 1, 1)] * 3,                         # three segments
    ]
    for segs in bad:
        with pytest.raises(fa.FaError, match="INVALID_ARG"):
            fa.ring_step(q, k, v, segs, 128, out, lse, acc=acc, layout="BSND")
    with pytest.raises(fa.FaError, match="INVALID_ARG"):     # a running result is needed but missing
        fa.ring_step(q, k, v, [(0, 0, 128, -1, 0, 1)], 128, out, lse, acc=None, layout="BSND")
    big = torch.zeros(shape, device="cuda")                  # an fp32 acc whose first half is q
    q_in_acc = big.view(torch.bfloat16).view(-1)[:q.numel()].view(shape)
    with pytest.raises(fa.FaError, match="ALIAS"):
        fa.ring_step(q_in_acc, k, v, [(0, 0, 128, -1, 1, 0)], 128, out, lse, acc=big, layout="BSND")
    fa.check_device_status()


RING_CASES = [
    # world, layout, dtype, B, H, S, D, causal
    (1, "BHSD", torch.bfloat16, 1, 2, 512, 128, True),
    (2, "BSND", torch.bfloat16, 1, 2, 800, 128, True),      # chunks of 200 rows
    (2, "BHSD", torch.float16, 2, 2, 1000, 64, False),      # chunks of 250 rows
    (4, "BHSD", torch.bfloat16, 1, 3, 1032, 128, True),     # chunks of 129 rows
    (4, "BSND", torch.float16, 1, 2, 2048, 128, True),
    (3, "BSND", torch.bfloat16, 1, 2, 1536, 128, False),
    (8, "BSND", torch.float16, 1, 2, 2048, 64, False),      # 16 chunks of 128 rows
    (8, "BHSD", torch.bfloat16, 2, 2, 1040, 128, True),     # 16 chunks of 65 rows
]


@pytest.mark.parametrize("case", RING_CASES, ids=lambda c: f"w{c[0]}_{c[1]}_{str(c[2])[6:]}_S{c[5]}_D{c[6]}_"
                                                         f"{'c' if c[7] else 'n'}")
def test_emulated_ring_matches_oracle(orc, case):
    _need_gpu()
    world, layout, dtype, B, H, S, D, causal = case
    q, k, v = _qkv(layout, dtype, B, H, S, D, seed=S + world)
    o, lse = ring.ring_attention_emulated(q.cuda(), k.cuda(), v.cuda(), world, causal=causal, layout=layout)
    fa.check_device_status()
    o_ref, l_ref = orc.fwd(q, k, v, layout=layout, causal=causal, scale=1.0 / math.sqrt(D))
    err_o = float(np.max(np.abs(_head_major(o, layout) - o_ref)))
    err_l = float(np.max(np.abs(lse.double().cpu().numpy() - l_ref)))
    print(f"PARITY ring w{world} {layout} {dtype} S{S} D{D} causal={causal}: max|dO| {err_o:.3e} "
          f"max|dLSE| {err_l:.3e}")
    assert err_o <= O_TOL[dtype] and err_l <= LSE_TOL


@pytest.mark.parametrize("world,layout", [(2, "BSND"), (3, "BHSD")])
def test_emulated_ring_with_reversed_pairs_matches_oracle(orc, world, layout):
    # held chunks in descending order: segments that start at the second held chunk, and steps that need
    # two fa_fwd_ring_step launches (two segments of one query chunk)
    _need_gpu()
    ids = lambda r, w: (2 * w - 1 - r, r)
    dtype, S, D = torch.bfloat16, 2 * world * 150, 128
    q, k, v = _qkv(layout, dtype, 1, 2, S, D, seed=S + 7)
    o, lse = ring.ring_attention_emulated(q.cuda(), k.cuda(), v.cuda(), world, causal=True, layout=layout,
                                          chunk_ids_of=ids)
    fa.check_device_status()
    o_ref, l_ref = orc.fwd(q, k, v, layout=layout, causal=True, scale=1.0 / math.sqrt(D))
    err_o = float(np.max(np.abs(_head_major(o, layout) - o_ref)))
    err_l = float(np.max(np.abs(lse.double().cpu().numpy() - l_ref)))
    print(f"PARITY ring reversed w{world} {layout}: max|dO| {err_o:.3e} max|dLSE| {err_l:.3e}")
    assert err_o <= O_TOL[dtype] and err_l <= LSE_TOL


def test_ring_forward_without_process_group_is_plain_attention(orc):
    _need_gpu()
    import torch.distributed as dist
    assert not (dist.is_available() and dist.is_initialized())
    q, k, v = _qkv("BSND", torch.bfloat16, 1, 2, 600, 128, seed=9)
    qs, ks, vs = (ring.shard(t, 0, 1, "BSND").cuda() for t in (q, k, v))
    o, lse = ring.ring_attention_forward(qs, ks, vs, causal=True, layout="BSND")
    # world 1, causal: chunk 0 sees itself (diagonal) and chunk 1 sees chunks 0 and 1; compare with the oracle
    o_ref, l_ref = orc.fwd(q, k, v, layout="BSND", causal=True, scale=1.0 / math.sqrt(128))
    got = ring.unshard([o.cpu()], "BSND")
    got_l = ring.unshard([lse.cpu()], "BSND", seq_dim=2)
    assert float(np.max(np.abs(_head_major(got, "BSND") - o_ref))) <= 2e-2
    assert float(np.max(np.abs(got_l.double().numpy() - l_ref))) <= LSE_TOL


def test_long_sequence_over_eight_ranks_sampled_rows(orc):
    # the 64K-row, 8-head causal bf16 workload (BHSD, D = 128), as 8 ranks of 8K rows
    _need_gpu()
    B, H, S, D, world = 1, 8, 65536, 128, 8
    q, k, v = _qkv("BHSD", torch.bfloat16, B, H, S, D, seed=45)
    o, lse = ring.ring_attention_emulated(q.cuda(), k.cuda(), v.cuda(), world, causal=True, layout="BHSD")
    fa.check_device_status()
    rng = np.random.default_rng(3)
    rows_s = np.unique(np.concatenate([[0, 1, 4095, 4096, 8191, 8192, S - 1],
                                       rng.integers(0, S, 40)]))
    heads = np.arange(H)
    flat = (heads[:, None] * S + rows_s[None, :]).reshape(-1)
    o_ref, l_ref = orc.fwd(q, k, v, layout="BHSD", causal=True, scale=1.0 / math.sqrt(D), rows=flat)
    got = o[0].reshape(H * S, D)[torch.as_tensor(flat, device=o.device)].double().cpu().numpy()
    got_l = lse[0].reshape(H * S)[torch.as_tensor(flat, device=o.device)].double().cpu().numpy()
    err_o, err_l = float(np.max(np.abs(got - o_ref))), float(np.max(np.abs(got_l - l_ref)))
    print(f"PARITY ring w8 BHSD bf16 S65536 H8 causal (sampled {flat.size} rows): max|dO| {err_o:.3e} "
          f"max|dLSE| {err_l:.3e}")
    assert err_o <= 2e-2 and err_l <= LSE_TOL
