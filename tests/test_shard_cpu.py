"""The head partition across GPUs (attention_forward_19_b200.shard), on the CPU.

* head_cost equals a brute-force count of the (query tile, key tile) pairs
  that hold at least one visible (query, key) pair -- the tiles the kernel
  visits -- for ragged and causal shapes.
* partition's largest share equals the brute-force optimum over every
  contiguous split, every item lands in exactly one range, in order, and
  equal costs give ranges that differ by at most one item.
* head_rows covers every element of O and LSE exactly once over the ranges.
* As gloo ranks (world 2 and 3), each rank computes only its heads (with the
  fp64 oracle standing in for the kernel), all_gather_heads assembles the
  result, and every rank ends with the single-rank result, bit for bit.
* The benchmark's shard plan: weak scaling gives rank r exactly batches
  [r B0, (r+1) B0) drawn from its own seed; strong scaling splits one problem.
"""
import datetime
import itertools
import os
import random
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from attention_forward_19_b200 import shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def brute_tile_steps(Sq, Sk, causal):
    steps = 0
    for qt in range(0, Sq, 128):
        for kt in range(0, Sk, 128):
            rows = range(qt, min(qt + 128, Sq))
            if any((not causal) or kt <= i for i in rows):     # key kt (the tile's first) visible to some row
                steps += 1
    return steps


@pytest.mark.parametrize("Sq,Sk", [(1, 1), (7, 7), (128, 128), (129, 129), (300, 1000), (1000, 300), (513, 257),
                                   (4096, 4096), (16000, 16000)])
@pytest.mark.parametrize("causal", [False, True])
def test_head_cost_counts_visited_tiles(Sq, Sk, causal):
    assert shard.head_cost(Sq, Sk, causal) == brute_tile_steps(Sq, Sk, causal)


def test_head_cost_of_the_timed_workload():
    # 64 query tiles of a causal 8192-row head visit 1 + 2 + ... + 64 key tiles
    assert shard.head_cost(8192, 8192, True) == 64 * 65 // 2
    assert shard.head_cost(0, 10, True) == 0


def brute_best(costs, world):
    n = len(costs)
    best = None
    for cuts in itertools.combinations_with_replacement(range(n + 1), world - 1):
        bounds = (0,) + cuts + (n,)
        m = max(sum(costs[bounds[r]:bounds[r + 1]]) for r in range(world))
        best = m if best is None else min(best, m)
    return best


def check_ranges(ranges, n, world):
    assert len(ranges) == world
    pos = 0
    for b, c in ranges:
        assert c >= 0 and b == pos, ranges
        pos += c
    assert pos == n


@pytest.mark.parametrize("seed", range(40))
def test_partition_is_optimal_and_exact_cover(seed):
    rnd = random.Random(seed)
    n = rnd.randint(1, 9)
    world = rnd.randint(1, 4)
    costs = [rnd.choice([0, 1, 2, 5, 9, 30]) for _ in range(n)]
    ranges = shard.partition(costs, world)
    check_ranges(ranges, n, world)
    got = max(sum(costs[b:b + c]) for b, c in ranges)
    assert got == brute_best(costs, world), (costs, world, ranges)


@pytest.mark.parametrize("n,world", [(80, 8), (80, 3), (8, 8), (2, 8), (256, 8), (5, 2), (1, 1)])
def test_equal_costs_give_even_ranges(n, world):
    ranges = shard.partition([7] * n, world)
    check_ranges(ranges, n, world)
    counts = [c for _, c in ranges]
    assert max(counts) - min(counts) <= 1
    assert max(counts) == -(-n // world)


def test_head_ranges_of_the_timed_workload():
    assert shard.head_ranges(2, 40, 8192, 8192, True, 8) == [(10 * r, 10) for r in range(8)]
    assert shard.head_ranges(1, 8, 65536, 65536, True, 8) == [(r, 1) for r in range(8)]
    assert shard.head_ranges(2, 40, 8192, 8192, True, 1) == [(0, 80)]


@pytest.mark.parametrize("layout", ["BSND", "BHSD"])
def test_head_rows_cover_every_element_once(layout):
    B, H, S, D = 3, 5, 4, 2
    o = torch.zeros((B, S, H, D) if layout == "BSND" else (B, H, S, D))
    lse = torch.zeros((B, H, S))
    for begin, count in shard.partition([1] * (B * H), 4):
        for t in (o, lse):
            for view in shard.head_rows(t, begin, count, layout, H):
                view += 1
    assert torch.all(o == 1) and torch.all(lse == 1)
    # a range that starts and ends inside batches
    o.zero_()
    for view in shard.head_rows(o, 3, 4, layout, H):      # heads (0,3), (0,4), (1,0), (1,1)
        view += 1
    ob = o.permute(0, 2, 1, 3) if layout == "BSND" else o
    marked = {(b, h) for b in range(B) for h in range(H) if bool(torch.all(ob[b, h] == 1))}
    assert marked == {(0, 3), (0, 4), (1, 0), (1, 1)}
    assert int((ob != 0).sum()) == 4 * S * D


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_heads(w, q, k, v, begin, count, o, lse):
    """Computes heads [begin, begin + count) with the fp64 oracle into o / lse (in place)."""
    from oracle import attn
    rows = np.arange(begin * w.Sq, (begin + count) * w.Sq, dtype=np.int64)
    o_r, l_r = attn.default().fwd(q, k, v, layout=w.layout, causal=w.causal, scale=float(np.float32(w.scale)),
                                  rows=rows)
    o_r = torch.from_numpy(o_r).reshape(count, w.Sq, w.D)
    l_r = torch.from_numpy(l_r).reshape(count, w.Sq)
    pos = 0
    for ov, lv in zip(shard.head_rows(o, begin, count, w.layout, w.H),
                      shard.head_rows(lse, begin, count, w.layout, w.H)):
        nh = lv.shape[0]
        blk = o_r[pos:pos + nh]
        ov.copy_(blk.permute(1, 0, 2) if w.layout == "BSND" else blk)
        lv.copy_(l_r[pos:pos + nh])
        pos += nh


def _gather_worker(rank, world, port, layout, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from fa_inputs import Workload, make_qkv
        w = Workload("shard", "bf16", layout, 2, 3, 200, 333, 64, True, 0.125, seed=77)   # 6 heads
        q, k, v = make_qkv(w)                   # every rank holds the whole problem
        ranges = shard.head_ranges(w.B, w.H, w.Sq, w.Sk, w.causal, world)
        o = torch.full(q.shape, float("nan"), dtype=torch.float64)
        lse = torch.full((w.B, w.H, w.Sq), float("nan"), dtype=torch.float64)
        b, c = ranges[rank]
        _oracle_heads(w, q, k, v, b, c, o, lse)
        own_only = int(torch.isnan(lse).sum())
        shard.all_gather_heads(o, lse, ranges, w.layout)
        out[rank] = (ranges, own_only, o.numpy().copy(), lse.numpy().copy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("layout", ["BSND", "BHSD"])
def test_gloo_ranks_assemble_the_single_rank_result(world, layout):
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, layout, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(out)
    from fa_inputs import Workload, make_qkv
    from oracle import attn
    w = Workload("shard", "bf16", layout, 2, 3, 200, 333, 64, True, 0.125, seed=77)
    q, k, v = make_qkv(w)
    o_ref, lse_ref = attn.default().fwd(q, k, v, layout=layout, causal=True, scale=float(np.float32(w.scale)))
    for r in range(world):
        ranges, own_only, o, lse = res[r]
        check_ranges(ranges, w.B * w.H, world)
        assert own_only == (w.B * w.H - ranges[r][1]) * w.Sq     # before the gather: only its own rows
        ob = np.transpose(o, (0, 2, 1, 3)) if layout == "BSND" else o
        assert np.array_equal(ob, o_ref) and np.array_equal(lse, lse_ref)


@pytest.mark.parametrize("world", [1, 2, 3])
def test_bench_weak_plan_gives_each_rank_its_own_batches(world):
    import bench
    from fa_inputs import Workload, make_qkv
    w0 = Workload("plan", "fp16", "BSND", 2, 3, 130, 130, 64, True, 0.125, seed=5)
    wg, ranges = bench.shard_plan(w0, world, strong=False)
    assert (wg.B, wg.H) == (w0.B * world, w0.H)
    assert ranges == [(r * w0.B * w0.H, w0.B * w0.H) for r in range(world)]
    for rank in range(world):
        q, k, v = bench.rank_inputs(w0, wg, rank, world, False, "cpu")
        own = make_qkv(bench.rank_workload(w0, rank))
        mine = slice(rank * w0.B, (rank + 1) * w0.B)
        for t, o in zip((q, k, v), own):
            assert torch.equal(t[mine], o)
            rest = torch.cat([t[:rank * w0.B], t[(rank + 1) * w0.B:]])
            assert world == 1 or (rest.numel() > 0 and bool(torch.all(rest == 0)))


def test_bench_strong_plan_splits_one_problem():
    import bench
    from fa_inputs import WORKLOADS, make_qkv
    w0 = WORKLOADS[bench.BENCH_WORKLOAD]
    wg, ranges = bench.shard_plan(w0, 8, strong=True)
    assert wg == w0 and ranges == [(10 * r, 10) for r in range(8)]
    small = WORKLOADS["fp16_bsnd_b1_h2_s512_d64"]
    q, _, _ = bench.rank_inputs(small, small, 1, 2, True, "cpu")
    assert torch.equal(q, make_qkv(small)[0])                 # every rank holds the same whole problem
