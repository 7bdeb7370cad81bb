"""Host logic of ring (context-parallel) attention, on the CPU.

The schedule, the sharding and the exchange of attention_forward_19_b200.ring
run here with the two compute steps supplied by the oracle (attention of one
block, and the merge of partial results), in fp64, so that any wrong block,
mask, source rank or merge order shows as a large error.  The ranks are either
emulated in one process or run as gloo processes exchanging chunks through
torch.distributed.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from attention_forward_19_b200 import ring
from ring_oracle_ops import OracleOps

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _qkv(layout, B=1, H=2, S=48, D=16, seed=5):
    g = torch.Generator().manual_seed(seed)
    shape = (B, S, H, D) if layout == "BSND" else (B, H, S, D)
    return [torch.randn(shape, generator=g, dtype=torch.float64) for _ in range(3)]


def _oracle_whole(q, k, v, layout, causal, scale):
    from oracle import attn as oracle_attn
    o, l = oracle_attn.default().fwd(q, k, v, layout=layout, causal=causal, scale=scale)
    o = torch.from_numpy(o)
    return (o.permute(0, 2, 1, 3) if layout == "BSND" else o), torch.from_numpy(l)


# ----------------------------------------------------------------------------- schedule


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_chunks_partition_the_sequence(world):
    ids = [c for r in range(world) for c in ring.zigzag_chunk_ids(r, world)]
    assert sorted(ids) == list(range(2 * world))


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_every_visible_key_is_used_exactly_once(world, causal):
    # expand the chunk-level plan to element level and compare with the mask itself
    Sc = 3
    S = 2 * world * Sc
    count = np.zeros((S, S), dtype=int)
    for r in range(world):
        plan = ring.contribution_plan(r, world, causal)
        mine = ring.zigzag_chunk_ids(r, world)
        for i, blocks in enumerate(plan):
            assert blocks[0][3] and blocks[-1][4]
            assert sum(b[3] for b in blocks) == 1 and sum(b[4] for b in blocks) == 1
            for (t, j, diag, _, _) in blocks:
                c = ring.zigzag_chunk_ids(ring.ring_source(r, world, t), world)[j]
                a = mine[i]
                for qi in range(Sc):
                    for kj in range(Sc):
                        if diag and kj > qi:
                            continue
                        count[a * Sc + qi, c * Sc + kj] += 1
    mask = np.tril(np.ones((S, S), dtype=int)) if causal else np.ones((S, S), dtype=int)
    assert np.array_equal(count, mask)


def reversed_zigzag(rank, world):
    """The zigzag pair in the other order: a rank's held chunks are then not in ascending order, so a
    step can need a segment that starts at the second held chunk, or two segments for one query chunk."""
    return (2 * world - 1 - rank, rank)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("ids", [ring.zigzag_chunk_ids, reversed_zigzag], ids=["zigzag", "reversed"])
def test_step_segments_cover_every_visible_key_exactly_once(world, causal, ids):
    # the fa_fwd_ring_step segments of every rank and step, expanded to (global row, global key) pairs
    Sc = 3
    S = 2 * world * Sc
    count = np.zeros((S, S), dtype=int)
    for r in range(world):
        mine = ids(r, world)
        for t, segs in enumerate(ring.step_plan(r, world, causal, ids)):
            held = ids(ring.ring_source(r, world, t), world)
            for (row0, key0, keys, off, _, _) in ring.fa_segments(segs, Sc):
                for rr in range(Sc):
                    grow = mine[(row0 + rr) // Sc] * Sc + (row0 + rr) % Sc
                    for c in range(keys):
                        if off >= 0 and c > rr + off:
                            continue
                        count[grow, held[(key0 + c) // Sc] * Sc + (key0 + c) % Sc] += 1
    mask = np.tril(np.ones((S, S), dtype=int)) if causal else np.ones((S, S), dtype=int)
    assert np.array_equal(count, mask)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_step_plan_first_and_last_and_one_launch_per_step(world, causal):
    for r in range(world):
        plan = ring.step_plan(r, world, causal)
        for i in range(2):
            seq = [g for segs in plan for g in segs if g[0] == i]
            assert seq and seq[0][4] and seq[-1][5]
            assert sum(g[4] for g in seq) == 1 and sum(g[5] for g in seq) == 1
        for segs in plan:
            # zigzag: at most one segment per query chunk, so each step is one launch
            assert len({g[0] for g in segs}) == len(segs) <= 2
            assert len(ring.launch_batches(segs)) == (1 if segs else 0)
            # only a segment's last key chunk may be the diagonal block, and keys start at chunk 0
            assert all(g[1] == 0 and g[2] in (1, 2) for g in segs)
    # with causal zigzag chunks every step has work on every rank
    if causal:
        assert all(ring.step_plan(r, world, True)[t] for r in range(world) for t in range(world))


def test_reversed_pairs_need_later_key_chunks_and_two_launches():
    plan = ring.step_plan(0, 2, True, reversed_zigzag)
    # step 0: query chunk 0 (global 3) sees held chunk 0 (global 3, the diagonal) and then chunk 1 (global 0,
    # fully visible): two segments for one query chunk, so two launches; query chunk 1 (global 0) sees
    # only held chunk 1 (key0 = Sc), its diagonal
    assert plan[0] == [(0, 0, 1, True, True, False), (0, 1, 2, False, False, False), (1, 1, 2, True, True, True)]
    assert [len(b) for b in ring.launch_batches(plan[0])] == [2, 1]
    assert ring.fa_segments([plan[0][2]], 5) == [(5, 5, 5, 0, 1, 1)]


def test_launch_batches_split_repeated_query_chunks():
    segs = [(0, 0, 1, False, True, False), (0, 1, 2, False, False, True), (1, 0, 2, True, True, True)]
    assert ring.launch_batches(segs) == [[segs[0], segs[2]], [segs[1]]]


def test_zigzag_balances_causal_work():
    world = 4
    work = []
    for r in range(world):
        plan = ring.contribution_plan(r, world, True)
        work.append(sum(0.5 if d else 1.0 for blocks in plan for (_, _, d, _, _) in blocks))
    assert len(set(work)) == 1


@pytest.mark.parametrize("layout", ["BSND", "BHSD"])
def test_shard_unshard_round_trip(layout):
    x = _qkv(layout, S=24)[0]
    parts = [ring.shard(x, r, 3, layout) for r in range(3)]
    dim = 1 if layout == "BSND" else 2
    assert all(p.is_contiguous() and p.shape[dim] == 8 for p in parts)      # two chunks of 4 rows
    # rank 1 holds chunks 1 and 4, in that order
    assert torch.equal(parts[1], torch.cat([x.narrow(dim, 4, 4), x.narrow(dim, 16, 4)], dim=dim))
    assert torch.equal(ring.unshard(parts, layout), x)
    with pytest.raises(ValueError):
        ring.shard(x, 0, 5, layout)            # 24 rows are not a multiple of 10


# ----------------------------------------------------------------------------- emulated ranks, oracle compute


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("layout", ["BSND", "BHSD"])
@pytest.mark.parametrize("ids", [ring.zigzag_chunk_ids, reversed_zigzag], ids=["zigzag", "reversed"])
def test_emulated_ring_with_oracle_steps_matches_whole_attention(world, causal, layout, ids):
    q, k, v = _qkv(layout, S=2 * world * 6)
    scale = 0.3
    ops = OracleOps(layout, scale)
    o, l = ring.ring_attention_emulated(q, k, v, world, causal=causal, scale=scale, layout=layout,
                                        ops=ring.BlockwiseStep(ops), chunk_ids_of=ids)
    o_ref, l_ref = _oracle_whole(q, k, v, layout, causal, scale)
    assert float((o - o_ref).abs().max()) < 1e-12
    assert float((l - l_ref).abs().max()) < 1e-12
    n_blocks = (2 * world) * (2 * world + 1) // 2 if causal else (2 * world) ** 2
    assert len(ops.calls) == n_blocks
    assert sum(ops.calls) == (2 * world if causal else 0)   # one diagonal block per chunk


# ----------------------------------------------------------------------------- gloo ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, layout, causal, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from attention_forward_19_b200 import ring as ring_mod
        q, k, v = _qkv(layout, S=2 * world * 5)
        mine = [ring_mod.shard(t, rank, world, layout) for t in (q, k, v)]
        ops = ring_mod.BlockwiseStep(OracleOps(layout, 0.25))
        o, l = ring_mod.ring_steps(*mine, rank, world, ring_mod.P2PExchange(), ops, causal)
        out[rank] = (o.numpy(), l.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,layout", [(2, True, "BSND"), (3, True, "BHSD"), (2, False, "BHSD")])
def test_gloo_ring_exchange_matches_whole_attention(world, causal, layout):
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_gloo_worker, args=(r, world, port, layout, causal, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(out)
    o = ring.unshard([torch.from_numpy(res[r][0]) for r in range(world)], layout)
    l = ring.unshard([torch.from_numpy(res[r][1]) for r in range(world)], layout, seq_dim=2)
    q, k, v = _qkv(layout, S=2 * world * 5)
    o_ref, l_ref = _oracle_whole(q, k, v, layout, causal, 0.25)
    assert float((o - o_ref).abs().max()) < 1e-12
    assert float((l - l_ref).abs().max()) < 1e-12


def _gloo_subgroup_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from attention_forward_19_b200 import ring as ring_mod
        members = [0, 2]                       # global ranks 0 and 2 are group ranks 0 and 1
        group = dist.new_group(members)
        if rank in members:
            grank = members.index(rank)
            q, k, v = _qkv("BHSD", S=2 * 2 * 5)
            mine = [ring_mod.shard(t, grank, 2, "BHSD") for t in (q, k, v)]
            ex = ring_mod.P2PExchange(group)
            assert (ex.rank, ex.world) == (grank, 2)
            # the peers are named by their global ranks: the other member, in both directions
            assert ex.next == ex.prev == members[1 - grank]
            o, l = ring_mod.ring_steps(*mine, grank, 2, ex, ring_mod.BlockwiseStep(OracleOps("BHSD", 0.25)), True)
            out[grank] = (o.numpy(), l.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_ring_on_a_subgroup_maps_group_ranks_to_global_ranks():
    world = 3
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_gloo_subgroup_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(out)
    o = ring.unshard([torch.from_numpy(res[r][0]) for r in range(2)], "BHSD")
    l = ring.unshard([torch.from_numpy(res[r][1]) for r in range(2)], "BHSD", seq_dim=2)
    q, k, v = _qkv("BHSD", S=2 * 2 * 5)
    o_ref, l_ref = _oracle_whole(q, k, v, "BHSD", True, 0.25)
    assert float((o - o_ref).abs().max()) < 1e-12
    assert float((l - l_ref).abs().max()) < 1e-12
