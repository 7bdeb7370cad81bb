"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on the CPU.

The forward pass shards by independent (batch, head) problems: under weak
scaling each rank owns one workload's worth of heads, drawn from its own seed
(rank_workload), and the only collectives are a barrier and a max of the
timing.  These tests check that logic without a GPU; the partition itself and
the reassembly of O are tested in test_shard_cpu.py.
"""
import argparse
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from fa_inputs import WORKLOADS, make_qkv
        w0 = WORKLOADS["fp16_bsnd_b1_h2_s512_d64"]
        w = bench.rank_workload(w0, rank)
        q, _, _ = make_qkv(w)
        # each rank's inputs differ; gather a fingerprint of them
        fp = torch.tensor([float(q.float().sum()), float(w.seed)], dtype=torch.float64)
        fps = [torch.zeros_like(fp) for _ in range(world)]
        dist.all_gather(fps, fp)
        t_max = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
        args = argparse.Namespace(steps=2, warmup=3, ref_seconds=1.0, workload=bench.BENCH_WORKLOAD, bh=None)
        ref = bench.run_reference(args, rank, world) if rank != 0 else "rank0-skipped"
        dist.barrier()
        out[rank] = (t_max, [f.tolist() for f in fps], ref)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_host_logic():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        t_max, fps, ref = res[r]
        assert t_max == 11.0, "timing must be the max over ranks"
        assert fps[0][1] != fps[1][1] and fps[0][0] != fps[1][0], "ranks must draw different inputs"
    assert res[1][2] is None, "the reference arm runs on rank 0 only"


def test_single_rank_max_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


@pytest.mark.parametrize("rank", [0, 1, 7])
def test_rank_workload_keeps_shape(rank):
    import bench
    from fa_inputs import WORKLOADS
    w0 = WORKLOADS[bench.BENCH_WORKLOAD]
    w = bench.rank_workload(w0, rank)
    assert (w.B, w.H, w.Sq, w.Sk, w.D, w.causal, w.dtype) == (w0.B, w0.H, w0.Sq, w0.Sk, w0.D, w0.causal, w0.dtype)
    assert w.seed == w0.seed + 1000 * rank
