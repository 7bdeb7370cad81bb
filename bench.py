"""Benchmark of the B200 FlashAttention forward (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {native,reference}]

A step is one attention forward over the workload
bf16 BHSD B=2 H=40 Sq=Sk=8192 D=128, causal, scale 1/sqrt(128), q/k/v ~ N(0,1).
The metric is attention-forward TFLOP/s with the causal-halved flop count
4*B*H*Sq*Sk*D/2.  Timing: W untimed warm-up steps, then exactly K steps
between a barrier + torch.cuda.synchronize() on both sides, timed with CUDA
events on the stream the kernel is launched on.  With N > 1 ranks (torchrun)
the heads of one problem are split into contiguous ranges of equal work
(attention_forward_19_b200.shard), and each rank computes its range with
fa_fwd_heads in place; there is no collective on the data path, and the time
is the max over ranks.  By default the problem is the workload repeated once
per rank along the batch axis, so each rank's share is one workload (weak
scaling); --strong splits the workload itself.  --allgather adds an all-gather
of every rank's O/LSE rows to each step.  The inputs (3 x 168 MB per workload)
are larger than the 126 MB L2, so no flush is done between steps.

--impl reference runs the fp64 CPU oracle (the parity reference) on rank 0
on a bounded row sample of the same workload, each step one sample.

--backward times the backward pass (fa_bwd: dq, dk, dv from the forward's o
and lse) on the same workload instead, and prints its own JSON line; its
metric counts 2.5x the forward's flops (five tile products to the forward's
two, the usual convention), kernel time only.  --backward --atomic times
the non-deterministic variant (fa_bwd_atomic: dQ added up across key tiles).

--ring times ring (context-parallel) attention instead: ONE sequence split
over the N ranks (strong scaling; default workload bf16 BHSD B=1 H=8
S=65536 D=128 causal), each rank holding its zigzag pair of chunks and
passing key/value chunks on over NCCL point-to-point.  A step is the whole
ring; the time is the max over ranks and the value the whole sequence's
flops / that time.  Each rank runs one fa_fwd_ring_step launch per ring step
(the step's blocks attended and merged in one kernel).  With N = 1 the ring
has one rank (its two chunks: one launch).  --ring --emulate-ranks W on one
GPU runs the schedule of W virtual ranks one after another (the transfers
replaced by lookups) and reports each virtual rank's share of the flops over
its own time; the value projects W GPUs as the whole sequence's flops over
the slowest virtual rank's time.

--splitkv [N] times the workload (no mask only) through fa_fwd_splitkv, the
keys split into N ranges (default: enough work units for every SM), next to
the one-pass kernel on the same inputs.

--proj times attention followed by its output projection (fa_fwd_proj:
y = o w_o^T with E = H * D output features, w_o seeded N(0, 1/(H D))) on the
same workload; the value counts both parts' flops, and the attention kernel
and the projection kernel are also timed alone (events around each).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from fa_inputs import BENCH_WORKLOAD, WORKLOADS, make_dout, make_qkv  # noqa: E402

METRIC = "attn fwd TFLOP/s (causal-halved) and % of B200 dense fp16/bf16 tensor peak"
UNIT = "TFLOP/s"
SPEC_PEAK_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SRC = os.path.join(ROOT, "attention_forward_19_b200", "csrc", "fa_fwd.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "fa_fwd_bf16_bhsd_b2_h40_s8192_d128_causal.dram.json")


def kernel_hash():
    with open(KERNEL_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def workload_config(w, n_gpus):
    return {
        "workload": w.name, "model": "attention forward (no weights)", "B": w.B, "H": w.H, "Sq": w.Sq,
        "Sk": w.Sk, "D": w.D, "layout": w.layout, "causal": w.causal, "scale": w.scale, "dtype": w.dtype,
        "global_batch": w.B * n_gpus, "seq_len": w.Sq, "parallelism": f"dp{n_gpus} (independent heads per rank)",
        "l2": (f"no flush: inputs 3 x {w.B * w.H * w.Sq * w.D * 2 / 1e6:.0f} MB > 126 MB L2"
               if w.B * w.H * w.Sq * w.D * 2 > 126e6 else "no flush: the inputs fit in L2 (a latency-bound case)"),
        "inputs": "seeded N(0,1), fp32 randn rounded to bf16",
    }


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self._t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle


def oracle_sample(w, target_s, max_rows=None, threads=0):
    """Times the fp64 oracle on stratified rows of w for about target_s seconds.

    Returns (tflops, seconds, rows, threads): flops count 4*D per visible (query, key) pair.
    """
    import numpy as np
    from oracle import attn
    orc = attn.default()
    q, k, v = make_qkv(w)
    nthreads = threads if threads > 0 else orc.max_threads()
    rng = np.random.default_rng(12345)
    total_rows = w.B * w.H * w.Sq
    flops = 0.0
    done = 0
    t0 = time.perf_counter()
    batch = 64
    while True:
        rows = rng.integers(0, total_rows, size=batch, dtype=np.int64)
        i = rows % w.Sq
        vis = np.minimum(i + 1, w.Sk) if w.causal else np.full_like(i, w.Sk)
        orc.fwd(q, k, v, layout=w.layout, causal=w.causal, scale=float(np.float32(w.scale)), rows=rows,
                threads=nthreads)
        flops += float(4.0 * w.D * vis.sum())
        done += batch
        el = time.perf_counter() - t0
        if el >= target_s or (max_rows is not None and done >= max_rows):
            break
        batch = min(batch * 2, 8192)
    return flops / el / 1e12, el, done, nthreads


# ----------------------------------------------------------------------------- native arm


RING_WORKLOAD = "bf16_bhsd_b1_h8_s65536_d128_causal"


def bench_workload(args):
    """The timed workload; --workload / --bh select another one (profiling runs only)."""
    name = args.workload
    if name is None:
        name = RING_WORKLOAD if getattr(args, "ring", False) else BENCH_WORKLOAD
    w = WORKLOADS[name]
    if args.bh:
        b, h = (int(x) for x in args.bh.split(","))
        w = w.with_(B=b, H=h, name=f"{w.name}_b{b}_h{h}")
    if getattr(args, "sqsk", None):
        sq, sk = (int(x) for x in args.sqsk.split(","))
        w = w.with_(Sq=sq, Sk=sk, name=f"{w.name}_q{sq}_k{sk}")
    return w


def rank_workload(w0, rank):
    """Weak scaling: every rank runs the full workload on its own inputs (seed offset by rank)."""
    return w0.with_(seed=w0.seed + 1000 * rank)


def shard_plan(w0, world, strong):
    """The problem the ranks share and each rank's (head_begin, head_count).

    Weak scaling (default): the problem is the workload repeated along the batch
    axis once per rank (B = world * B0), so each rank's balanced share is one
    workload's worth of heads.  Strong scaling: the problem is the workload
    itself, split into balanced head ranges."""
    from attention_forward_19_b200 import shard
    wg = w0 if strong or world == 1 else w0.with_(B=w0.B * world, name=f"{w0.name}_x{world}")
    ranges = shard.head_ranges(wg.B, wg.H, wg.Sq, wg.Sk, wg.causal, world)
    return wg, ranges


def rank_inputs(w0, wg, rank, world, strong, device):
    """q, k, v of the shared problem on this rank, in the whole problem's shape.

    Strong scaling: every rank holds the same whole problem (one seed).  Weak
    scaling: rank r draws its own batches [r B0, (r + 1) B0) -- exactly its head
    range -- from its own seed (rank_workload); the other batches stay zero and
    are never read by this rank."""
    if strong or world == 1:
        return make_qkv(wg, device=device)
    from fa_inputs import DTYPES
    dt = DTYPES[wg.dtype]
    q = torch.zeros(wg.q_shape(), dtype=dt, device=device)
    k = torch.zeros(wg.kv_shape(), dtype=dt, device=device)
    v = torch.zeros(wg.kv_shape(), dtype=dt, device=device)
    mine = slice(rank * w0.B, (rank + 1) * w0.B)
    for dst, src in zip((q, k, v), make_qkv(rank_workload(w0, rank), device=device)):
        dst[mine].copy_(src)
    return q, k, v


def max_over_ranks(ms, world, device):
    """The slowest rank's time (a scalar all-reduce; no data-path collective)."""
    if world == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def run_native(args, rank, world, local_rank):
    import attention_forward_19_b200 as fa
    from attention_forward_19_b200 import shard
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w0 = bench_workload(args)
    wg, ranges = shard_plan(w0, world, args.strong)
    h0, hc = ranges[rank]
    q, k, v = rank_inputs(w0, wg, rank, world, args.strong, dev)
    o = torch.zeros_like(q)
    lse = torch.zeros((wg.B, wg.H, wg.Sq), dtype=torch.float32, device=dev)
    # work counter of the dynamic schedule (fa_fwd_heads with a workspace); zeroed by the library
    # before every launch
    ws = torch.empty(fa.fa_fwd_workspace_size(), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.flash_attention_forward(q, k, v, layout=wg.layout, causal=wg.causal, scale=wg.scale, out=o, lse=lse,
                                   stream=stream, schedule="dynamic", workspace=ws, heads=(h0, hc))
        if args.allgather and world > 1:
            shard.all_gather_heads(o, lse, ranges, wg.layout)

    for _ in range(args.warmup):
        step()
    fa.check_device_status(stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(cvd.split(",")[local_rank].strip() if cvd else str(local_rank))
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    ms_local = e0.elapsed_time(e1)
    fa.check_device_status(stream)
    ms_total = max_over_ranks(ms_local, world, dev)
    ms_step = ms_total / args.steps
    flops_rank = shard.flops_of_heads(hc, wg.Sq, wg.Sk, wg.D, wg.causal)
    flops = shard.flops_of_heads(wg.B * wg.H, wg.Sq, wg.Sk, wg.D, wg.causal)   # all ranks together
    value = flops * args.steps / (ms_total * 1e-3) / 1e12

    if args.no_e2e:
        if rank == 0:
            print(f"{wg.name}: {ms_step:.4f} ms/step, {value:.1f} TFLOP/s (no e2e, no baseline)", flush=True)
        return None
    # End to end through the public API: this rank's input rows from pinned host memory -> device ->
    # kernel -> this rank's result rows (with --allgather, the whole result) back to pinned host memory.
    # The rank's heads are split into chunks that pipeline over three streams: the host-to-device copy
    # of chunk g + 1 and the device-to-host copy of chunk g - 1 run while the kernel computes chunk g
    # (fa_fwd_heads on the chunk's heads).
    e2e_steps = max(3, min(args.steps, 10))
    nchunk = max(1, min(args.e2e_chunks, hc)) if not (args.allgather and world > 1) else 1
    bounds = [h0 + (hc * c) // nchunk for c in range(nchunk + 1)]
    chunks = [(bounds[c], bounds[c + 1] - bounds[c]) for c in range(nchunk)]
    dev_in = [[view for t in (q, k, v) for view in shard.head_rows(t, b0, n0, wg.layout, wg.H)] for b0, n0 in chunks]
    host_in = [[view.cpu().pin_memory() for view in views] for views in dev_in]
    if args.allgather and world > 1:
        dev_out = [[o, lse]]
    else:
        dev_out = [[view for t in (o, lse) for view in shard.head_rows(t, b0, n0, wg.layout, wg.H)]
                   for b0, n0 in chunks]
    host_out = [[torch.empty(view.shape, dtype=view.dtype, pin_memory=True) for view in views] for views in dev_out]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_step():
        start = torch.cuda.Event()
        start.record(stream)
        s_in.wait_event(start)
        ready = []
        for c in range(nchunk):
            with torch.cuda.stream(s_in):
                for dst, src in zip(dev_in[c], host_in[c]):
                    dst.copy_(src, non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_in)
                ready.append(e)
        done = []
        for c, (b0, n0) in enumerate(chunks):
            stream.wait_event(ready[c])
            fa.flash_attention_forward(q, k, v, layout=wg.layout, causal=wg.causal, scale=wg.scale, out=o,
                                       lse=lse, stream=stream, schedule="dynamic", workspace=ws, heads=(b0, n0))
            e = torch.cuda.Event()
            e.record(stream)
            done.append(e)
        if args.allgather and world > 1:
            shard.all_gather_heads(o, lse, ranges, wg.layout)
            e = torch.cuda.Event()
            e.record(stream)
            done = [e]
        for c in range(len(dev_out)):
            s_out.wait_event(done[c])
            with torch.cuda.stream(s_out):
                for dst, src in zip(host_out[c], dev_out[c]):
                    dst.copy_(src, non_blocking=True)
        fin = torch.cuda.Event()
        fin.record(s_out)
        stream.wait_event(fin)

    e2e_step()
    barrier()
    torch.cuda.synchronize(dev)
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    a1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), world, dev)
    fa.check_device_status(stream)
    e2e_value = flops * e2e_steps / (e2e_ms * 1e-3) / 1e12
    h2d = sum(t.numel() * t.element_size() for views in host_in for t in views)
    d2h = sum(t.numel() * t.element_size() for views in host_out for t in views)

    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops_rank / (ms_step * 1e-3) / 1e12
    traffic = None
    traffic_note = "no ncu capture of this kernel version"
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f)
        if tr.get("workload") != w0.name:
            traffic_note = f"the ncu traffic capture is of {tr.get('workload')}, not this workload"
        elif tr.get("kernel_sha256_16") == kernel_hash():
            traffic = tr.get("dram_bytes_per_launch")
            traffic_note = tr.get("note", "")
        else:
            traffic_note = "ncu capture is of an older kernel version"
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        tf, secs, nrows, thr = oracle_sample(w0, target_s=args.cpu_seconds)
        cpu = {"value": tf, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": f"{nrows} random query rows of the same workload (fp64, all their visible keys), "
                         f"{secs:.1f} s"}
    cfg = workload_config(w0, world)
    cfg.update({
        "global_batch": wg.B,
        "parallelism": (f"heads{world}: contiguous balanced ranges of the B*H = {wg.B * wg.H} heads "
                        f"(fa_fwd_heads in place), {'O/LSE all-gathered' if args.allgather and world > 1 else 'no collective on the data path'}"),
        "head_ranges": [list(r) for r in ranges],
    })
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if args.strong else "weak",
        "vs_baseline": None, "dtype": wg.dtype, "data": "synthetic",
        "config": cfg,
        "pct_of_spec_peak": 100.0 * value / world / SPEC_PEAK_TFLOPS,
        "pct_of_measured_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
                                    if peak_kind == "measured" else "fallback 1590 TFLOP/s",
                     "frac_of_sustained": achieved / float(peaks["bf16_tflops_sustained"]),
                     "frac_of_spec_2250": achieved / SPEC_PEAK_TFLOPS,
                     "algorithmic_flops_per_launch": flops_rank, "traffic_note": traffic_note},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                "pipeline": f"{nchunk} head chunks over three streams (copy in, fa_fwd_heads, copy out)"},
        "gpu_launches": args.steps,
        "clocks": clk,
        "kernel": "fa::fa_fwd_kernel<128, true> via fa_fwd_heads (dynamic schedule; libfa_fwd.so)",
        "gpu_launches_note": "one fa_fwd_kernel launch per step (plus the library's 4-byte cudaMemsetAsync of the work counter)",
    }
    return line


def run_backward(args, rank, world, local_rank):
    """Times the backward pass on the workload (kernel time; one JSON line)."""
    import attention_forward_19_b200 as fa
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w0 = bench_workload(args)
    w = rank_workload(w0, rank)
    q, k, v = make_qkv(w, device=dev)
    do = make_dout(w, device=dev)
    stream = torch.cuda.current_stream(dev)
    o, lse = fa.flash_attention_forward(q, k, v, layout=w.layout, causal=w.causal, scale=w.scale, stream=stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    det = not args.atomic
    nbytes = fa.fa_bwd_workspace_size(w.B, w.H, w.Sq) if det else fa.fa_bwd_atomic_workspace_size(w.B, w.H, w.Sq, w.D)
    ws = torch.empty(max(16, nbytes), dtype=torch.uint8, device=dev)

    def step():
        fa.flash_attention_backward(q, k, v, o, lse, do, layout=w.layout, causal=w.causal, scale=w.scale, dq=dq,
                                    dk=dk, dv=dv, stream=stream, workspace=ws, deterministic=det)

    for _ in range(args.warmup):
        step()
    fa.check_device_status(stream)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(cvd.split(",")[local_rank].strip() if cvd else str(local_rank))
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    fa.check_device_status(stream)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_step = ms_total / args.steps
    flops = 2.5 * w.flops()
    value = world * flops * args.steps / (ms_total * 1e-3) / 1e12
    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (ms_step * 1e-3) / 1e12
    return {
        "metric": "attn bwd TFLOP/s (2.5x the causal-halved forward flops)"
                  + ("" if det else ", non-deterministic variant"), "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w0, world),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                     "traffic": None,
                     "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
                                    if peak_kind == "measured" else "fallback 1590 TFLOP/s",
                     "algorithmic_flops_per_step": flops,
                     "note": "the pass computes S and dP twice (7 tile products), the metric counts 5" if det
                     else "one kernel per key tile (5 tile products) plus bulk fp32 reductions of dQ"},
        "gpu_launches": 3 * args.steps,
        "gpu_launches_note": "per step: prep, dK/dV and dQ kernels" if det
        else "per step: prep, the dK/dV/dQ kernel and the dQ conversion (plus a memset of the accumulator)",
        "clocks": clk,
    }


def run_ring(args, rank, world, local_rank):
    """Times ring attention of one sequence over the ranks (strong scaling; one JSON line)."""
    import attention_forward_19_b200 as fa
    from attention_forward_19_b200 import ring
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = bench_workload(args)
    if args.emulate_ranks:
        if world != 1:
            raise SystemExit("--emulate-ranks runs on one GPU")
        return run_ring_emulated(args, w, dev)
    if w.Sq != w.Sk or w.Sq % (2 * world):
        raise SystemExit(f"--ring needs Sq == Sk and a multiple of {2 * world} rows")
    q, k, v = make_qkv(w)                       # the same whole sequence on every rank, then its shard
    q, k, v = (ring.shard(t, rank, world, w.layout).to(dev) for t in (q, k, v))
    stream = torch.cuda.current_stream(dev)

    def step():
        return ring.ring_attention_forward(q, k, v, causal=w.causal, scale=w.scale, layout=w.layout)

    for _ in range(args.warmup):
        step()
    fa.check_device_status(stream)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(cvd.split(",")[local_rank].strip() if cvd else str(local_rank))
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    fa.check_device_status(stream)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_step = ms_total / args.steps
    flops = w.flops()
    value = flops * args.steps / (ms_total * 1e-3) / 1e12
    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    launches = ring_launches(ring.step_plan(0, world, w.causal))
    cfg = workload_config(w, world)
    cfg.update({"global_batch": w.B, "parallelism": f"cp{world} (ring over NCCL point-to-point, zigzag chunks)"})
    return {
        "metric": "ring attn fwd TFLOP/s (causal-halved, one sequence over all ranks)", "value": value,
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": cfg,
        "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak, "unit": UNIT,
                     "frac": value / world / peak, "traffic": None,
                     "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
                                    if peak_kind == "measured" else "fallback 1590 TFLOP/s",
                     "note": "per-GPU share of the whole sequence's flops over the slowest rank's time"},
        "gpu_launches": launches * args.steps,
        "gpu_launches_note": f"rank 0 per step: {launches} fa_fwd_ring_step launches (one per ring step)",
        "clocks": clk,
    }


def ring_launches(plan):
    """fa_fwd_ring_step launches of a rank's step plan."""
    from attention_forward_19_b200 import ring
    return sum(len(ring.launch_batches(segs)) for segs in plan)


def run_ring_emulated(args, w, dev):
    """--ring --emulate-ranks W on one GPU: each virtual rank's ring (K timed repetitions) in turn."""
    import attention_forward_19_b200 as fa
    from attention_forward_19_b200 import ring
    W = args.emulate_ranks
    if w.Sq != w.Sk or w.Sq % (2 * W):
        raise SystemExit(f"--ring needs Sq == Sk and a multiple of {2 * W} rows")
    q, k, v = make_qkv(w)
    qs, ks, vs = ([ring.shard(t, r, W, w.layout).to(dev) for r in range(W)] for t in (q, k, v))
    del q, k, v
    stream = torch.cuda.current_stream(dev)
    ops = ring.CudaStepOps(w.layout, w.scale)
    per_rank = []
    for r in range(W):
        def step():
            return ring.ring_steps(qs[r], ks[r], vs[r], r, W, ring.LocalExchange(r, W, ks, vs), ops, w.causal)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        plan = ring.contribution_plan(r, W, w.causal)
        rank_flops = sum(w.flops() / (2 * W) ** 2 / (0.5 if w.causal else 1.0) * (0.5 if d else 1.0)
                         for blocks in plan for (_, _, d, _, _) in blocks)
        ms = e0.elapsed_time(e1) / args.steps
        per_rank.append((ms, rank_flops / (ms * 1e-3) / 1e12))
    fa.check_device_status(stream)
    worst = max(ms for ms, _ in per_rank)
    cfg = workload_config(w, 1)
    cfg.update({"global_batch": w.B, "parallelism": f"cp{W} emulated on one GPU (zigzag chunks, no transfers)"})
    return {
        "metric": f"ring attn fwd TFLOP/s, {W} ranks emulated on one GPU (projected: whole sequence over the "
                  f"slowest virtual rank)", "value": w.flops() / (worst * 1e-3) / 1e12, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": worst, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": cfg,
        "per_rank_ms": [round(ms, 4) for ms, _ in per_rank],
        "per_rank_share_tflops": [round(t, 1) for _, t in per_rank],
        "gpu_launches": ring_launches(ring.step_plan(0, W, w.causal)) * args.steps * W,
    }


def run_splitkv(args, rank, world, local_rank):
    """--splitkv [N]: the workload (no mask) through fa_fwd_splitkv, N key ranges (0: the binding's default
    for this size), timed next to the one-pass kernel on the same inputs; one JSON line."""
    import attention_forward_19_b200 as fa
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world != 1:
        raise SystemExit("--splitkv runs on one GPU")
    w = bench_workload(args)
    if w.causal:
        raise SystemExit("--splitkv applies no mask: pick a workload without causal masking")
    q, k, v = make_qkv(w, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    n = args.splitkv if args.splitkv > 0 else fa.default_splits(w.B, w.H, w.Sq, w.Sk, sms)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_fwd_splitkv_workspace_size(w.B, w.H, w.Sq, w.D, n), dtype=torch.uint8, device=dev)
    ws1 = torch.empty(fa.fa_fwd_workspace_size(), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def split():
        fa.flash_attention_forward_splitkv(q, k, v, layout=w.layout, scale=w.scale, nsplit=n, out=o, lse=lse,
                                           workspace=ws, stream=stream)

    def one_pass():
        fa.flash_attention_forward(q, k, v, layout=w.layout, causal=False, scale=w.scale, out=o, lse=lse,
                                   workspace=ws1, stream=stream)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(cvd.split(",")[local_rank].strip() if cvd else str(local_rank))
    clocks.start()
    time.sleep(0.3)
    ms_one = timed(one_pass)
    ms = timed(split)
    clk = clocks.stop()
    fa.check_device_status(stream)
    flops = w.flops()
    value = flops / (ms * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    cfg = workload_config(w, 1)
    cfg.update({"global_batch": w.B, "parallelism": f"split-KV: {n} key ranges, partials merged by a second kernel"})
    return {
        "metric": "attn fwd TFLOP/s, split-KV (fa_fwd_splitkv: the keys split across CTAs)", "value": value,
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": cfg,
        "one_pass_ms_per_step": ms_one, "one_pass_value": flops / (ms_one * 1e-3) / 1e12,
        "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": UNIT, "frac": value / peak,
                     "traffic": None, "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"},
        "gpu_launches": 2 * args.steps,
        "gpu_launches_note": "per step: the ring-step kernel in its split mode and the merge kernel",
        "clocks": clk,
    }


def run_proj(args, rank, world, local_rank):
    """Times attention + output projection (fa_fwd_proj) and each kernel alone (one JSON line)."""
    import attention_forward_19_b200 as fa
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w0 = bench_workload(args)
    w = rank_workload(w0, rank)
    q, k, v = make_qkv(w, device=dev)
    E = w.H * w.D
    g = torch.Generator(device="cpu").manual_seed(w.seed + 600)
    w_o = (torch.randn((E, w.H * w.D), generator=g) / math.sqrt(w.H * w.D)).to(q.dtype).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
    y = torch.empty((w.B, w.Sq, E), dtype=q.dtype, device=dev)
    ws = torch.empty(fa.fa_fwd_workspace_size(), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fused():
        fa.flash_attention_forward_proj(q, k, v, w_o, layout=w.layout, causal=w.causal, scale=w.scale, out=o,
                                        lse=lse, y=y, stream=stream, workspace=ws)

    def attn():
        fa.flash_attention_forward(q, k, v, layout=w.layout, causal=w.causal, scale=w.scale, out=o, lse=lse,
                                   stream=stream, workspace=ws)

    def proj():
        fa.out_projection(o, w_o, layout=w.layout, y=y, stream=stream)

    def timed(fn, steps):
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dev) / steps

    for _ in range(args.warmup):
        fused()
    fa.check_device_status(stream)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(cvd.split(",")[local_rank].strip() if cvd else str(local_rank))
    clocks.start()
    time.sleep(0.3)
    ms_step = timed(fused, args.steps)
    clk = clocks.stop()
    ms_attn = timed(attn, max(3, args.steps // 2))
    ms_proj = timed(proj, max(3, args.steps // 2))
    fa.check_device_status(stream)
    f_attn = w.flops()
    f_proj = 2.0 * w.B * w.Sq * w.H * w.D * E
    value = world * (f_attn + f_proj) / (ms_step * 1e-3) / 1e12
    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    src = (f"{peak_kind} bf16 burst (MEASURED_PEAKS.json bf16_tflops)" if peak_kind == "measured"
           else "fallback 1590 TFLOP/s")
    a_attn = f_attn / (ms_attn * 1e-3) / 1e12
    a_proj = f_proj / (ms_proj * 1e-3) / 1e12
    cfg = workload_config(w0, world)
    cfg.update({"model": "attention forward + output projection (random-init w_o, E = H * D)", "E": E})
    return {
        "metric": "attn fwd + out-proj TFLOP/s (causal-halved attention flops + 2 B S (H D) E)", "value": value,
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": cfg,
        "roofline": {"bound": "tensor", "achieved": a_attn, "peak": peak, "unit": UNIT, "frac": a_attn / peak,
                     "traffic": None, "peak_source": src, "kernel": "fa_fwd_kernel (dominant), timed alone",
                     "ms_per_launch": ms_attn},
        "roofline_proj": {"bound": "tensor", "achieved": a_proj, "peak": peak, "unit": UNIT,
                          "frac": a_proj / peak, "traffic": None, "peak_source": src,
                          "kernel": "proj_kernel (fa_out_proj), timed alone", "ms_per_launch": ms_proj,
                          "algorithmic_flops_per_launch": f_proj},
        "gpu_launches": 2 * args.steps,
        "gpu_launches_note": "per step: one fa_fwd_kernel and one proj_kernel launch",
        "clocks": clk,
    }


# ----------------------------------------------------------------------------- reference arm


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = bench_workload(args)
    per_step = max(0.5, args.ref_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, target_s=per_step)
    vals, secs, rows = [], 0.0, 0
    thr = None
    for _ in range(args.steps):
        tf, s, n, thr = oracle_sample(w, target_s=per_step)
        vals.append(tf)
        secs += s
        rows += n
    value = statistics.mean(vals)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": f"each step: random query rows of the workload for ~{per_step:.1f} s "
                                   f"({rows} rows in total), fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="time the kernel only (profiling runs)")
    ap.add_argument("--workload", choices=list(WORKLOADS), default=None,
                    help=f"default {BENCH_WORKLOAD} ({RING_WORKLOAD} with --ring)")
    ap.add_argument("--bh", default=None, help="override B,H of the workload (profiling runs)")
    ap.add_argument("--sqsk", default=None, help="override Sq,Sk of the workload (profiling and split-KV runs)")
    ap.add_argument("--backward", action="store_true", help="time the backward pass instead (its own JSON line)")
    ap.add_argument("--atomic", action="store_true", help="with --backward: the non-deterministic variant")
    ap.add_argument("--ring", action="store_true", help="time ring attention of one sequence over the ranks")
    ap.add_argument("--proj", action="store_true", help="time attention + output projection (fa_fwd_proj)")
    ap.add_argument("--splitkv", type=int, default=-1, nargs="?", const=0,
                    help="time the workload (no mask) through fa_fwd_splitkv with this many key ranges (0 or no "
                         "value: the default for its size) next to the one-pass kernel")
    ap.add_argument("--emulate-ranks", type=int, default=0,
                    help="with --ring on one GPU: time the schedule of this many virtual ranks")
    ap.add_argument("--strong", action="store_true",
                    help="split the workload itself across the ranks (default: weak scaling, one workload per rank)")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="head chunks of the end-to-end pipeline (1: copy in, compute, copy out in sequence)")
    ap.add_argument("--allgather", action="store_true",
                    help="after the pass, all-gather every rank's O/LSE rows so each rank holds the whole result")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=torch.device("cuda", local_rank))
        try:
            run = (run_ring if args.ring else run_proj if args.proj else run_backward if args.backward
                   else run_splitkv if args.splitkv >= 0 else run_native)
            line = run(args, rank, world, local_rank)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
