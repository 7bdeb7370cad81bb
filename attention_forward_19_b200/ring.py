"""Context-parallel (ring) attention forward: one long sequence over several GPUs.

Page "FlashAttention in ops-transformer on Ascend NPU" (ai6s.net/6a0d3bfb),
section "what else is in the ops-transformer repository", lists ring attention
as the operator for very long sequences; page "64K long-sequence
FlashAttention" (ai6s.net/6a140d07), section "performance tuning tips"
(multi-card parallelism), splits a 64K sequence as 8K per card.  This module
is that split for self-attention (Sq = Sk = S):

* The sequence is cut into 2W chunks of S / 2W rows (W ranks).  Rank r holds
  query, key and value chunks r and 2W - 1 - r ("zigzag"), so that with the
  causal mask every rank has the same amount of visible work.
* W steps: at step t rank r holds the key/value chunks of rank (r - t) mod W,
  sends them on to rank r + 1 and receives the next ones from rank r - 1
  (NCCL point-to-point on its own stream, into this GPU's memory, while the
  current chunks are being used).  No load reads another GPU's memory.
* For every (query chunk, key chunk) pair the key chunk is either entirely
  visible (an earlier chunk, or no mask), the diagonal block (the same chunk:
  the causal mask within it is exactly the top-left mask of fa_fwd), or
  entirely masked (a later chunk: skipped).  Each visible block is one fa_fwd
  call; its normalised partial (O, LSE) is merged into a running fp32 result
  by fa_lse_merge, and the last merge writes the output in the input dtype.

Local tensors are chunk-major so that every chunk is contiguous: q, k, v of a
rank are [n, B, Sc, H, D] (layout "BSND") or [n, B, H, Sc, D] ("BHSD") with n
chunks of Sc rows, and the LSE is [n, B, H, Sc].  shard() and unshard() convert
from and to whole-sequence tensors.

The per-block compute and merge are plain callables, so the schedule and the
exchange can be run on the CPU with other implementations of those two steps.
"""
import math

import torch


# ----------------------------------------------------------------------------- schedule (host logic)


def zigzag_chunk_ids(rank, world):
    """Global chunk indices (of 2 * world) that rank holds: r and 2W - 1 - r."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    return (rank, 2 * world - 1 - rank)


def chunk_visibility(q_chunk, k_chunk, causal):
    """How key chunk k_chunk is seen by query chunk q_chunk (equal chunk sizes, one sequence).

    Returns None when no key is visible (causal, a later chunk), False when every key is visible,
    True for the diagonal block, where the causal mask within the block applies."""
    if not causal:
        return False
    if k_chunk > q_chunk:
        return None
    return k_chunk == q_chunk


def ring_source(rank, world, step):
    """The rank whose key/value chunks rank holds at `step`."""
    return (rank - step) % world


def contribution_plan(rank, world, causal, chunk_ids_of=zigzag_chunk_ids):
    """For each local query chunk, the blocks that contribute to it, in the order they are computed.

    Returns plan[i] = [(step, j, diagonal, first, last), ...]: at `step`, key/value chunk j of the
    chunks then held; `first` and `last` mark the first and the last contributing block."""
    mine = chunk_ids_of(rank, world)
    plan = []
    for a in mine:
        blocks = []
        for t in range(world):
            theirs = chunk_ids_of(ring_source(rank, world, t), world)
            for j, c in enumerate(theirs):
                vis = chunk_visibility(a, c, causal)
                if vis is not None:
                    blocks.append((t, j, vis))
        if not blocks:
            raise ValueError(f"query chunk {a} sees no key chunk")
        plan.append([(t, j, d, n == 0, n == len(blocks) - 1) for n, (t, j, d) in enumerate(blocks)])
    return plan


def _seq_dim(layout):
    if layout == "BSND":
        return 1
    if layout == "BHSD":
        return 2
    raise ValueError(f"layout must be 'BSND' or 'BHSD', not {layout!r}")


def shard(x, rank, world, layout, chunk_ids_of=zigzag_chunk_ids):
    """This rank's chunks of a whole-sequence tensor [B, S, H, D] / [B, H, S, D], chunk-major."""
    dim = _seq_dim(layout)
    S = x.shape[dim]
    if S % (2 * world):
        raise ValueError(f"sequence length {S} is not a multiple of 2 * world = {2 * world}")
    chunks = x.chunk(2 * world, dim=dim)
    return torch.stack([chunks[c] for c in chunk_ids_of(rank, world)]).contiguous()


def unshard(parts, layout, chunk_ids_of=zigzag_chunk_ids, seq_dim=None):
    """Whole-sequence tensor from every rank's chunk-major part (parts[r] of rank r).

    seq_dim: the sequence axis of one chunk (default from the layout; 2 for the LSE [B, H, Sc])."""
    world = len(parts)
    dim = _seq_dim(layout) if seq_dim is None else seq_dim
    by_id = {}
    for r, p in enumerate(parts):
        for i, c in enumerate(chunk_ids_of(r, world)):
            by_id[c] = p[i]
    return torch.cat([by_id[c] for c in range(2 * world)], dim=dim)


# ----------------------------------------------------------------------------- the two compute steps


class CudaBlockOps:
    """The block attention (fa_fwd) and the merge (fa_lse_merge) through the C ABI."""

    acc_dtype = torch.float32      # the running result
    lse_dtype = torch.float32      # what fa_fwd and fa_lse_merge write

    def __init__(self, layout, scale):
        from . import flash_attention_forward, lse_merge, fa_fwd_workspace_size
        self.layout, self.scale = layout, scale
        self._fwd, self._merge = flash_attention_forward, lse_merge
        self._ws_bytes = fa_fwd_workspace_size()
        self._ws = None

    def block(self, q, k, v, diagonal, o, lse):
        if self._ws is None or self._ws.device != q.device:
            self._ws = torch.empty(self._ws_bytes, dtype=torch.uint8, device=q.device)
        self._fwd(q, k, v, layout=self.layout, causal=bool(diagonal), scale=self.scale, out=o, lse=lse,
                  workspace=self._ws)

    def merge(self, o_part, lse_part, o_acc, lse_acc, o_out, lse_out, accumulate, final):
        self._merge(o_part, lse_part, o_acc, lse_acc, out=o_out, lse_out=lse_out, layout=self.layout,
                    accumulate=accumulate, final=final)


# ----------------------------------------------------------------------------- exchanges


class P2PExchange:
    """Passes key/value chunks one rank on with torch.distributed point-to-point operations.

    post() starts sending the current chunks to rank + 1 and receiving the next ones from
    rank - 1 into a second pair of buffers; wait() completes both (on NCCL the current stream
    waits for the transfer; the host does not block).  Two buffer pairs alternate, so a
    buffer is received into only after its earlier send and use are complete."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        g = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
        self.next = g((self.rank + 1) % self.world)
        self.prev = g((self.rank - 1) % self.world)
        self._bufs = None

    def post(self, step, k, v):
        if step == self.world - 1:
            return None
        if self._bufs is None:
            self._bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
        rk, rv = self._bufs[step % 2]
        d = self.dist
        ops = [d.P2POp(d.isend, k, self.next, self.group), d.P2POp(d.isend, v, self.next, self.group),
               d.P2POp(d.irecv, rk, self.prev, self.group), d.P2POp(d.irecv, rv, self.prev, self.group)]
        return d.batch_isend_irecv(ops), rk, rv

    def wait(self, handle):
        reqs, rk, rv = handle
        for r in reqs:
            r.wait()
        return rk, rv


class LocalExchange:
    """Stands in for the ring on one device: every virtual rank's chunks are at hand, so the
    chunks held at each step are looked up instead of received (the same schedule, no transfer)."""

    def __init__(self, rank, world, ks, vs):
        self.rank, self.world, self.ks, self.vs = rank, world, ks, vs

    def post(self, step, k, v):
        if step == self.world - 1:
            return None
        return ring_source(self.rank, self.world, step + 1)

    def wait(self, src):
        return self.ks[src], self.vs[src]


# ----------------------------------------------------------------------------- driver


def ring_steps(q, k, v, rank, world, exchange, ops, causal, chunk_ids_of=zigzag_chunk_ids):
    """Runs one rank's part of ring attention; returns (o like q, lse [n, B, H, Sc]).

    q, k, v: this rank's chunk-major tensors.  exchange: post(step, k, v) / wait(handle) giving
    the next step's chunks.  ops: block(q, k, v, diagonal, o, lse) and merge(...), acc_dtype."""
    if q.shape != k.shape or k.shape != v.shape:
        raise ValueError("ring attention here is self-attention: q, k and v chunks must have one shape")
    n = q.shape[0]
    if n != len(chunk_ids_of(rank, world)):
        raise ValueError(f"expected {len(chunk_ids_of(rank, world))} chunks, got {n}")
    layout = ops.layout
    if layout == "BSND":
        B, Sc, H, _ = q.shape[1:]
    else:
        B, H, Sc, _ = q.shape[1:]
    plan = contribution_plan(rank, world, causal, chunk_ids_of)
    out = torch.empty_like(q)
    lse = torch.empty((n, B, H, Sc), dtype=ops.lse_dtype, device=q.device)
    needs_merge = any(len(p) > 1 for p in plan)
    if needs_merge:
        acc = torch.empty(q.shape, dtype=ops.acc_dtype, device=q.device)
        acc_lse = torch.empty((n, B, H, Sc), dtype=ops.acc_dtype, device=q.device)
        part = torch.empty_like(q[0])
        part_lse = torch.empty((B, H, Sc), dtype=ops.lse_dtype, device=q.device)
    by_step = [[[] for _ in range(n)] for _ in range(world)]
    for i, blocks in enumerate(plan):
        for (t, j, diag, first, last) in blocks:
            by_step[t][i].append((j, diag, first, last))
    cur_k, cur_v = k, v
    for t in range(world):
        handle = exchange.post(t, cur_k, cur_v)
        for i in range(n):
            for (j, diag, first, last) in by_step[t][i]:
                if first and last:       # a single block: its result is the output
                    ops.block(q[i], cur_k[j], cur_v[j], diag, out[i], lse[i])
                    continue
                ops.block(q[i], cur_k[j], cur_v[j], diag, part, part_lse)
                ops.merge(part, part_lse, acc[i], acc_lse[i], out[i], lse[i], accumulate=not first, final=last)
        if handle is not None:
            cur_k, cur_v = exchange.wait(handle)
    return out, lse


def ring_attention_forward(q, k, v, causal=False, scale=None, layout="BSND", group=None,
                           chunk_ids_of=zigzag_chunk_ids):
    """Ring attention over the ranks of `group` (torch.distributed, one GPU per rank).

    q, k, v: this rank's chunk-major CUDA tensors (see shard()).  Returns (o, lse) for this
    rank's query chunks: o like q, lse fp32 [n, B, H, Sc].  scale=None uses 1/sqrt(D)."""
    import torch.distributed as dist
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if dist.is_available() and dist.is_initialized():
        exchange = P2PExchange(group)
        rank, world = exchange.rank, exchange.world
    else:
        rank, world = 0, 1
        exchange = LocalExchange(0, 1, [k], [v])
    return ring_steps(q, k, v, rank, world, exchange, CudaBlockOps(layout, scale), causal, chunk_ids_of)


def ring_attention_emulated(q, k, v, world, causal=False, scale=None, layout="BSND",
                            chunk_ids_of=zigzag_chunk_ids, ops=None):
    """The ring schedule of `world` ranks run one rank after another on one device.

    q, k, v: whole-sequence tensors [B, S, H, D] / [B, H, S, D].  Returns whole-sequence (o, lse)
    assembled from the virtual ranks' results: the same blocks and merges as the real ring, with
    the transfers replaced by lookups (LocalExchange)."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    ops = CudaBlockOps(layout, scale) if ops is None else ops
    qs = [shard(q, r, world, layout, chunk_ids_of) for r in range(world)]
    ks = [shard(k, r, world, layout, chunk_ids_of) for r in range(world)]
    vs = [shard(v, r, world, layout, chunk_ids_of) for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        o, l = ring_steps(qs[r], ks[r], vs[r], r, world, LocalExchange(r, world, ks, vs), ops, causal, chunk_ids_of)
        outs.append(o)
        lses.append(l)
    return unshard(outs, layout, chunk_ids_of), unshard(lses, layout, chunk_ids_of, seq_dim=2)
