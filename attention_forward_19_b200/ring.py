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
  entirely masked (a later chunk: skipped).
* A step's blocks form at most one "segment" per query chunk: the query chunk
  against a run of consecutive held key chunks, of which only the last may be
  the diagonal block (a causal mask offset by the full chunks before it).
  All segments of a step run as ONE launch of fa_fwd_ring_step, which merges
  each segment's result into the running result of its rows in the attention
  epilogue (fp32 O in a buffer, the LSE in the output LSE) and writes the
  output in the input dtype at the rows' last segment.

Local tensors hold a rank's chunks concatenated along the sequence axis, in
the order of chunk_ids_of: q, k, v of a rank are [B, n * Sc, H, D] (layout
"BSND") or [B, H, n * Sc, D] ("BHSD"), and the LSE is [B, H, n * Sc].
shard() and unshard() convert from and to whole-sequence tensors.

The step is a plain callable, so the schedule and the exchange can also run on
the CPU with the step composed of other implementations of block attention and
the merge (BlockwiseStep).
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
    """This rank's rows of a whole-sequence tensor [B, S, H, D] / [B, H, S, D]: its chunks concatenated
    along the sequence axis in chunk_ids_of order."""
    dim = _seq_dim(layout)
    S = x.shape[dim]
    if S % (2 * world):
        raise ValueError(f"sequence length {S} is not a multiple of 2 * world = {2 * world}")
    chunks = x.chunk(2 * world, dim=dim)
    return torch.cat([chunks[c] for c in chunk_ids_of(rank, world)], dim=dim).contiguous()


def unshard(parts, layout, chunk_ids_of=zigzag_chunk_ids, seq_dim=None):
    """Whole-sequence tensor from every rank's part (parts[r] of rank r, as shard() gives it).

    seq_dim: the sequence axis (default from the layout; 2 for the LSE [B, H, S])."""
    world = len(parts)
    dim = _seq_dim(layout) if seq_dim is None else seq_dim
    by_id = {}
    for r, p in enumerate(parts):
        ids = chunk_ids_of(r, world)
        for c, piece in zip(ids, p.chunk(len(ids), dim=dim)):
            by_id[c] = piece
    return torch.cat([by_id[c] for c in range(2 * world)], dim=dim)


def step_plan(rank, world, causal, chunk_ids_of=zigzag_chunk_ids):
    """The segments rank computes at each step: plan[t] = [(i, j_lo, j_hi, diagonal, first, last), ...].

    Segment (i, j_lo, j_hi, ...) is local query chunk i against held key chunks j_lo .. j_hi - 1, all
    entirely visible except the last when `diagonal`; first / last: the segment holds the first / the
    last contributing block of chunk i.  A step's blocks for one query chunk that do not form such a
    run become several segments (none do for the zigzag assignment)."""
    plan = [[] for _ in range(world)]
    for i, blocks in enumerate(contribution_plan(rank, world, causal, chunk_ids_of)):
        by_step = {}
        for (t, j, diag, first, last) in blocks:
            by_step.setdefault(t, []).append((j, diag, first, last))
        for t, bl in sorted(by_step.items()):
            bl.sort()
            run = [bl[0]]
            for b in bl[1:]:
                if b[0] == run[-1][0] + 1 and not run[-1][1]:
                    run.append(b)
                else:
                    plan[t].append((i, run[0][0], run[-1][0] + 1, run[-1][1], run[0][2], run[-1][3]))
                    run = [b]
            plan[t].append((i, run[0][0], run[-1][0] + 1, run[-1][1], run[0][2], run[-1][3]))
    return plan


# ----------------------------------------------------------------------------- the two compute steps


def fa_segments(segments, Sc):
    """fa_fwd_ring_step segments (row0, key0, keys, causal_offset, first, last) of a step's segments:
    local query chunk i is rows [i Sc, (i + 1) Sc); held key chunks j_lo .. j_hi - 1 are keys
    [j_lo Sc, j_hi Sc); a diagonal last chunk is the causal mask offset by the full chunks before it."""
    return [(i * Sc, j_lo * Sc, (j_hi - j_lo) * Sc, (j_hi - 1 - j_lo) * Sc if diag else -1, int(first), int(last))
            for (i, j_lo, j_hi, diag, first, last) in segments]


def launch_batches(segments):
    """The step's segments in launches of at most two, no query chunk twice in one launch (in order)."""
    batches, pending = [], list(segments)
    while pending:
        batch, used, rest = [], set(), []
        for g in pending:
            if g[0] in used or len(batch) == 2:
                rest.append(g)
            else:
                batch.append(g)
                used.add(g[0])
        batches.append(batch)
        pending = rest
    return batches


def _chunk(t, dim, i, Sc):
    return t.narrow(dim, i * Sc, Sc)


class CudaStepOps:
    """A step's segments through fa_fwd_ring_step: one launch per step (segments of one query chunk
    that a step splits further go to further launches)."""

    acc_dtype = torch.float32      # the running O
    lse_dtype = torch.float32      # the running and final LSE

    def __init__(self, layout, scale):
        from . import ring_step, fa_fwd_workspace_size
        self.layout, self.scale = layout, scale
        self._step = ring_step
        self._ws_bytes = fa_fwd_workspace_size()
        self._ws = None
        self.launches = 0

    def step(self, q, k, v, segments, Sc, out, lse, acc):
        if self._ws is None or self._ws.device != q.device:
            self._ws = torch.empty(self._ws_bytes, dtype=torch.uint8, device=q.device)
        for batch in launch_batches(segments):
            self._step(q, k, v, fa_segments(batch, Sc), Sc, out, lse, acc=acc, layout=self.layout,
                       scale=self.scale, workspace=self._ws)
            self.launches += 1


class BlockwiseStep:
    """A step composed of block attention and the merge of partial results, block by block:
    block(q, k, v, diagonal, o, lse) writes one block's normalised result, and
    merge(o_part, lse_part, o_acc, lse_acc, o_out, lse_out, accumulate, final) merges it into the
    running result.  The running LSE is kept in the output LSE, as fa_fwd_ring_step keeps it."""

    def __init__(self, block_ops):
        self.ops = block_ops
        self.layout = block_ops.layout
        self.acc_dtype, self.lse_dtype = block_ops.acc_dtype, block_ops.lse_dtype

    def step(self, q, k, v, segments, Sc, out, lse, acc):
        dim = _seq_dim(self.layout)
        for (i, j_lo, j_hi, diag, first, last) in segments:
            q_i, o_i, a_i = (_chunk(t, dim, i, Sc) for t in (q, out, acc if acc is not None else out))
            l_i = _chunk(lse, 2, i, Sc)
            for j in range(j_lo, j_hi):
                d = diag and j == j_hi - 1
                f = first and j == j_lo
                z = last and j == j_hi - 1
                if f and z:   # a single block: its result is the output
                    self.ops.block(q_i, _chunk(k, dim, j, Sc), _chunk(v, dim, j, Sc), d, o_i, l_i)
                    continue
                part = torch.empty(q_i.shape, dtype=q.dtype, device=q.device)
                part_lse = torch.empty(l_i.shape, dtype=self.lse_dtype, device=q.device)
                self.ops.block(q_i, _chunk(k, dim, j, Sc), _chunk(v, dim, j, Sc), d, part, part_lse)
                self.ops.merge(part, part_lse, a_i, l_i, o_i, l_i, accumulate=not f, final=z)


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
    """Runs one rank's part of ring attention; returns (o like q, lse [B, H, n * Sc]).

    q, k, v: this rank's local tensors (shard()).  exchange: post(step, k, v) / wait(handle) giving the
    next step's chunks.  ops: step(q, k, v, segments, Sc, out, lse, acc) (CudaStepOps or BlockwiseStep),
    acc_dtype, lse_dtype, layout."""
    if q.shape != k.shape or k.shape != v.shape:
        raise ValueError("ring attention here is self-attention: q, k and v must have one shape")
    n = len(chunk_ids_of(rank, world))
    layout = ops.layout
    dim = _seq_dim(layout)
    if layout == "BSND":
        B, S_loc, H, _ = q.shape
    else:
        B, H, S_loc, _ = q.shape
    if S_loc % n:
        raise ValueError(f"{S_loc} local rows do not split into {n} chunks")
    Sc = S_loc // n
    plan = step_plan(rank, world, causal, chunk_ids_of)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S_loc), dtype=ops.lse_dtype, device=q.device)
    needs_acc = any(not (g[4] and g[5]) for segs in plan for g in segs)
    acc = torch.empty(q.shape, dtype=ops.acc_dtype, device=q.device) if needs_acc else None
    cur_k, cur_v = k, v
    for t in range(world):
        handle = exchange.post(t, cur_k, cur_v)
        if plan[t]:
            ops.step(q, cur_k, cur_v, plan[t], Sc, out, lse, acc)
        if handle is not None:
            cur_k, cur_v = exchange.wait(handle)
    return out, lse


def ring_attention_forward(q, k, v, causal=False, scale=None, layout="BSND", group=None,
                           chunk_ids_of=zigzag_chunk_ids):
    """Ring attention over the ranks of `group` (torch.distributed, one GPU per rank).

    q, k, v: this rank's local CUDA tensors (see shard()).  Returns (o, lse) for this rank's query
    rows: o like q, lse fp32 [B, H, n * Sc].  scale=None uses 1/sqrt(D)."""
    import torch.distributed as dist
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if dist.is_available() and dist.is_initialized():
        exchange = P2PExchange(group)
        rank, world = exchange.rank, exchange.world
    else:
        rank, world = 0, 1
        exchange = LocalExchange(0, 1, [k], [v])
    return ring_steps(q, k, v, rank, world, exchange, CudaStepOps(layout, scale), causal, chunk_ids_of)


def ring_attention_emulated(q, k, v, world, causal=False, scale=None, layout="BSND",
                            chunk_ids_of=zigzag_chunk_ids, ops=None):
    """The ring schedule of `world` ranks run one rank after another on one device.

    q, k, v: whole-sequence tensors [B, S, H, D] / [B, H, S, D].  Returns whole-sequence (o, lse)
    assembled from the virtual ranks' results: the same steps as the real ring, with the transfers
    replaced by lookups (LocalExchange).  ops: a step implementation (default CudaStepOps)."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    ops = CudaStepOps(layout, scale) if ops is None else ops
    qs = [shard(q, r, world, layout, chunk_ids_of) for r in range(world)]
    ks = [shard(k, r, world, layout, chunk_ids_of) for r in range(world)]
    vs = [shard(v, r, world, layout, chunk_ids_of) for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        o, l = ring_steps(qs[r], ks[r], vs[r], r, world, LocalExchange(r, world, ks, vs), ops, causal, chunk_ids_of)
        outs.append(o)
        lses.append(l)
    return unshard(outs, layout, chunk_ids_of), unshard(lses, layout, chunk_ids_of, seq_dim=2)
