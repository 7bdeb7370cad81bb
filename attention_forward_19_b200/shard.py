"""The heads of one attention problem split across GPUs (one process per GPU).

Every (batch, head) pair is an independent attention problem, so a forward
pass over B * H heads shards across ranks with no exchange during the pass
(page "64K long-sequence FlashAttention" (ai6s.net/6a140d07), section
"performance tuning tips", multi-card model parallelism; the split of the work
into balanced shares follows section "multi-AI-Core load balancing").  Each
rank owns a contiguous range of the flattened heads g = b * H + h, computes it
with fa_fwd_heads in place in the whole problem's tensors, and writes only its
own rows of O and LSE.  If every rank needs the whole result, all_gather_heads
then sends each rank's rows to the others (NCCL broadcasts on GPUs, gloo in
the CPU tests); the pass itself never waits on another rank.

The ranges balance work, not head counts: a head's cost is the number of
key/value tile steps the kernel runs for it (its work units' key tiles, the
same count the kernel's schedule walks), and the ranges minimise the largest
rank's cost.  In a dense batch every head costs the same, so the ranges differ
by at most one head.
"""
BM = 128          # query rows per tile
BN = 128          # keys per key/value tile


def head_cost(Sq, Sk, causal):
    """Key/value tile steps of one head: for every 128-row query tile, the key tiles it visits
    (causal: up to the tile holding its last visible key, which is its last row)."""
    if Sq <= 0 or Sk <= 0:
        return 0
    tk = (Sk + BN - 1) // BN
    if not causal:
        return ((Sq + BM - 1) // BM) * tk
    steps = 0
    for first in range(0, Sq, BM):
        last_row = min(first + BM, Sq) - 1
        steps += min(last_row, Sk - 1) // BN + 1
    return steps


def _ranks_needed(costs, cap):
    n, acc = 1, 0
    for c in costs:
        if acc + c > cap:
            n += 1
            acc = c
        else:
            acc += c
    return n


def partition(costs, world):
    """Contiguous ranges [(begin, count)] of the items, one per rank, whose largest summed cost
    is the least possible; among such splits, the boundaries are placed where the running cost
    crosses r / world of the total when that keeps the bound (an even split), else greedily.
    Ranks may get count 0 when there are fewer items than ranks."""
    costs = [int(c) for c in costs]
    if world < 1:
        raise ValueError("world must be >= 1")
    if any(c < 0 for c in costs):
        raise ValueError("costs must be >= 0")
    n = len(costs)
    if n == 0:
        return [(0, 0)] * world
    lo, hi = max(costs), sum(costs)
    while lo < hi:                               # least cap that `world` contiguous ranges can meet
        mid = (lo + hi) // 2
        if _ranks_needed(costs, mid) <= world:
            hi = mid
        else:
            lo = mid + 1
    cap = lo
    prefix = [0]
    for c in costs:
        prefix.append(prefix[-1] + c)
    total = prefix[-1]
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        i = min(range(bounds[-1], n + 1), key=lambda j: (abs(prefix[j] - target), j))
        bounds.append(i)
    bounds.append(n)
    even = [(bounds[r], bounds[r + 1] - bounds[r]) for r in range(world)]
    if max(prefix[b + c] - prefix[b] for b, c in even) <= cap:
        return even
    out, begin, acc = [], 0, 0
    for i, c in enumerate(costs):
        if acc + c > cap and len(out) < world - 1:
            out.append((begin, i - begin))
            begin, acc = i, 0
        acc += c
    out.append((begin, n - begin))
    out.extend([(n, 0)] * (world - len(out)))
    return out


def head_ranges(B, H, Sq, Sk, causal, world):
    """The balanced contiguous head ranges [(head_begin, head_count)] of a dense B x H problem."""
    return partition([head_cost(Sq, Sk, causal)] * (B * H), world)


def head_rows(t, begin, count, layout, H):
    """Views of the rows of heads [begin, begin + count) in a 4-D q/k/v/o-shaped tensor t (BSND
    [B, S, H, D] or BHSD [B, H, S, D]) or in a 3-D [B, H, S] LSE tensor: one view per batch the
    range touches.  BHSD and LSE rows of a head range are one contiguous block per batch; BSND
    rows are strided (heads are the inner axis)."""
    views = []
    g = begin
    while g < begin + count:
        b, h0 = divmod(g, H)
        h1 = min(H, h0 + (begin + count - g))
        if t.dim() == 3 or layout == "BHSD":
            views.append(t[b, h0:h1])
        else:
            views.append(t[b, :, h0:h1])
        g += h1 - h0
    return views


def all_gather_heads(o, lse, ranges, layout, group=None):
    """Sends every rank's head rows of o and lse to all ranks (in place: on return every rank's
    o and lse hold the whole result).  ranges[r] = (head_begin, head_count) of rank r.  Contiguous
    row blocks are broadcast directly; strided ones (BSND) through a packed copy."""
    import torch
    import torch.distributed as dist
    H = lse.shape[1]
    me = dist.get_rank(group) if group is not None else dist.get_rank()
    for src, (begin, count) in enumerate(ranges):
        if count == 0:
            continue
        gsrc = dist.get_global_rank(group, src) if group is not None else src
        for t in (o, lse):
            for view in head_rows(t, begin, count, layout, H):
                if view.is_contiguous():
                    dist.broadcast(view, gsrc, group=group)
                else:
                    buf = view.contiguous() if me == src else torch.empty(view.shape, dtype=view.dtype,
                                                                         device=view.device)
                    dist.broadcast(buf, gsrc, group=group)
                    if me != src:
                        view.copy_(buf)


def flops_of_heads(count, Sq, Sk, D, causal):
    """The metric's flops for `count` heads: 4 Sq Sk D each, halved when causal."""
    f = 4.0 * count * Sq * Sk * D
    return f / 2 if causal else f

