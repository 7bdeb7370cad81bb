"""Merge of partial attention results over disjoint key blocks, in fp64.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only the test suite, the package smoke
check and the benchmark may import it.  It shares no code with the CUDA path.

Attention split by key ranges (ring attention for long sequences: page
"FlashAttention in ops-transformer on Ascend NPU" (ai6s.net/6a0d3bfb),
section "what else is in the ops-transformer repository"; several cards per
64K sequence: page "64K long-sequence FlashAttention" (ai6s.net/6a140d07),
section "performance tuning tips", multi-card parallelism) yields per query
row one partial (O_i, LSE_i) per key block, each normalised over its own
block.  They combine by the running-max / running-sum update of page
"FlashAttention: long-text inference without running out of memory"
(ai6s.net/6a0d42d8), section "FlashAttention's answer: tiling + online
normalisation", taken one whole block at a time.  Reading taken: a block's
statistics, relative to the reference point m_b = LSE_i, are l_b = 1 (its
weights sum to one there) and o_b = O_i, because sum_j exp(s_j - LSE_i) = 1
and sum_j exp(s_j - LSE_i) v_j = O_i.  Then, block after block,

    m_new = max(m, m_b)
    l     = l * exp(m - m_new) + l_b * exp(m_b - m_new)
    o     = o * exp(m - m_new) + o_b * exp(m_b - m_new)

and the merged row is O = o / l, LSE = m + ln(l).  A block with LSE = -inf
(no visible key) contributes nothing.  Pinned in the tests against attention
computed directly over the whole key range (not through this module).
"""
import numpy as np


def merge_partials(o_parts, lse_parts):
    """o_parts: sequence of arrays [..., D]; lse_parts: matching arrays [...] (natural log).

    Returns (O, LSE) in fp64 over the union of the blocks.  Rows where every
    block is empty get O = 0 and LSE = -inf."""
    if len(o_parts) == 0 or len(o_parts) != len(lse_parts):
        raise ValueError("need one LSE array per partial output, and at least one of each")
    o_parts = [np.asarray(o, dtype=np.float64) for o in o_parts]
    lse_parts = [np.asarray(x, dtype=np.float64) for x in lse_parts]
    shape = lse_parts[0].shape
    m = np.full(shape, -np.inf)
    l = np.zeros(shape)
    o = np.zeros(o_parts[0].shape)
    for o_b, m_b in zip(o_parts, lse_parts):
        m_new = np.maximum(m, m_b)
        live = m_new > -np.inf
        safe = np.where(live, m_new, 0.0)
        a_old = np.where(live & (m > -np.inf), np.exp(np.where(live, m, 0.0) - safe), 0.0)
        a_blk = np.where(live & (m_b > -np.inf), np.exp(np.where(live, m_b, 0.0) - safe), 0.0)
        l = l * a_old + a_blk
        o = o * a_old[..., None] + o_b * a_blk[..., None]
        m = m_new
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where((l > 0)[..., None], o / np.where(l > 0, l, 1.0)[..., None], 0.0)
        lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return out, lse
