"""The online-softmax recurrence, written out in fp64 for small brute-force checks.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.

Page "FlashAttention: long-text inference without running out of memory"
(ai6s.net/6a0d42d8), section "FlashAttention's answer: tiling + online
normalisation", part 2 (Online Softmax): keep a running max m and a running
exp-sum l; for every new block of scores

    m_new = max(m_old, m_block)
    l_new = l_old * exp(m_old - m_new) + l_block * exp(m_block - m_new)

and use m_new, l_new for the softmax of the block.  The page states that the
result equals the global softmax.  Reading taken for what the page leaves
open: the weighted sum of V rows (the unnormalised output o) is carried and
rescaled exactly like l, block by block, and the output row is o / l at the
end; the row's log-sum-exp is m + ln(l).  (The same page also names the
rescale-as-you-go behaviour only in words; the "stable" variant printed on the
64K page is not followed: it merges the block max where the block's
log-sum-exp belongs.)

This module is checked against the two-pass oracle in the test suite: it pins
the recurrence that the CUDA kernel implements, not the oracle itself.
"""
import numpy as np


def block_stats(scores, vals):
    """m_block, l_block and the unnormalised o_block of one block of scores."""
    m_b = np.max(scores)
    e = np.exp(scores - m_b)
    return m_b, np.sum(e), e @ vals


def online_attention_row(scores, vals, block_sizes):
    """Attention output and log-sum-exp of one query row, block by block.

    scores: (Sk,) already-scaled, already-masked logits of the visible keys.
    vals: (Sk, D) the matching V rows.  block_sizes: positive ints summing to Sk.
    """
    scores = np.asarray(scores, dtype=np.float64)
    vals = np.asarray(vals, dtype=np.float64)
    if sum(block_sizes) != scores.shape[0] or min(block_sizes) <= 0:
        raise ValueError("block sizes must be positive and cover the row")
    m = -np.inf
    l = 0.0
    o = np.zeros(vals.shape[1], dtype=np.float64)
    start = 0
    for n in block_sizes:
        m_b, l_b, o_b = block_stats(scores[start:start + n], vals[start:start + n])
        m_new = max(m, m_b)
        a_old = np.exp(m - m_new) if m != -np.inf else 0.0
        a_blk = np.exp(m_b - m_new)
        l = l * a_old + l_b * a_blk
        o = o * a_old + o_b * a_blk
        m = m_new
        start += n
    return o / l, m + np.log(l)


def two_pass_row(scores, vals):
    """The same row the standard way: global max, global exp-sum, then the weighted sum."""
    scores = np.asarray(scores, dtype=np.float64)
    M = np.max(scores)
    e = np.exp(scores - M)
    L = np.sum(e)
    return (e @ np.asarray(vals, dtype=np.float64)) / L, M + np.log(L)
