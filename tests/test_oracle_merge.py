"""Pins of the oracle's merge of partial attention results (oracle/merge.py).

The merge is checked against attention computed directly over the whole key
range by the two-pass definition (oracle/online_softmax.two_pass_row and the C
oracle), never through the merge itself.
"""
import numpy as np
import pytest
import torch

from oracle import attn as oracle_attn
from oracle.merge import merge_partials
from oracle.online_softmax import two_pass_row


def _row_partials(scores, vals, sizes):
    o_parts, lse_parts, start = [], [], 0
    for n in sizes:
        o, l = two_pass_row(scores[start:start + n], vals[start:start + n])
        o_parts.append(o)
        lse_parts.append(np.float64(l))
        start += n
    return o_parts, lse_parts


@pytest.mark.parametrize("seed", range(6))
def test_merge_of_block_partials_equals_the_whole_row(seed):
    rng = np.random.default_rng(100 + seed)
    Sk, D = int(rng.integers(2, 60)), 8
    scores = rng.normal(0.0, 4.0, Sk)
    vals = rng.normal(size=(Sk, D))
    cuts = sorted(set(rng.integers(1, Sk, size=int(rng.integers(1, 6))).tolist()))
    sizes = np.diff([0] + cuts + [Sk]).tolist()
    if seed == 0:
        sizes = [1] * Sk                  # every block a single key
    o_parts, lse_parts = _row_partials(scores, vals, sizes)
    o, lse = merge_partials(o_parts, lse_parts)
    o_ref, lse_ref = two_pass_row(scores, vals)
    assert np.max(np.abs(o - o_ref)) < 1e-12
    assert abs(lse - lse_ref) < 1e-12


def test_merge_is_order_independent_and_single_partial_is_identity():
    rng = np.random.default_rng(7)
    o_parts = [rng.normal(size=(3, 5, 16)) for _ in range(4)]
    lse_parts = [rng.normal(0, 3, size=(3, 5)) for _ in range(4)]
    a = merge_partials(o_parts, lse_parts)
    b = merge_partials(o_parts[::-1], lse_parts[::-1])
    assert np.max(np.abs(a[0] - b[0])) < 1e-12 and np.max(np.abs(a[1] - b[1])) < 1e-12
    one = merge_partials(o_parts[:1], lse_parts[:1])
    assert np.array_equal(one[0], o_parts[0]) and np.allclose(one[1], lse_parts[0], rtol=0, atol=1e-15)


def test_empty_partials_contribute_nothing():
    rng = np.random.default_rng(8)
    o0, l0 = rng.normal(size=(4, 8)), rng.normal(size=4)
    empty_o, empty_l = np.zeros((4, 8)), np.full(4, -np.inf)
    o, l = merge_partials([empty_o, o0, empty_o], [empty_l, l0, empty_l])
    assert np.max(np.abs(o - o0)) < 1e-15 and np.max(np.abs(l - l0)) < 1e-15
    o, l = merge_partials([empty_o, empty_o], [empty_l, empty_l])
    assert np.all(o == 0) and np.all(l == -np.inf)


def test_equal_lse_partials_average_with_log2_offset():
    # two blocks of equal total weight: O is the mean, LSE grows by ln 2 (closed form)
    o_a, o_b = np.array([[1.0, 3.0]]), np.array([[5.0, -1.0]])
    o, l = merge_partials([o_a, o_b], [np.array([0.25]), np.array([0.25])])
    assert np.allclose(o, [[3.0, 1.0]], rtol=0, atol=1e-15)
    assert abs(l[0] - (0.25 + np.log(2.0))) < 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_key_split_of_c_oracle_merges_to_the_whole(causal):
    # attention over keys [0, Sk) from the C oracle, against merged partials over key
    # blocks; a causal split is taken on a query block that lies below every key block,
    # so that every block is fully visible and the mask of the whole is the plain one
    g = torch.Generator().manual_seed(11)
    B, H, S, D = 1, 2, 48, 16
    q = torch.randn(B, H, S, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, H, S, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, H, S, D, generator=g, dtype=torch.float64)
    orc = oracle_attn.default()
    o_ref, l_ref = orc.fwd(q, k, v, layout="BHSD", causal=causal)
    if causal:
        qb = q[:, :, 32:]                     # rows 32..47 see keys 0..row
        parts = [(k[:, :, :16], v[:, :, :16], False), (k[:, :, 16:32], v[:, :, 16:32], False),
                 (k[:, :, 32:], v[:, :, 32:], True)]
        o_ref, l_ref = o_ref[:, :, 32:], l_ref[:, :, 32:]
    else:
        qb = q
        parts = [(k[:, :, a:b], v[:, :, a:b], False) for a, b in ((0, 5), (5, 6), (6, 30), (30, 48))]
    o_parts, l_parts = [], []
    for kb, vb, diag in parts:
        o, l = orc.fwd(qb.contiguous(), kb.contiguous(), vb.contiguous(), layout="BHSD", causal=diag)
        o_parts.append(o)
        l_parts.append(l)
    o, l = merge_partials(o_parts, l_parts)
    assert np.max(np.abs(o - o_ref)) < 1e-12
    assert np.max(np.abs(l - l_ref)) < 1e-12
