"""Pins of the oracle's packed variable-length entry (fwd_varlen), on the CPU.

Each sequence of a packed batch is the standard attention on its own rows.
The pins check the packing against facts that do not come from the oracle:
torch's own softmax per sequence, the scale = 0 closed form (mean of the
sequence's visible value rows, LSE = ln(count)), and isolation (another
sequence's keys and values do not matter).  A wrong offset or a leak across
sequences fails them.
"""
import math

import numpy as np
import pytest
import torch

from oracle_pins import textbook

LENGTHS = [(5, 9), (0, 4), (17, 17), (1, 3), (40, 11)]   # (query rows, keys) per sequence


def packed(lengths, H=2, D=8, seed=3, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    tq = sum(a for a, _ in lengths)
    tk = sum(b for _, b in lengths)
    q = torch.randn(tq, H, D, generator=g).to(dtype)
    k = torch.randn(tk, H, D, generator=g).to(dtype)
    v = torch.randn(tk, H, D, generator=g).to(dtype)
    cu_q = np.concatenate([[0], np.cumsum([a for a, _ in lengths])]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum([b for _, b in lengths])]).astype(np.int32)
    return q, k, v, cu_q, cu_k


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_matches_textbook_per_sequence(orc, causal):
    q, k, v, cu_q, cu_k = packed(LENGTHS)
    scale = 0.37
    o, lse = orc.fwd_varlen(q, k, v, cu_q, cu_k, causal=causal, scale=scale)
    for b in range(len(LENGTHS)):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if q1 == q0:
            continue
        # [S, H, D] -> [1, H, S, D]
        to4 = lambda x: x.permute(1, 0, 2).unsqueeze(0)
        ot, lt = textbook(to4(q[q0:q1]), to4(k[k0:k1]), to4(v[k0:k1]), causal, scale)
        assert np.max(np.abs(o[q0:q1] - ot[0].permute(1, 0, 2).numpy())) < 1e-12
        assert np.max(np.abs(lse[:, q0:q1] - lt[0].numpy())) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_scale_zero_is_mean_of_own_rows(orc, causal):
    q, k, v, cu_q, cu_k = packed(LENGTHS, dtype=torch.float64)
    o, lse = orc.fwd_varlen(q, k, v, cu_q, cu_k, causal=causal, scale=0.0)
    vv = v.numpy()
    for b in range(len(LENGTHS)):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        for i in range(q1 - q0):
            n = min(i + 1, k1 - k0) if causal else k1 - k0
            assert np.max(np.abs(o[q0 + i] - vv[k0:k0 + n].mean(axis=0))) < 1e-12
            assert np.max(np.abs(lse[:, q0 + i] - math.log(n))) < 1e-12


def test_varlen_sequences_are_isolated(orc):
    q, k, v, cu_q, cu_k = packed(LENGTHS)
    o1, l1 = orc.fwd_varlen(q, k, v, cu_q, cu_k, causal=True, scale=0.3)
    k2, v2 = k.clone(), v.clone()
    k2[cu_k[2]:cu_k[3]] = -k2[cu_k[2]:cu_k[3]]
    v2[cu_k[2]:cu_k[3]] = v2[cu_k[2]:cu_k[3]] * 2
    o2, l2 = orc.fwd_varlen(q, k2, v2, cu_q, cu_k, causal=True, scale=0.3)
    inside = np.zeros(o1.shape[0], dtype=bool)
    inside[cu_q[2]:cu_q[3]] = True
    assert np.array_equal(o1[~inside], o2[~inside]) and np.array_equal(l1[:, ~inside], l2[:, ~inside])
    assert not np.allclose(o1[inside], o2[inside])


def test_varlen_queries_without_keys_rejected(orc):
    q, k, v, cu_q, cu_k = packed([(3, 4), (2, 0)])
    with pytest.raises(ValueError):
        orc.fwd_varlen(q, k, v, cu_q, cu_k)


def test_varlen_row_subset_matches_full(orc):
    q, k, v, cu_q, cu_k = packed(LENGTHS)
    o, lse = orc.fwd_varlen(q, k, v, cu_q, cu_k, causal=True, scale=0.5)
    rows = np.array([0, 4, 5, 22, 23, 60, 61, 62], dtype=np.int64)
    os_, ls = orc.fwd_varlen(q, k, v, cu_q, cu_k, causal=True, scale=0.5, rows=rows)
    assert np.array_equal(os_, o[rows]) and np.array_equal(ls, lse[:, rows])
