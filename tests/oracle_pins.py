"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each pin_* function takes an oracle handle and raises AssertionError when the
oracle disagrees with a value fixed by the pages or by mathematics: a
hand-worked golden example with exact fractions, closed forms (scale = 0,
a single key, causal row 0, constant V), invariances (causal mask,
permutation of the keys, layout), a textbook cross-check against torch's
own softmax / logsumexp, and the row-subset API.  test_oracle.py runs them
against the oracle, and also against builds with planted mistakes to show
that every planted mistake is caught by at least one pin.
"""
import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _to_layout(x_bhsd, layout):
    """[B, H, S, D] -> the given layout (a copy)."""
    x = torch.as_tensor(x_bhsd)
    return x.permute(0, 2, 1, 3).contiguous() if layout == "BSND" else x.contiguous()


def _randn(shape, seed, std=1.0, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * std).to(dtype)


def textbook(q, k, v, causal, scale):
    """torch CPU fp64: softmax(scale * q k^T + top-left causal mask) v and logsumexp ([B,H,S,D] inputs)."""
    q, k, v = (t.to(torch.float64) for t in (q, k, v))
    s = torch.matmul(q, k.transpose(-2, -1)) * scale
    if causal:
        Sq, Sk = s.shape[-2], s.shape[-1]
        mask = torch.triu(torch.ones(Sq, Sk, dtype=torch.bool), diagonal=1)
        s = s.masked_fill(mask, float("-inf"))
    return torch.matmul(torch.softmax(s, dim=-1), v), torch.logsumexp(s, dim=-1)


# --------------------------------------------------------------------------- golden


def pin_golden_hand_worked(orc):
    with open(os.path.join(GOLDEN, "hand_worked_pow2.json")) as f:
        g = json.load(f)
    q = torch.tensor(g["q"], dtype=torch.float64)
    k = torch.tensor(g["k"], dtype=torch.float64)
    v = torch.tensor(g["v"], dtype=torch.float64)
    for case in g["cases"]:
        scale = {"ln2": math.log(2.0), "-ln2": -math.log(2.0)}[case["scale"]]
        o_ref = np.array(case["o"], dtype=np.float64)
        o_ref = o_ref[..., 0] / o_ref[..., 1]
        lse_ref = np.array(case["lse_exp"], dtype=np.float64)
        lse_ref = np.log(lse_ref[..., 0] / lse_ref[..., 1])
        for layout in ("BHSD", "BSND"):
            for dt in (torch.float64, torch.float16, torch.bfloat16):
                o, lse = orc.fwd(_to_layout(q, layout).to(dt), _to_layout(k, layout).to(dt),
                                 _to_layout(v, layout).to(dt), layout=layout,
                                 causal=case["causal"], scale=scale)
                assert np.max(np.abs(o - o_ref)) < 1e-14, (case["name"], layout, dt)
                assert np.max(np.abs(lse - lse_ref)) < 1e-14, (case["name"], layout, dt)


# --------------------------------------------------------------------------- textbook


TEXTBOOK_SHAPES = [
    # B, H, Sq, Sk, D, causal
    (1, 1, 1, 1, 8, False), (1, 2, 5, 7, 16, False), (2, 3, 9, 9, 8, True),
    (1, 2, 13, 6, 4, True), (1, 1, 6, 13, 4, True), (2, 1, 17, 33, 64, False),
    (1, 2, 40, 40, 128, True),
]


def pin_textbook_cross_check(orc):
    for n, (B, H, Sq, Sk, D, causal) in enumerate(TEXTBOOK_SHAPES):
        q = _randn((B, H, Sq, D), 100 + n)
        k = _randn((B, H, Sk, D), 200 + n)
        v = _randn((B, H, Sk, D), 300 + n)
        scale = 0.3 + 0.1 * n
        o_t, lse_t = textbook(q, k, v, causal, scale)
        for layout in ("BHSD", "BSND"):
            o, lse = orc.fwd(_to_layout(q, layout), _to_layout(k, layout), _to_layout(v, layout),
                             layout=layout, causal=causal, scale=scale)
            assert np.max(np.abs(o - o_t.numpy())) < 1e-12, (n, layout)
            assert np.max(np.abs(lse - lse_t.numpy())) < 1e-12, (n, layout)
    # 16-bit inputs: the oracle decodes the very bits torch holds
    for dt in (torch.float16, torch.bfloat16):
        q = _randn((1, 2, 11, 32), 7, dtype=dt)
        k = _randn((1, 2, 19, 32), 8, dtype=dt)
        v = _randn((1, 2, 19, 32), 9, dtype=dt)
        o_t, lse_t = textbook(q, k, v, True, 0.25)
        o, lse = orc.fwd(q, k, v, layout="BHSD", causal=True, scale=0.25)
        assert np.max(np.abs(o - o_t.numpy())) < 1e-12
        assert np.max(np.abs(lse - lse_t.numpy())) < 1e-12


# --------------------------------------------------------------------------- closed forms


def pin_scale_zero_is_mean(orc):
    """scale = 0: uniform weights over the visible keys -> O = mean of those V rows, LSE = ln(count)."""
    for (Sq, Sk, causal) in [(3, 1000, False), (5, 16001, False), (37, 37, True), (9, 4, True)]:
        q = _randn((1, 2, Sq, 8), 11)
        k = _randn((1, 2, Sk, 8), 12)
        v = _randn((1, 2, Sk, 8), 13)
        o, lse = orc.fwd(q, k, v, layout="BHSD", causal=causal, scale=0.0)
        vn = v.numpy()
        for i in range(Sq):
            n = min(i + 1, Sk) if causal else Sk
            assert np.max(np.abs(o[:, :, i] - vn[:, :, :n].mean(axis=2))) < 1e-12
            assert np.max(np.abs(lse[:, :, i] - math.log(n))) < 1e-12


def pin_single_key(orc):
    """Sk = 1: O = V[0] and LSE = scale * q . k0 (softmax over one element is 1)."""
    q = _randn((2, 3, 6, 16), 21)
    k = _randn((2, 3, 1, 16), 22)
    v = _randn((2, 3, 1, 16), 23)
    scale = 0.7
    for causal in (False, True):
        o, lse = orc.fwd(q, k, v, layout="BHSD", causal=causal, scale=scale)
        assert np.max(np.abs(o - v.numpy())) < 1e-14
        dots = np.einsum("bhid,bhd->bhi", q.numpy(), k.numpy()[:, :, 0])
        assert np.max(np.abs(lse - scale * dots)) < 1e-12


def pin_causal_row0(orc):
    """Causal: query 0 sees key 0 only -> O[0] = V[0], LSE[0] = scale * q0 . k0."""
    q = _randn((1, 2, 9, 8), 31)
    k = _randn((1, 2, 9, 8), 32)
    v = _randn((1, 2, 9, 8), 33)
    o, lse = orc.fwd(q, k, v, layout="BHSD", causal=True, scale=0.5)
    assert np.max(np.abs(o[:, :, 0] - v.numpy()[:, :, 0])) < 1e-14
    d0 = np.einsum("bhd,bhd->bh", q.numpy()[:, :, 0], k.numpy()[:, :, 0])
    assert np.max(np.abs(lse[:, :, 0] - 0.5 * d0)) < 1e-12


def pin_constant_v(orc):
    """V rows all equal to c -> O = c for every row (the weights sum to one)."""
    q = _randn((1, 2, 10, 8), 41)
    k = _randn((1, 2, 12, 8), 42)
    c = _randn((8,), 43)
    v = c.expand(1, 2, 12, 8).contiguous()
    for causal in (False, True):
        o, _ = orc.fwd(q, k, v, layout="BHSD", causal=causal, scale=1.3)
        assert np.max(np.abs(o - c.numpy())) < 1e-13


# --------------------------------------------------------------------------- invariances


def pin_causal_mask_ignores_future(orc):
    """Causal: changing K/V rows j > i leaves O[i] and LSE[i] unchanged; rows j <= i do change it."""
    Sq = Sk = 12
    q = _randn((1, 1, Sq, 8), 51)
    k = _randn((1, 1, Sk, 8), 52)
    v = _randn((1, 1, Sk, 8), 53)
    o, lse = orc.fwd(q, k, v, layout="BHSD", causal=True, scale=0.4)
    i = 5
    k2, v2 = k.clone(), v.clone()
    k2[:, :, i + 1:] += 3.0
    v2[:, :, i + 1:] -= 2.0
    o2, lse2 = orc.fwd(q, k2, v2, layout="BHSD", causal=True, scale=0.4)
    assert np.array_equal(o[:, :, : i + 1], o2[:, :, : i + 1])
    assert np.array_equal(lse[:, :, : i + 1], lse2[:, :, : i + 1])
    assert np.max(np.abs(o[:, :, i + 1:] - o2[:, :, i + 1:])) > 1e-3
    k3 = k.clone()
    k3[:, :, i] += 1.0
    o3, _ = orc.fwd(q, k3, v, layout="BHSD", causal=True, scale=0.4)
    assert np.max(np.abs(o[:, :, i] - o3[:, :, i])) > 1e-6


def pin_key_permutation_invariance(orc):
    """Non-causal: permuting the K and V rows together leaves every output row unchanged."""
    q = _randn((1, 2, 7, 16), 61)
    k = _randn((1, 2, 29, 16), 62)
    v = _randn((1, 2, 29, 16), 63)
    perm = torch.randperm(29, generator=torch.Generator().manual_seed(64))
    o, lse = orc.fwd(q, k, v, layout="BHSD", causal=False, scale=0.6)
    o2, lse2 = orc.fwd(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(),
                       layout="BHSD", causal=False, scale=0.6)
    assert np.max(np.abs(o - o2)) < 1e-12
    assert np.max(np.abs(lse - lse2)) < 1e-12
    # and the output does depend on which V row goes with which K row
    o3, _ = orc.fwd(q, k, v[:, :, perm].contiguous(), layout="BHSD", causal=False, scale=0.6)
    assert np.max(np.abs(o - o3)) > 1e-3


def pin_layout_equivalence(orc):
    """The same data in BSND and BHSD gives the same result (the oracle returns [B, H, S, D])."""
    q = _randn((2, 3, 11, 8), 71)
    k = _randn((2, 3, 13, 8), 72)
    v = _randn((2, 3, 13, 8), 73)
    for causal in (False, True):
        a = orc.fwd(q, k, v, layout="BHSD", causal=causal, scale=0.5)
        b = orc.fwd(_to_layout(q, "BSND"), _to_layout(k, "BSND"), _to_layout(v, "BSND"),
                    layout="BSND", causal=causal, scale=0.5)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def pin_weights_are_a_distribution(orc):
    """Every row's softmax weights are >= 0, sum to 1, and are 0 exactly on masked keys."""
    B, H, Sq, Sk, D = 1, 2, 6, 9, 8
    q = _randn((B, H, Sq, D), 81)
    k = _randn((B, H, Sk, D), 82)
    v = _randn((B, H, Sk, D), 83)
    for causal in (False, True):
        for row in range(B * H * Sq):
            w = orc.weights(q, k, v, row=row, layout="BHSD", causal=causal, scale=0.9)
            i = row % Sq
            assert np.all(w >= 0.0)
            assert abs(w.sum() - 1.0) < 1e-14
            if causal:
                assert np.all(w[i + 1:] == 0.0) and np.all(w[: i + 1] > 0.0)
            else:
                assert np.all(w > 0.0)


def pin_rows_subset_matches_full(orc):
    q = _randn((2, 2, 15, 8), 91)
    k = _randn((2, 2, 15, 8), 92)
    v = _randn((2, 2, 15, 8), 93)
    o, lse = orc.fwd(q, k, v, layout="BHSD", causal=True, scale=0.5)
    rows = np.array([0, 14, 15, 33, 59], dtype=np.int64)
    o_r, lse_r = orc.fwd(q, k, v, layout="BHSD", causal=True, scale=0.5, rows=rows)
    assert np.array_equal(o_r, o.reshape(-1, 8)[rows])
    assert np.array_equal(lse_r, lse.reshape(-1)[rows])


ALL_PINS = [
    pin_golden_hand_worked, pin_textbook_cross_check, pin_scale_zero_is_mean, pin_single_key,
    pin_causal_row0, pin_constant_v, pin_causal_mask_ignores_future,
    pin_key_permutation_invariance, pin_layout_equivalence, pin_weights_are_a_distribution,
    pin_rows_subset_matches_full,
]
