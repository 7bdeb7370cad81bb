"""Pins of the backward oracle (oracle/attn_bwd.py) to facts outside it: torch
autograd through the textbook forward, central finite differences, the
explicit softmax Jacobian, and closed forms (sum over keys of dK is 0, sum of
dV is the sum of dO, identical keys give dQ = 0, causal row 0 has dQ = 0,
causal dK/dV of key j ignore queries i < j)."""
import numpy as np
import pytest
import torch

from oracle import attn_bwd
from oracle_pins import textbook


def rnd(shape, seed, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64).to(dtype)


SHAPES = [  # B, H, Sq, Sk, D, causal, layout
    (1, 2, 9, 9, 8, False, "BHSD"),
    (2, 1, 7, 12, 8, True, "BHSD"),
    (1, 3, 12, 5, 4, True, "BSND"),
    (1, 1, 16, 16, 16, False, "BSND"),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", [torch.float64, torch.bfloat16])
def test_matches_autograd(shape, dtype):
    B, H, Sq, Sk, D, causal, layout = shape
    scale = 0.43
    q, k, v = rnd((B, H, Sq, D), 1, dtype), rnd((B, H, Sk, D), 2, dtype), rnd((B, H, Sk, D), 3, dtype)
    do = rnd((B, H, Sq, D), 4, dtype)
    to_lay = (lambda t: t.permute(0, 2, 1, 3).contiguous()) if layout == "BSND" else (lambda t: t)
    o, lse, dq, dk, dv = attn_bwd.attention_fwd_bwd(to_lay(q), to_lay(k), to_lay(v), to_lay(do), layout=layout,
                                                    causal=causal, scale=scale)
    qt, kt, vt = (t.to(torch.float64).clone().requires_grad_(True) for t in (q, k, v))
    ot, lt = textbook(qt, kt, vt, causal, scale)
    (ot * do.to(torch.float64)).sum().backward()
    assert np.max(np.abs(o - ot.detach().numpy())) < 1e-12
    assert np.max(np.abs(lse - lt.detach().numpy())) < 1e-12
    assert np.max(np.abs(dq - qt.grad.numpy())) < 1e-11
    assert np.max(np.abs(dk - kt.grad.numpy())) < 1e-11
    assert np.max(np.abs(dv - vt.grad.numpy())) < 1e-11


def test_finite_differences():
    B, H, Sq, Sk, D = 1, 1, 4, 5, 3
    q, k, v, do = rnd((B, H, Sq, D), 5), rnd((B, H, Sk, D), 6), rnd((B, H, Sk, D), 7), rnd((B, H, Sq, D), 8)
    scale, causal, h = 0.7, True, 1e-6
    _, _, dq, dk, dv = attn_bwd.attention_fwd_bwd(q, k, v, do, causal=causal, scale=scale)

    def loss(q_, k_, v_):
        o, _ = textbook(q_, k_, v_, causal, scale)
        return float((o * do).sum())

    for name, t, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 0, 0), (0, 0, 2, 1), (0, 0, 3, 2)]:
            if idx[2] >= t.shape[2]:
                continue
            tp, tm = t.clone(), t.clone()
            tp[idx] += h
            tm[idx] -= h
            args_p = {"q": (tp, k, v), "k": (q, tp, v), "v": (q, k, tp)}[name]
            args_m = {"q": (tm, k, v), "k": (q, tm, v), "v": (q, k, tm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) < 1e-7, (name, idx, fd, g[idx])


def test_softmax_jacobian_closed_form():
    g = np.random.default_rng(3)
    s = g.normal(size=(6, 9))
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dp = g.normal(size=(6, 9))
    closed = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    assert np.max(np.abs(attn_bwd.softmax_backward_rows(dp, p) - closed)) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_sums_over_keys(causal):
    B, H, Sq, Sk, D = 1, 2, 11, 11, 8
    q, k, v, do = rnd((B, H, Sq, D), 9), rnd((B, H, Sk, D), 10), rnd((B, H, Sk, D), 11), rnd((B, H, Sq, D), 12)
    _, _, dq, dk, dv = attn_bwd.attention_fwd_bwd(q, k, v, do, causal=causal, scale=0.3)
    assert np.max(np.abs(dk.sum(axis=2))) < 1e-12
    assert np.max(np.abs(dv.sum(axis=2) - do.numpy().sum(axis=2))) < 1e-12


def test_identical_keys_give_zero_dq():
    B, H, Sq, Sk, D = 1, 1, 6, 7, 4
    q, v, do = rnd((B, H, Sq, D), 13), rnd((B, H, Sk, D), 14), rnd((B, H, Sq, D), 15)
    k = rnd((B, H, 1, D), 16).expand(B, H, Sk, D).contiguous()
    _, _, dq, _, _ = attn_bwd.attention_fwd_bwd(q, k, v, do, scale=0.9)
    assert np.max(np.abs(dq)) < 1e-13


def test_causal_row0_and_future_independence():
    B, H, S, D = 1, 1, 8, 4
    q, k, v, do = rnd((B, H, S, D), 17), rnd((B, H, S, D), 18), rnd((B, H, S, D), 19), rnd((B, H, S, D), 20)
    _, _, dq, dk, dv = attn_bwd.attention_fwd_bwd(q, k, v, do, causal=True, scale=0.5)
    assert np.max(np.abs(dq[0, 0, 0])) < 1e-15          # row 0 attends to key 0 only: dS = 0
    do2 = do.clone()
    do2[0, 0, :3] += 1.0                                  # queries 0..2 change
    _, _, _, dk2, dv2 = attn_bwd.attention_fwd_bwd(q, k, v, do2, causal=True, scale=0.5)
    assert np.array_equal(dk[0, 0, 3:], dk2[0, 0, 3:]) and np.array_equal(dv[0, 0, 3:], dv2[0, 0, 3:])
    assert not np.allclose(dv[0, 0, :3], dv2[0, 0, :3])
