"""Planted mistakes in the Python oracles (merge of partial results, output
projection): each wrong variant, written here on the CPU, must fail at least
one of the pins that the real oracle passes.  This shows the pins are strong
enough to catch a dropped term, a wrong sign or index, or a transposed operand.
"""
import numpy as np
import pytest
import torch

from oracle import merge as merge_mod
from oracle import proj as proj_mod
from oracle.online_softmax import two_pass_row


# ----------------------------------------------------------------------------- merge


def _merge_variant(plant):
    """A merge with one planted mistake (plant = 0: the real oracle)."""
    if plant == 0:
        return merge_mod.merge_partials

    def merged(o_parts, lse_parts):
        o_parts = [np.asarray(o, dtype=np.float64) for o in o_parts]
        lse_parts = [np.asarray(x, dtype=np.float64) for x in lse_parts]
        m = np.full(lse_parts[0].shape, -np.inf)
        l = np.zeros(lse_parts[0].shape)
        o = np.zeros(o_parts[0].shape)
        for o_b, m_b in zip(o_parts, lse_parts):
            m_new = np.maximum(m, m_b)
            a_old = np.where(m > -np.inf, np.exp(m - m_new), 0.0)
            a_blk = np.where(m_b > -np.inf, np.exp(m_b - m_new), 0.0)
            if plant == 1:                       # the running sum is not rescaled
                l = l + a_blk
            elif plant == 2:                     # the block's weight has the wrong sign in the exponent
                a_blk = np.where(m_b > -np.inf, np.exp(m_new - m_b), 0.0)
                l = l * a_old + a_blk
            else:
                l = l * a_old + a_blk
            if plant == 3:                       # the running output is not rescaled
                o = o + o_b * a_blk[..., None]
            else:
                o = o * a_old[..., None] + o_b * a_blk[..., None]
            m = m_new
        if plant == 4:                           # LSE without the running sum
            return o / l[..., None], m
        if plant == 5:                           # output not normalised
            return o, m + np.log(l)
        return o / l[..., None], m + np.log(l)
    return merged


def _merge_pins_pass(merge):
    """The pins of tests/test_oracle_merge.py as one predicate."""
    rng = np.random.default_rng(5)
    for trial in range(4):
        Sk, D = int(rng.integers(8, 40)), 4
        scores = rng.normal(0.0, 4.0, Sk)
        vals = rng.normal(size=(Sk, D))
        cuts = sorted(set(rng.integers(1, Sk, size=3).tolist()))
        sizes = np.diff([0] + cuts + [Sk]).tolist()
        o_parts, lse_parts, start = [], [], 0
        for n in sizes:
            o, l = two_pass_row(scores[start:start + n], vals[start:start + n])
            o_parts.append(o)
            lse_parts.append(np.float64(l))
            start += n
        o, lse = merge(o_parts, lse_parts)
        o_ref, lse_ref = two_pass_row(scores, vals)
        if not (np.max(np.abs(o - o_ref)) < 1e-12 and abs(lse - lse_ref) < 1e-12):
            return False
    o, l = merge([np.array([[1.0, 3.0]]), np.array([[5.0, -1.0]])], [np.array([0.25]), np.array([0.25])])
    return bool(np.allclose(o, [[3.0, 1.0]], rtol=0, atol=1e-15) and abs(l[0] - (0.25 + np.log(2.0))) < 1e-15)


def test_real_merge_passes_the_pins():
    assert _merge_pins_pass(_merge_variant(0))


@pytest.mark.parametrize("plant", [1, 2, 3, 4, 5])
def test_planted_merge_mistake_fails_a_pin(plant):
    assert not _merge_pins_pass(_merge_variant(plant))


# ----------------------------------------------------------------------------- projection


def _proj_variant(plant):
    if plant == 0:
        return proj_mod.out_proj

    def projected(o, w, layout="BSND"):
        oa = torch.as_tensor(o).double().numpy()
        if layout == "BHSD":
            oa = oa.transpose(0, 2, 1, 3)
        B, S, H, D = oa.shape
        wa = torch.as_tensor(w).double().numpy()
        if plant == 1:                           # inputs flattened dim-major instead of head-major
            a = oa.transpose(0, 1, 3, 2).reshape(B, S, H * D)
        elif plant == 2:                         # the last head dropped
            a = oa.copy()
            a[:, :, H - 1, :] = 0.0
            a = a.reshape(B, S, H * D)
        elif plant == 3:                         # the layout flag ignored (BHSD read as BSND)
            a = torch.as_tensor(o).double().numpy().reshape(B, S, H * D)
        else:
            a = oa.reshape(B, S, H * D)
        if plant == 4:                           # the weight used untransposed (square case only)
            return a @ wa
        return a @ wa.T
    return projected


def _proj_pins_pass(proj):
    g = torch.Generator().manual_seed(1)
    B, S, H, D = 1, 5, 3, 4
    o_bsnd = torch.randn(B, S, H, D, generator=g, dtype=torch.float64)
    for layout in ("BSND", "BHSD"):
        o = o_bsnd if layout == "BSND" else o_bsnd.permute(0, 2, 1, 3).contiguous()
        y = proj(o, torch.eye(H * D, dtype=torch.float64), layout)
        for h in range(H):
            if not np.array_equal(y[0, :, h * D:(h + 1) * D], o_bsnd[0, :, h].numpy()):
                return False
    w = torch.randn(H * D, H * D, generator=g, dtype=torch.float64)       # square, so a transpose still runs
    y = proj(o_bsnd, w, "BSND")
    for s in range(S):
        for n in range(H * D):
            acc = sum(float(o_bsnd[0, s, h, d]) * float(w[n, h * D + d]) for h in range(H) for d in range(D))
            if abs(y[0, s, n] - acc) > 1e-12:
                return False
    return True


def test_real_projection_passes_the_pins():
    assert _proj_pins_pass(_proj_variant(0))


@pytest.mark.parametrize("plant", [1, 2, 3, 4])
def test_planted_projection_mistake_fails_a_pin(plant):
    assert not _proj_pins_pass(_proj_variant(plant))


# ----------------------------------------------------------------------------- backward


def _bwd_variant(plant):
    """The backward of one (batch, head) with one planted mistake (plant = 0: the oracle's own function)."""
    from oracle import attn_bwd

    if plant == 0:
        def real(q, k, v, do, causal, scale):
            _, _, dq, dk, dv = attn_bwd.attention_fwd_bwd(q[None, None], k[None, None], v[None, None],
                                                          do[None, None], layout="BHSD", causal=causal, scale=scale)
            return dq[0, 0], dk[0, 0], dv[0, 0]
        return real

    def wrong(q, k, v, do, causal, scale):
        q, k, v, do = (t.double().numpy() for t in (q, k, v, do))
        Sq, Sk = q.shape[0], k.shape[0]
        s = scale * (q @ k.T)
        if causal:
            s = np.where(np.arange(Sk)[None, :] <= np.arange(Sq)[:, None], s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o = p @ v
        dv = (p @ do) if plant == 1 else (p.T @ do)             # 1: P where P^T belongs (square case)
        dp = do @ v.T
        d_row = (do * o).sum(axis=1, keepdims=True)
        ds = p * dp if plant == 2 else p * (dp - d_row)           # 2: the row sum D dropped
        dq = (ds @ k) if plant == 3 else scale * (ds @ k)         # 3: dQ without the scale
        dk = scale * (ds @ q) if plant == 4 else scale * (ds.T @ q)   # 4: dS where dS^T belongs
        return dq, dk, dv
    return wrong


def _bwd_pin_passes(bwd):
    """Agreement with torch autograd through the textbook forward (the first pin of test_oracle_bwd.py)."""
    g = torch.Generator().manual_seed(3)
    S, D, scale = 9, 8, 0.43
    q, k, v, do = (torch.randn(S, D, generator=g, dtype=torch.float64) for _ in range(4))
    for causal in (False, True):
        dq, dk, dv = bwd(q, k, v, do, causal, scale)
        qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
        s = scale * qt @ kt.T
        if causal:
            s = s.masked_fill(torch.triu(torch.ones(S, S, dtype=torch.bool), 1), float("-inf"))
        (torch.softmax(s, dim=-1) @ vt * do).sum().backward()
        for mine, ref in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
            if not np.max(np.abs(np.asarray(mine) - ref.numpy())) < 1e-10:
                return False
    return True


def test_real_backward_passes_the_autograd_pin():
    assert _bwd_pin_passes(_bwd_variant(0))


@pytest.mark.parametrize("plant", [1, 2, 3, 4])
def test_planted_backward_mistake_fails_the_autograd_pin(plant):
    assert not _bwd_pin_passes(_bwd_variant(plant))
