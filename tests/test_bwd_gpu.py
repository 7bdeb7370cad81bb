"""GPU parity of the backward pass (fa_bwd) against the fp64 backward oracle,
through the C ABI, with the GPU forward's o and lse as its inputs (the normal
use).

Tolerance (no bound on the pages or in the target, which covers the forward):
each gradient is rounded once to the input dtype, and the weights P and dS are
rounded to it before the tile products; both are relative errors of at most
the unit roundoff u (2^-8 bf16, 2^-11 fp16).  The test allows 4u relative to
the largest entry of each reference gradient: max |g - g_ref| <=
4u * max |g_ref| (bf16: 2^-6, fp16: 2^-9).  Measured errors are 1.5-2x u.

The non-deterministic variant (fa_bwd_atomic, D = 64 and 128) is held to the
same bound on the same cases, and on more D = 64 shapes; its dQ is summed in
fp32 in whatever order the key tiles finish, so two runs may differ in dq by
fp32 rounding, while dk and dv are reproducible.
"""
import math

import numpy as np
import pytest
import torch

import attention_forward_19_b200 as fa
from fa_inputs import WORKLOADS, Workload, make_dout, make_qkv
from oracle import attn_bwd

pytestmark = pytest.mark.gpu

REL_TOL = {"bf16": 2.0 ** -6, "fp16": 2.0 ** -9}


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def W(dtype, layout, B, H, Sq, Sk, D, causal, scale=None, seed=3, qk_std=1.0):
    return Workload(f"{dtype}_{layout}_b{B}_h{H}_q{Sq}_k{Sk}_d{D}_{'c' if causal else 'n'}", dtype, layout, B, H, Sq,
                    Sk, D, causal, 1.0 / math.sqrt(D) if scale is None else scale, qk_std=qk_std, seed=seed)


def run(w, deterministic=True):
    q, k, v = make_qkv(w)
    do = make_dout(w)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.flash_attention_forward(qd, kd, vd, layout=w.layout, causal=w.causal, scale=w.scale)
    dq, dk, dv = fa.flash_attention_backward(qd, kd, vd, o, lse, dod, layout=w.layout, causal=w.causal,
                                             scale=w.scale, deterministic=deterministic)
    fa.check_device_status()
    return (q, k, v, do), (dq, dk, dv)


def to_bhsd(t, layout):
    t = t.cpu().to(torch.float64)
    return (t.permute(0, 2, 1, 3) if layout == "BSND" else t).numpy()


def check(w, inputs, grads, tag="bwd"):
    q, k, v, do = inputs
    _, _, rq, rk, rv = attn_bwd.attention_fwd_bwd(q, k, v, do, layout=w.layout, causal=w.causal,
                                                  scale=float(np.float32(w.scale)))
    # A gradient that cancels to (nearly) zero in exact arithmetic -- dQ with a
    # single key, where dP - D is 0 -- keeps the fp32 rounding of that
    # difference; its scale is floored at 1e-3 of the problem's largest
    # gradient entry.
    floor = 1e-3 * max(np.max(np.abs(rq)), np.max(np.abs(rk)), np.max(np.abs(rv)), 1e-6)
    for name, g, r in (("dq", grads[0], rq), ("dk", grads[1], rk), ("dv", grads[2], rv)):
        gg = to_bhsd(g, w.layout)
        assert np.all(np.isfinite(gg)), name
        err = np.max(np.abs(gg - r))
        bound = REL_TOL[w.dtype] * max(np.max(np.abs(r)), floor)
        print(f"PARITY {tag} {w.name} {name}: max|err| {err:.3e} bound {bound:.3e}")
        assert err <= bound, (name, err, bound)


CASES = [
    W("bf16", "BHSD", 1, 2, 256, 256, 128, False),
    W("bf16", "BHSD", 1, 2, 256, 256, 128, True),
    W("fp16", "BSND", 1, 2, 200, 333, 64, True),
    W("bf16", "BHSD", 1, 1, 1000, 1000, 128, True),
    W("bf16", "BSND", 1, 2, 384, 1000, 128, False),
    W("bf16", "BHSD", 1, 2, 1000, 384, 128, True),
    W("fp16", "BHSD", 2, 2, 513, 513, 128, False),
    W("bf16", "BHSD", 2, 3, 1, 1, 128, False),
    W("bf16", "BSND", 1, 2, 127, 129, 64, True),
    W("fp16", "BSND", 1, 2, 129, 127, 128, True),
    W("bf16", "BHSD", 1, 2, 700, 700, 128, False, qk_std=3.0),
    W("bf16", "BHSD", 1, 2, 300, 700, 128, True, scale=0.0),
    W("bf16", "BHSD", 1, 2, 300, 700, 128, True, scale=-0.09),
    W("fp16", "BHSD", 1, 1, 2048, 2048, 128, True),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_oracle(w):
    _need_gpu()
    inputs, grads = run(w)
    check(w, inputs, grads)


D64_CASES = [
    W("bf16", "BHSD", 1, 2, 256, 256, 64, False),
    W("fp16", "BHSD", 2, 2, 513, 513, 64, True),
    W("bf16", "BSND", 1, 3, 1000, 700, 64, True),
    W("fp16", "BSND", 1, 2, 300, 1001, 64, False),
    W("bf16", "BHSD", 1, 1, 1, 1, 64, False),
    W("fp16", "BSND", 1, 2, 512, 512, 64, False, scale=0.125),
]


@pytest.mark.parametrize("w", CASES + D64_CASES, ids=lambda w: w.name)
def test_atomic_backward_matches_oracle(w):
    _need_gpu()
    inputs, grads = run(w, deterministic=False)
    check(w, inputs, grads, tag="bwd-atomic")


def test_atomic_backward_reproducible_dk_dv_and_close_dq():
    _need_gpu()
    w = W("bf16", "BHSD", 2, 3, 1500, 1500, 128, True)
    _, g1 = run(w, deterministic=False)
    _, g2 = run(w, deterministic=False)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    dq1, dq2 = g1[0].double(), g2[0].double()
    assert float((dq1 - dq2).abs().max()) <= 2.0 ** -8 * float(dq1.abs().max())
    _, gd = run(w, deterministic=True)
    for a, b in zip(g1, gd):      # both within 4u of the exact gradients, so within 8u of each other
        a, b = a.double(), b.double()
        assert float((a - b).abs().max()) <= 2 * REL_TOL["bf16"] * float(b.abs().max())


@pytest.mark.parametrize("D", [64, 128])
def test_atomic_and_deterministic_agree(D):
    """Both variants are within 4u of the exact gradients, so within 8u of each other; dk, dv of
    the atomic variant are reproducible run to run."""
    _need_gpu()
    w = W("fp16", "BHSD", 2, 2, 900, 900, D, True)
    _, ga = run(w, deterministic=False)
    _, ga2 = run(w, deterministic=False)
    assert torch.equal(ga[1], ga2[1]) and torch.equal(ga[2], ga2[2])
    _, gd = run(w, deterministic=True)
    for a, b in zip(ga, gd):
        a, b = a.double(), b.double()
        assert float((a - b).abs().max()) <= 2 * REL_TOL["fp16"] * float(b.abs().max())


def test_backward_deterministic_and_layouts_agree():
    _need_gpu()
    w = W("bf16", "BHSD", 1, 3, 700, 900, 128, True)
    _, g1 = run(w)
    _, g2 = run(w)
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))
    ws = w.with_(layout="BSND")
    q, k, v = make_qkv(w)
    do = make_dout(w)
    to_bsnd = lambda t: t.permute(0, 2, 1, 3).contiguous().cuda()
    qs, ks, vs, dos = to_bsnd(q), to_bsnd(k), to_bsnd(v), to_bsnd(do)
    o, lse = fa.flash_attention_forward(qs, ks, vs, layout="BSND", causal=True, scale=w.scale)
    dq, dk, dv = fa.flash_attention_backward(qs, ks, vs, o, lse, dos, layout="BSND", causal=True, scale=w.scale)
    fa.check_device_status()
    for a, b in zip(g1, (dq, dk, dv)):
        assert torch.equal(a, b.permute(0, 2, 1, 3))


def test_no_query_rows_gives_zero_dk_dv():
    _need_gpu()
    k = torch.randn(1, 2, 300, 128, device="cuda").to(torch.bfloat16)
    q = torch.zeros(1, 2, 0, 128, device="cuda", dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 0, device="cuda")
    dk = torch.full_like(k, 3.0)
    dv = torch.full_like(k, 3.0)
    fa.flash_attention_backward(q, k, k, q, lse, q, layout="BHSD", causal=True, dk=dk, dv=dv)
    fa.check_device_status()
    assert bool((dk == 0).all()) and bool((dv == 0).all())


@pytest.mark.parametrize("deterministic", [True, False])
def test_full_size_invariants(deterministic):
    """The bf16 BHSD 2x40x8192x128 causal shape: per head, the keys' dK sum to 0
    and the keys' dV sum to the queries' dO sum (the rows of P sum to 1)."""
    _need_gpu()
    w = WORKLOADS["bf16_bhsd_b2_h40_s8192_d128_causal"].with_(B=1, H=8)
    q, k, v = make_qkv(w, device="cuda")
    do = make_dout(w, device="cuda")
    o, lse = fa.flash_attention_forward(q, k, v, layout="BHSD", causal=True, scale=w.scale)
    dq, dk, dv = fa.flash_attention_backward(q, k, v, o, lse, do, layout="BHSD", causal=True, scale=w.scale,
                                             deterministic=deterministic)
    fa.check_device_status()
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t.float()).all())
    dk64, dv64, do64 = dk.double(), dv.double(), do.double()
    # the sums cancel exactly in exact arithmetic; allow 8u of the sum of magnitudes
    u = 2.0 ** -8
    sdk = (dk64.sum(dim=2).abs() / dk64.abs().sum(dim=2)).max().item()
    assert sdk <= 8 * u, sdk
    ddv = ((dv64.sum(dim=2) - do64.sum(dim=2)).abs() / dv64.abs().sum(dim=2)).max().item()
    assert ddv <= 8 * u, ddv
