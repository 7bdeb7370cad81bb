"""GPU parity of the output projection (fa_out_proj) and of attention + projection (fa_fwd_proj).

fa_out_proj is checked element by element against the fp64 oracle on seeded
inputs.  The bound follows from the arithmetic: the 16-bit products are exact
in fp32, the K-term fp32 sum is off by at most gamma_K * sum_k |O W|
(gamma_K = K u / (1 - K u), u = 2^-24), and the result is rounded to nearest
in the output type (half an ulp: 2^-9 relative for bf16, 2^-12 for fp16 in
the normal range, 2^-25 absolute below it).  A missing k-block or a wrong
head or feature index is far outside it.  fa_fwd_proj is checked by
properties: its o is bitwise the attention kernel's output (within the
attention bounds of the oracle) and its y is bitwise fa_out_proj of that o.
"""
import math

import numpy as np
import pytest
import torch

import attention_forward_19_b200 as fa
from oracle.proj import out_proj

pytestmark = pytest.mark.gpu

HALF_ULP = {torch.bfloat16: 2.0 ** -9, torch.float16: 2.0 ** -12}


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _inputs(layout, dtype, B, S, H, D, E, seed):
    g = torch.Generator().manual_seed(seed)
    o = torch.randn(B, S, H, D, generator=g)
    if layout == "BHSD":
        o = o.permute(0, 2, 1, 3).contiguous()
    w = torch.randn(E, H * D, generator=g) / math.sqrt(H * D)
    return o.to(dtype), w.to(dtype)


def _check(y_gpu, o, w, layout, dtype, tokens=None):
    """Bound check of y_gpu [B, S, E] against the oracle, on all tokens or on (b, s) pairs."""
    y_ref = out_proj(o, w, layout)
    oa = o.double()
    if layout == "BHSD":
        oa = oa.permute(0, 2, 1, 3)
    B, S, H, D = oa.shape
    absum = oa.reshape(B, S, H * D).abs().numpy() @ w.double().abs().numpy().T
    got = y_gpu.double().cpu().numpy()
    if tokens is not None:
        bi, si = tokens
        y_ref, absum, got = y_ref[bi, si], absum[bi, si], got[bi, si]
    K = H * D
    gamma = K * 2.0 ** -24 / (1 - K * 2.0 ** -24)
    bound = 2 * HALF_ULP[dtype] * np.abs(y_ref) + 1.01 * gamma * absum + 2.0 ** -25
    err = np.abs(got - y_ref)
    assert np.all(err <= bound), (float(np.max(err - bound)), float(np.max(err)))
    return float(np.max(err))


CASES = [
    # layout, dtype, B, S, H, D, E
    ("BSND", torch.bfloat16, 1, 1000, 4, 128, 320),    # ragged token tile, E not a multiple of 256
    ("BHSD", torch.bfloat16, 2, 129, 3, 64, 96),
    ("BHSD", torch.float16, 1, 256, 8, 128, 1024),
    ("BSND", torch.float16, 2, 7, 2, 64, 32),
    ("BSND", torch.bfloat16, 1, 1, 1, 128, 64),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}_{str(c[1])[6:]}_B{c[2]}_S{c[3]}_H{c[4]}_D{c[5]}_E{c[6]}")
def test_out_proj_matches_oracle(case):
    _need_gpu()
    layout, dtype, B, S, H, D, E = case
    o, w = _inputs(layout, dtype, B, S, H, D, E, seed=S + E)
    y = fa.out_projection(o.cuda(), w.cuda(), layout=layout)
    fa.check_device_status()
    err = _check(y, o, w, layout, dtype)
    print(f"PARITY out_proj {layout} {dtype} B{B} S{S} H{H} D{D} E{E}: max|dY| {err:.3e}")


@pytest.mark.parametrize("layout", ["BSND", "BHSD"])
def test_identity_weight_copies_the_heads(layout):
    _need_gpu()
    B, S, H, D = 1, 300, 4, 64
    o, _ = _inputs(layout, torch.bfloat16, B, S, H, D, 32, seed=3)
    w = torch.eye(H * D, dtype=torch.bfloat16)
    y = fa.out_projection(o.cuda(), w.cuda(), layout=layout).cpu()
    o_bsnd = o if layout == "BSND" else o.permute(0, 2, 1, 3)
    assert torch.equal(y, o_bsnd.reshape(B, S, H * D))


def test_out_proj_full_size_sampled_tokens():
    # the projection of the bf16 B=2 H=40 S=8192 D=128 attention output (E = H * D = 5120), BHSD
    _need_gpu()
    B, S, H, D, E = 2, 8192, 40, 128, 5120
    o, w = _inputs("BHSD", torch.bfloat16, B, S, H, D, E, seed=44)
    y = fa.out_projection(o.cuda(), w.cuda(), layout="BHSD")
    fa.check_device_status()
    rng = np.random.default_rng(0)
    si = np.concatenate([[0, 127, 128, S - 1], rng.integers(0, S, 28)])
    bi = np.concatenate([[0, 1, 0, 1], rng.integers(0, B, 28)])
    o_s = o[bi, :, si, :].unsqueeze(1).contiguous()          # [n, 1, H, D] BSND of the sampled tokens
    y_s = y[torch.as_tensor(bi), torch.as_tensor(si)].unsqueeze(1)
    err = _check(y_s, o_s, w, "BSND", torch.bfloat16)
    print(f"PARITY out_proj BHSD bf16 B2 S8192 H40 D128 E5120 (sampled {len(si)} tokens): max|dY| {err:.3e}")


@pytest.mark.parametrize("layout,causal,dtype,D", [("BSND", True, torch.bfloat16, 128),
                                                  ("BHSD", False, torch.bfloat16, 128),
                                                  ("BHSD", True, torch.float16, 64)])
def test_fwd_proj_is_attention_then_projection(orc, layout, causal, dtype, D):
    _need_gpu()
    B, S, H, E = 1, 777, 4, 384
    g = torch.Generator().manual_seed(17)
    shape = (B, S, H, D) if layout == "BSND" else (B, H, S, D)
    q, k, v = (torch.randn(shape, generator=g).to(dtype) for _ in range(3))
    w = (torch.randn(E, H * D, generator=g) / math.sqrt(H * D)).to(dtype)
    qd, kd, vd, wd = q.cuda(), k.cuda(), v.cuda(), w.cuda()
    y, o, lse = fa.flash_attention_forward_proj(qd, kd, vd, wd, layout=layout, causal=causal)
    o2, lse2 = fa.flash_attention_forward(qd, kd, vd, layout=layout, causal=causal)
    y2 = fa.out_projection(o2, wd, layout=layout)
    fa.check_device_status()
    assert torch.equal(o, o2) and torch.equal(lse, lse2) and torch.equal(y, y2)
    o_ref, l_ref = orc.fwd(q, k, v, layout=layout, causal=causal, scale=1.0 / math.sqrt(D))
    o_got = (o.permute(0, 2, 1, 3) if layout == "BSND" else o).double().cpu().numpy()
    assert float(np.max(np.abs(o_got - o_ref))) <= (2e-2 if dtype == torch.bfloat16 else 1e-2)
    assert float(np.max(np.abs(lse.double().cpu().numpy() - l_ref))) <= 1e-3
