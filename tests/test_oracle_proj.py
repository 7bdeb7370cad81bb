"""Pins of the oracle's output projection (oracle/proj.py).

Independent of the numpy matmul it uses: identity and selector weights (closed
forms), a pure-Python loop over a tiny case, and, for the composition with
attention, a one-key closed form.
"""

import numpy as np
import pytest
import torch

from oracle.proj import attention_out_proj, out_proj


@pytest.mark.parametrize("layout", ["BSND", "BHSD"])
def test_identity_weight_returns_the_heads_concatenated(layout):
    g = torch.Generator().manual_seed(1)
    B, S, H, D = 2, 5, 3, 4
    o_bsnd = torch.randn(B, S, H, D, generator=g, dtype=torch.float64)
    o = o_bsnd if layout == "BSND" else o_bsnd.permute(0, 2, 1, 3).contiguous()
    y = out_proj(o, torch.eye(H * D, dtype=torch.float64), layout)
    for b in range(B):
        for s in range(S):
            for h in range(H):
                assert np.array_equal(y[b, s, h * D:(h + 1) * D], o_bsnd[b, s, h].numpy())


def test_selector_rows_pick_one_head_element():
    g = torch.Generator().manual_seed(2)
    B, S, H, D = 1, 4, 2, 8
    o = torch.randn(B, S, H, D, generator=g, dtype=torch.float64)
    picks = [(1, 3), (0, 0), (1, 7)]                 # (head, dim) per output feature
    w = torch.zeros(len(picks), H * D, dtype=torch.float64)
    for n, (h, d) in enumerate(picks):
        w[n, h * D + d] = 1.0
    y = out_proj(o, w)
    for n, (h, d) in enumerate(picks):
        assert np.array_equal(y[0, :, n], o[0, :, h, d].numpy())


def test_tiny_case_against_plain_loops():
    g = torch.Generator().manual_seed(3)
    B, S, H, D, E = 1, 3, 2, 2, 3
    o = torch.randn(B, S, H, D, generator=g, dtype=torch.float64)
    w = torch.randn(E, H * D, generator=g, dtype=torch.float64)
    y = out_proj(o, w)
    for s in range(S):
        for n in range(E):
            acc = 0.0
            for h in range(H):
                for d in range(D):
                    acc += float(o[0, s, h, d]) * float(w[n, h * D + d])
            assert abs(y[0, s, n] - acc) < 1e-13


def test_bf16_inputs_are_decoded_exactly():
    o = torch.tensor([[[[1.0078125, -3.0]]]], dtype=torch.bfloat16)   # exactly representable
    w = torch.tensor([[2.0, 0.5]], dtype=torch.bfloat16)
    assert out_proj(o, w)[0, 0, 0] == 1.0078125 * 2.0 - 1.5


def test_composition_single_key_closed_form():
    # one key: attention returns V[0] for every query, so Y = V[0] W^T per token
    g = torch.Generator().manual_seed(4)
    B, H, S, D, E = 1, 2, 3, 8, 5
    q = torch.randn(B, S, H, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, 1, H, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, 1, H, D, generator=g, dtype=torch.float64)
    w = torch.randn(E, H * D, generator=g, dtype=torch.float64)
    y, o, lse = attention_out_proj(q, k, v, w, layout="BSND", scale=0.5)
    expect = (v[0, 0].reshape(H * D) @ w.T).numpy()
    for s in range(S):
        assert np.max(np.abs(y[0, s] - expect)) < 1e-12
    assert np.max(np.abs(lse[0, :, :] - 0.5 * np.einsum("shd,hd->hs", q[0].numpy(), k[0, 0].numpy()))) < 1e-12
