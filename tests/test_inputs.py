"""CPU tests of the seeded input generator (fa_inputs): the plain recipe and
the structured lead values that the forced-branch GPU tests rely on."""
import math

import torch

from fa_inputs import DTYPES, Workload, make_qkv

LOG2E = 1.4426950408889634


def test_plain_recipe_is_three_seeded_normal_draws():
    w = Workload("t", "bf16", "BSND", 1, 2, 300, 500, 64, False, 0.1, qk_std=2.0, v_std=0.5, seed=5)
    q, k, v = make_qkv(w)
    g = torch.Generator().manual_seed(5)
    q2 = (torch.randn(w.q_shape(), generator=g) * 2.0).to(torch.bfloat16)
    k2 = (torch.randn(w.kv_shape(), generator=g) * 2.0).to(torch.bfloat16)
    v2 = (torch.randn(w.kv_shape(), generator=g) * 0.5).to(torch.bfloat16)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)


def test_lead_values_per_row_and_per_key_block_in_both_layouts():
    for layout in ("BSND", "BHSD"):
        w = Workload("t", "fp16", layout, 2, 3, 7, 300, 64, False, 0.1, q_lead=(1.0, 2.0, 3.0),
                     k_lead=(10.0, 20.0), seed=9)
        q, k, v = make_qkv(w)
        assert q.dtype == DTYPES["fp16"]
        qb = q.permute(0, 2, 1, 3) if layout == "BSND" else q
        kb = k.permute(0, 2, 1, 3) if layout == "BSND" else k
        for b in range(2):
            for h in range(3):
                assert qb[b, h, :, 0].tolist() == [1.0, 2.0, 3.0, 1.0, 2.0, 3.0, 1.0]
                assert kb[b, h, :, 0].tolist() == [10.0] * 128 + [20.0] * 128 + [10.0] * 44
        # the other elements keep the drawn values
        plain = make_qkv(w.with_(q_lead=(), k_lead=()))
        assert torch.equal(q[..., 1:], plain[0][..., 1:]) and torch.equal(k[..., 1:], plain[1][..., 1:])
        assert torch.equal(v, plain[2])


def test_ramp_lifts_lead_rows_by_the_intended_log2_step():
    """A query lead a and key leads 40 t / (scale log2e a) give a lead row a logit step of ~40 log2 units per tile."""
    D = 128
    scale = 1.0 / math.sqrt(D)
    a = 16.0
    c = scale * LOG2E * a
    w = Workload("t", "bf16", "BHSD", 1, 1, 4, 512, D, False, scale, q_lead=(a,),
                 k_lead=tuple(40.0 * t / c for t in range(4)))
    q, k, _ = make_qkv(w)
    for t in range(1, 4):
        step = float(q[0, 0, 0, 0].double() * (k[0, 0, 128 * t, 0].double() - k[0, 0, 128 * (t - 1), 0].double()))
        assert 39.0 < step * scale * LOG2E < 41.0
