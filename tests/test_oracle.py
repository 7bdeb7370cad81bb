"""CPU tests of the fp64 oracle: its pins, its decoders, the online-softmax
recurrence against it, and planted mistakes that the pins must catch."""
import numpy as np
import pytest
import torch

import oracle_pins
from oracle import attn
from oracle.online_softmax import online_attention_row, two_pass_row


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, pin):
    pin(orc)


def test_fp16_decoder_is_exact(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.decode_fp16(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decoder_is_exact(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.decode_bf16(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def _random_blocks(rng, n):
    sizes = []
    left = n
    while left:
        s = int(rng.integers(1, min(left, 9) + 1))
        sizes.append(s)
        left -= s
    return sizes


def test_online_recurrence_matches_two_pass(orc):
    """The block-by-block recurrence (running max m, running exp-sum l, rescaled
    output) reproduces the two-pass softmax and the oracle on brute-force inputs."""
    rng = np.random.default_rng(5)
    for trial in range(200):
        Sk = int(rng.integers(1, 65))
        D = int(rng.integers(1, 9))
        std = float(rng.choice([0.1, 1.0, 10.0, 50.0]))
        q = torch.from_numpy(rng.standard_normal((1, 1, 1, D)) * std)
        k = torch.from_numpy(rng.standard_normal((1, 1, Sk, D)) * std)
        v = torch.from_numpy(rng.standard_normal((1, 1, Sk, D)))
        scale = float(rng.uniform(-1, 1))
        scores = scale * (k[0, 0].numpy() @ q[0, 0, 0].numpy())
        blocks = [1] * Sk if trial % 7 == 0 else _random_blocks(rng, Sk)
        o_on, lse_on = online_attention_row(scores, v[0, 0].numpy(), blocks)
        o_tp, lse_tp = two_pass_row(scores, v[0, 0].numpy())
        o_or, lse_or = orc.fwd(q, k, v, layout="BHSD", causal=False, scale=scale)
        assert np.max(np.abs(o_on - o_tp)) < 1e-12
        assert abs(lse_on - lse_tp) < 1e-12 * max(1.0, abs(lse_tp))
        assert np.max(np.abs(o_on - o_or[0, 0, 0])) < 1e-12
        assert abs(lse_on - lse_or[0, 0, 0]) < 1e-12 * max(1.0, abs(lse_tp))


def test_oracle_rejects_bad_arguments(orc):
    q = torch.zeros(1, 1, 4, 8, dtype=torch.float64)
    with pytest.raises(RuntimeError):
        orc.fwd(q, q, q, layout="BHSD", rows=np.array([4]))   # row id out of range
    with pytest.raises(RuntimeError):
        orc.fwd(q, q, q, layout=7)


@pytest.mark.parametrize("plant", [1, 2, 3, 4, 5, 6, 7, 8])
def test_planted_mistake_is_caught(plant, tmp_path):
    """A deliberately wrong oracle build (wrong operand, off-by-one mask, scale
    twice, wrong V row, flipped exponent, wrong layout stride, no normalisation,
    max dropped from the LSE) fails at least one pin."""
    bad = attn.build_planted(plant, str(tmp_path))
    assert bad.plant == plant
    failures = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(bad)
        except (AssertionError, RuntimeError):
            failures.append(pin.__name__)
    assert failures, f"planted mistake {plant} passed every pin"
