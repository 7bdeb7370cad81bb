"""GPU parity on inputs built to drive the online softmax's rare branches.

The kernel keeps a per-row reference max m and moves it only when a key
tile's max exceeds it by more than tau = 15 log2 units (bf16: the moved
reference sits 8 above the tile max).  The exponentials of a tile are first
taken against the current m; a weight above 2^15 rejects that pass, and the
warp recomputes the tile against the exact max and rescales its O rows.  With
N(0, 1) inputs the first tile almost always sets a max that no later tile
beats by tau, so both branches would run only by chance.  Here the inputs set
element 0 of every query row and of every 128-key block (the generator's
q_lead / k_lead) so that the logits of chosen rows jump from tile to tile:

* "ramp": each key tile lifts the lead rows' logits by 40 log2 units (more
  than tau plus the bf16 headroom plus the noise), so every tile after the
  first rejects the speculative pass and rescales O; other rows in the same
  warps fall (-40 per tile), stay flat, or rise by 10 or 20 per tile, so a
  warp mixes rows that move with rows that do not.
* "sawtooth": with little noise, the tile offsets alternate between just
  under the acceptance bound (weights close to 2^15, in fp16 too), just over
  it, and deep falls.

Each case is compared element by element with the fp64 oracle.  The same
call with the library's branch counters on (fa_fwd_opts, branch_counts) must
give bit-identical output, and its counters must show that the branches ran.
The same library with threshold 0 and headroom 0 (the reference max moves at
every new maximum: the recurrence of page "FlashAttention: long-text
inference without running out of memory", section "tiling + online
normalisation", taken literally) is checked against the oracle on the same
inputs, on the small parity shapes and on sampled rows of the full-size
workloads.
"""
import math

import pytest
import torch

import attention_forward_19_b200 as fa
from fa_inputs import WORKLOADS, Workload, make_qkv, sample_rows
from test_parity_gpu import SMALL, compare_full, compare_rows

pytestmark = pytest.mark.gpu

LOG2E = 1.4426950408889634
TAU = 15.0                      # the product build's threshold (log2 units)
HEADROOM = {"fp16": 0.0, "bf16": 8.0}
LEAD_Q = 16.0                   # query lead value (exact in both dtypes)


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def ramp_case(dtype, layout, causal, D, Sq, Sk, seed):
    """Lead rows rise by 40 log2 units per key tile; the rest fall, stay flat or rise by 10 or 20."""
    scale = 1.0 / math.sqrt(D)
    c = scale * LOG2E * LEAD_Q                    # log2 units per unit of k_lead for a lead row
    tiles = (Sk + 127) // 128
    k_lead = tuple(40.0 * t / c for t in range(tiles))
    q_lead = (LEAD_Q, -LEAD_Q, 0.0, LEAD_Q / 2, LEAD_Q / 4, LEAD_Q)
    name = f"ramp_{dtype}_{layout}_{'c' if causal else 'n'}_d{D}_q{Sq}_k{Sk}"
    return Workload(name, dtype, layout, 1, 2, Sq, Sk, D, causal, scale, seed=seed, q_lead=q_lead, k_lead=k_lead)


def sawtooth_case(dtype, layout, causal, D, Sq, Sk, seed):
    """Tile offsets of the lead rows around the acceptance bound R = tau + headroom (log2 units)."""
    scale = 1.0 / math.sqrt(D)
    c = scale * LOG2E * LEAD_Q
    R = TAU + HEADROOM[dtype]
    offs = [0.0, R - 0.7, R - 1.0, -2 * R, R + 1.0, 2 * R + 0.5, 2 * R + 1.5, -R, 3 * R + 2.5, 3 * R + 2.0,
            4 * R + 3.5, 4 * R + 3.0, 4 * R + 2.9, 2 * R, 5 * R + 4.2, 5 * R + 4.0]
    tiles = (Sk + 127) // 128
    k_lead = tuple(offs[t % len(offs)] / c for t in range(tiles))
    q_lead = (LEAD_Q,) * 5 + (LEAD_Q / 2, 0.0, -LEAD_Q)
    name = f"saw_{dtype}_{layout}_{'c' if causal else 'n'}_d{D}_q{Sq}_k{Sk}"
    return Workload(name, dtype, layout, 1, 2, Sq, Sk, D, causal, scale, qk_std=0.25, seed=seed, q_lead=q_lead,
                    k_lead=k_lead)


CASES = []
for _i, (_dt, _lay, _causal) in enumerate([(d, l, c) for d in ("fp16", "bf16") for l in ("BSND", "BHSD")
                                           for c in (False, True)]):
    _Sq, _Sk = (1500, 1500) if _causal else (700, 2000)
    CASES.append(ramp_case(_dt, _lay, _causal, 128, _Sq, _Sk, seed=300 + _i))
    CASES.append(sawtooth_case(_dt, _lay, _causal, 128, _Sq, _Sk, seed=400 + _i))
CASES.append(ramp_case("bf16", "BHSD", True, 64, 1000, 1000, seed=320))
CASES.append(sawtooth_case("fp16", "BSND", False, 64, 300, 2100, seed=420))


TAU0 = {"rescale_threshold_log2": 0.0, "bf16_headroom_log2": 0.0}


def run(w, q, k, v, **opts):
    o, lse = fa.flash_attention_forward(q.cuda(), k.cuda(), v.cuda(), layout=w.layout, causal=w.causal,
                                        scale=w.scale, softmax_options=opts or None)
    fa.check_device_status()
    return o, lse


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_forced_branches_against_oracle(orc, w):
    _need_gpu()
    q, k, v = make_qkv(w)
    o, lse = run(w, q, k, v)
    compare_full(orc, w, q, k, v, o, lse)

    # the same call with the branch counters on: same bits, and the branches ran
    counts = torch.zeros(4, dtype=torch.int64, device="cuda")
    o2, l2 = run(w, q, k, v, branch_counts=counts)
    total, rejected, rescaled, near = counts.tolist()
    assert torch.equal(o, o2) and torch.equal(lse, l2)
    print(f"BRANCHES {w.name}: warp-tiles {total} rejected {rejected} rescaled {rescaled} near-bound {near}")
    assert total > 0
    if w.name.startswith("ramp"):
        # every warp holds lead rows, and each of their tiles rises by 40 > tau + headroom
        assert rejected >= 0.9 * total and rescaled >= 0.9 * total
    else:
        assert rejected > 0 and rescaled > 0 and near > 0


@pytest.mark.parametrize("w", CASES + SMALL, ids=lambda w: w.name)
def test_tau0_against_oracle(orc, w):
    _need_gpu()
    q, k, v = make_qkv(w)
    o, lse = run(w, q, k, v, **TAU0)
    compare_full(orc, w, q, k, v, o, lse)


@pytest.mark.parametrize("name", [n for n in WORKLOADS if n != "fp16_bsnd_b1_h2_s512_d64"])
def test_tau0_full_size_sampled_rows(orc, name):
    _need_gpu()
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    o, lse = run(w, q, k, v, **TAU0)
    rows = sample_rows(w, per_head_first=16, per_head_last=16, stride=509, max_rows=3000)
    compare_rows(orc, w, q, k, v, o, lse, rows)


def test_tau0_small_workload(orc):
    _need_gpu()
    w = WORKLOADS["fp16_bsnd_b1_h2_s512_d64"]
    q, k, v = make_qkv(w)
    o, lse = run(w, q, k, v, **TAU0)
    compare_full(orc, w, q, k, v, o, lse)
