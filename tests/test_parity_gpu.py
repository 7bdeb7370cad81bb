"""GPU parity: the CUDA kernel (through the C ABI) against the fp64 oracle.

Tolerances are the ones the target states: max |O_gpu - O_oracle| <= 1e-2
(fp16) / 2e-2 (bf16), and max |LSE_gpu - LSE_oracle| <= 1e-3.  Small shapes
are compared element by element; the five full-size workloads are compared
on a stratified sample of rows of every head, in the launch configuration the
benchmark times.
"""
import math

import numpy as np
import pytest
import torch

import attention_forward_19_b200 as fa
from fa_inputs import WORKLOADS, Workload, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

O_TOL = {"fp16": 1e-2, "bf16": 2e-2}
LSE_TOL = 1e-3


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_gpu(w: Workload, q, k, v, scale=None):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = fa.flash_attention_forward(qd, kd, vd, layout=w.layout, causal=w.causal,
                                        scale=w.scale if scale is None else scale)
    fa.check_device_status()
    return o, lse


def to_bhsd(x, layout):
    return x.permute(0, 2, 1, 3) if layout == "BSND" else x


def compare_full(orc, w, q, k, v, o, lse, scale=None):
    scale = w.scale if scale is None else scale
    o_ref, lse_ref = orc.fwd(q, k, v, layout=w.layout, causal=w.causal, scale=float(np.float32(scale)))
    o_gpu = to_bhsd(o.cpu(), w.layout).to(torch.float64).numpy()
    lse_gpu = lse.cpu().to(torch.float64).numpy()
    eo = np.max(np.abs(o_gpu - o_ref))
    el = np.max(np.abs(lse_gpu - lse_ref))
    print(f"PARITY {w.name}: max|dO| {eo:.3e} max|dLSE| {el:.3e} ({o_gpu.shape[0] if o_gpu.ndim == 2 else 'all'} rows)")
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(lse_gpu))
    assert eo <= O_TOL[w.dtype], f"{w.name}: max |dO| = {eo}"
    assert el <= LSE_TOL, f"{w.name}: max |dLSE| = {el}"
    return eo, el


def compare_rows(orc, w, q, k, v, o, lse, rows):
    rows = np.asarray(rows, dtype=np.int64)
    o_ref, lse_ref = orc.fwd(q, k, v, layout=w.layout, causal=w.causal, scale=float(np.float32(w.scale)),
                             rows=rows)
    ob = to_bhsd(o, w.layout).reshape(w.B * w.H * w.Sq, w.D)
    idx = torch.from_numpy(rows).to(o.device)
    o_gpu = ob.index_select(0, idx).cpu().to(torch.float64).numpy()
    lse_gpu = lse.reshape(-1).index_select(0, idx).cpu().to(torch.float64).numpy()
    eo = np.max(np.abs(o_gpu - o_ref))
    el = np.max(np.abs(lse_gpu - lse_ref))
    print(f"PARITY {w.name}: max|dO| {eo:.3e} max|dLSE| {el:.3e} ({o_gpu.shape[0] if o_gpu.ndim == 2 else 'all'} rows)")
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(lse_gpu))
    assert eo <= O_TOL[w.dtype], f"{w.name}: max |dO| = {eo} over {len(rows)} rows"
    assert el <= LSE_TOL, f"{w.name}: max |dLSE| = {el} over {len(rows)} rows"
    return eo, el


def W(dtype, layout, B, H, Sq, Sk, D, causal, scale=None, qk_std=1.0, seed=7):
    return Workload(f"{dtype}_{layout}_b{B}_h{H}_q{Sq}_k{Sk}_d{D}_{'c' if causal else 'n'}", dtype, layout,
                    B, H, Sq, Sk, D, causal, 1.0 / math.sqrt(D) if scale is None else scale,
                    qk_std=qk_std, seed=seed)


SMALL = [
    W("bf16", "BHSD", 1, 1, 128, 128, 128, False),
    W("bf16", "BHSD", 1, 2, 256, 256, 128, True),
    W("fp16", "BHSD", 1, 2, 256, 256, 128, False),
    W("bf16", "BHSD", 2, 3, 1, 1, 128, False),
    W("bf16", "BHSD", 1, 2, 7, 7, 128, True),
    W("fp16", "BSND", 1, 2, 127, 127, 64, False),
    W("fp16", "BSND", 1, 2, 129, 129, 64, True),
    W("bf16", "BSND", 1, 3, 1000, 1000, 128, True),
    W("bf16", "BHSD", 1, 2, 384, 1000, 128, False),
    W("bf16", "BHSD", 1, 2, 384, 1000, 128, True),
    W("bf16", "BHSD", 1, 2, 1000, 384, 128, True),
    W("fp16", "BHSD", 1, 2, 1000, 384, 128, False),
    W("bf16", "BHSD", 2, 2, 513, 257, 64, True),
    W("bf16", "BHSD", 1, 2, 640, 640, 64, False),
    W("fp16", "BHSD", 1, 1, 2048, 2048, 128, True),
    W("bf16", "BSND", 1, 2, 300, 16001, 128, False),
    W("bf16", "BSND", 1, 4, 1500, 1500, 128, False, qk_std=3.0),
    W("fp16", "BSND", 3, 5, 200, 333, 128, True),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_shapes_elementwise(orc, w):
    _need_gpu()
    q, k, v = make_qkv(w)
    o, lse = run_gpu(w, q, k, v)
    compare_full(orc, w, q, k, v, o, lse)


@pytest.mark.parametrize("scale", [0.0, -0.09, 0.5])
def test_scale_values(orc, scale):
    """scale is used as given: zero (uniform weights), negative, large."""
    _need_gpu()
    w = W("bf16", "BHSD", 1, 2, 300, 700, 128, True, scale=scale)
    q, k, v = make_qkv(w)
    o, lse = run_gpu(w, q, k, v)
    compare_full(orc, w, q, k, v, o, lse)


def test_workload_small_full_compare(orc):
    """The fp16 BSND 1x2x512x64 workload, every element."""
    _need_gpu()
    w = WORKLOADS["fp16_bsnd_b1_h2_s512_d64"]
    q, k, v = make_qkv(w)
    o, lse = run_gpu(w, q, k, v)
    assert tuple(o.shape) == (1, 512, 2, 64)
    compare_full(orc, w, q, k, v, o, lse)


@pytest.mark.parametrize("name", [n for n in WORKLOADS if n != "fp16_bsnd_b1_h2_s512_d64"])
def test_workload_full_size_sampled_rows(orc, name):
    """Full-size workloads in the benchmark's launch configuration, checked on
    the first and last 32 rows and every 257th row of every head."""
    _need_gpu()
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    o, lse = run_gpu(w, q, k, v)
    rows = sample_rows(w, per_head_first=32, per_head_last=32, stride=257, max_rows=6000)
    compare_rows(orc, w, q, k, v, o, lse, rows)


def test_full_size_scale_zero_is_running_mean():
    """scale = 0 at a long causal size: O[i] = mean(V[0..i]) and LSE[i] = ln(i + 1) exactly in math."""
    _need_gpu()
    w = W("bf16", "BHSD", 1, 2, 8192, 8192, 128, True, scale=0.0)
    q, k, v = make_qkv(w)
    o, lse = run_gpu(w, q, k, v)
    vs = v.to(torch.float64)
    ref = torch.cumsum(vs, dim=2) / torch.arange(1, w.Sk + 1, dtype=torch.float64).view(1, 1, -1, 1)
    assert (o.cpu().to(torch.float64) - ref).abs().max().item() <= O_TOL["bf16"]
    lref = torch.log(torch.arange(1, w.Sq + 1, dtype=torch.float64)).view(1, 1, -1)
    assert (lse.cpu().to(torch.float64) - lref).abs().max().item() <= LSE_TOL


def test_deterministic_bitwise():
    _need_gpu()
    w = WORKLOADS["bf16_bhsd_b2_h40_s8192_d128_causal"]
    q, k, v = make_qkv(w, device="cuda")
    o1, l1 = fa.flash_attention_forward(q, k, v, layout=w.layout, causal=True, scale=w.scale)
    o2, l2 = fa.flash_attention_forward(q, k, v, layout=w.layout, causal=True, scale=w.scale)
    fa.check_device_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_layouts_agree_bitwise(causal):
    """The same data in BSND and BHSD gives bit-identical results."""
    _need_gpu()
    w = W("bf16", "BHSD", 2, 3, 777, 901, 128, causal)
    q, k, v = make_qkv(w, device="cuda")
    o1, l1 = fa.flash_attention_forward(q, k, v, layout="BHSD", causal=causal, scale=w.scale)
    t = lambda x: x.transpose(1, 2).contiguous()
    o2, l2 = fa.flash_attention_forward(t(q), t(k), t(v), layout="BSND", causal=causal, scale=w.scale)
    fa.check_device_status()
    assert torch.equal(o1, o2.transpose(1, 2)) and torch.equal(l1, l2)


def test_causal_future_keys_do_not_matter():
    _need_gpu()
    w = W("fp16", "BHSD", 1, 2, 700, 700, 128, True)
    q, k, v = make_qkv(w, device="cuda")
    o1, l1 = fa.flash_attention_forward(q, k, v, layout="BHSD", causal=True, scale=w.scale)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 400:] = 5.0
    v2[:, :, 400:] = -7.0
    o2, l2 = fa.flash_attention_forward(q, k2, v2, layout="BHSD", causal=True, scale=w.scale)
    fa.check_device_status()
    assert torch.equal(o1[:, :, :400], o2[:, :, :400]) and torch.equal(l1[:, :, :400], l2[:, :, :400])


def test_constant_v_gives_constant_o():
    _need_gpu()
    w = W("bf16", "BSND", 1, 4, 1000, 1000, 64, False, qk_std=3.0)
    q, k, _ = make_qkv(w, device="cuda")
    v = torch.full_like(k, 0.75)
    o, _ = fa.flash_attention_forward(q, k, v, layout="BSND", causal=False, scale=w.scale)
    fa.check_device_status()
    assert (o.float() - 0.75).abs().max().item() <= 4e-3


def test_host_pointers_rejected():
    _need_gpu()
    q = torch.zeros(1, 128, 1, 64, dtype=torch.float16)
    dev = torch.zeros(1, 128, 1, 64, dtype=torch.float16, device="cuda")
    lse = torch.zeros(1, 1, 128, dtype=torch.float32, device="cuda")
    st = fa.fa_fwd(q.data_ptr(), dev.data_ptr(), dev.data_ptr(), torch.empty_like(dev).data_ptr(),
                   lse.data_ptr(), 1, 1, 128, 128, 64, fa.FA_BSND, 0, 0.125, fa.FA_FP16, None)
    assert st == fa.FA_ERR_NOT_DEVICE_POINTER
    with pytest.raises(fa.FaError):
        fa.flash_attention_forward(q, q, q, layout="BSND")


def test_stream_is_respected():
    _need_gpu()
    w = W("bf16", "BHSD", 1, 8, 1024, 1024, 128, True)
    q, k, v = make_qkv(w, device="cuda")
    ref, _ = fa.flash_attention_forward(q, k, v, layout="BHSD", causal=True, scale=w.scale)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        o, _ = fa.flash_attention_forward(q, k, v, layout="BHSD", causal=True, scale=w.scale)
    torch.cuda.current_stream().wait_stream(s)
    fa.check_device_status(s)
    assert torch.equal(o, ref)


SCHEDULE_CASES = [
    W("bf16", "BHSD", 2, 40, 8192, 8192, 128, True),
    W("bf16", "BSND", 1, 3, 1000, 1000, 128, True),
    W("fp16", "BHSD", 2, 5, 700, 1900, 64, False),
    W("bf16", "BHSD", 1, 8, 65536, 65536, 128, True),
]


@pytest.mark.parametrize("w", SCHEDULE_CASES, ids=lambda w: w.name)
def test_static_and_dynamic_schedules_agree_bitwise(w):
    """fa_fwd (static round-robin) and fa_fwd_ws (work counter) compute every
    unit the same way, so their outputs are bit-identical."""
    _need_gpu()
    q, k, v = make_qkv(w, device="cuda")
    o1, l1 = fa.flash_attention_forward(q, k, v, layout=w.layout, causal=w.causal, scale=w.scale, schedule="static")
    o2, l2 = fa.flash_attention_forward(q, k, v, layout=w.layout, causal=w.causal, scale=w.scale, schedule="dynamic")
    ws = torch.full((fa.fa_fwd_workspace_size(),), 255, dtype=torch.uint8, device="cuda")   # stale contents
    o3, l3 = fa.flash_attention_forward(q, k, v, layout=w.layout, causal=w.causal, scale=w.scale, workspace=ws)
    o4, l4 = fa.flash_attention_forward(q, k, v, layout=w.layout, causal=w.causal, scale=w.scale, workspace=ws)
    fa.check_device_status()
    for o, l in ((o2, l2), (o3, l3), (o4, l4)):
        assert torch.equal(o1, o) and torch.equal(l1, l)


def test_workspace_on_host_rejected():
    _need_gpu()
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    host_ws = torch.zeros(fa.fa_fwd_workspace_size(), dtype=torch.uint8)
    with pytest.raises(fa.FaError) as e:
        fa.flash_attention_forward(q, q, q, layout="BHSD", workspace=host_ws)
    assert e.value.status == fa.FA_ERR_NOT_DEVICE_POINTER
