"""CPU tests of the C ABI: the library loads, exports every function the header
declares, and rejects bad arguments before touching the GPU.

Only argument checks that return before the first CUDA call are exercised
here (fake, never-dereferenced pointer values); everything that needs a
device is in the gpu-marked tests.
"""
import ctypes
import os
import re

import pytest

import attention_forward_19_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_fwd.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return fa.load_library()


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names, "no declarations found in the header"
    for name in names:
        assert hasattr(lib, name), f"{name} declared in fa_fwd.h but not exported"
    assert sorted(fa.EXPORTED_SYMBOLS) == names


def test_exported_symbols_are_plain_c(lib):
    # nm-free check: the C names resolve through dlsym, i.e. they are not mangled
    for name in declared_functions():
        ctypes.cast(getattr(lib, name), ctypes.c_void_p)


def test_version_and_strings(lib):
    assert fa.fa_version() == 10000
    for code, name in [(0, "FA_OK"), (1, "FA_ERR_INVALID_ARG"), (2, "FA_ERR_UNSUPPORTED"),
                       (3, "FA_ERR_NOT_DEVICE_POINTER"), (4, "FA_ERR_MISALIGNED"), (5, "FA_ERR_ALIAS"),
                       (6, "FA_ERR_CUDA"), (7, "FA_ERR_TIMEOUT")]:
        assert fa.fa_status_string(code) == name
    assert fa.fa_status_string(99) == "FA_ERR_UNKNOWN"
    assert fa.fa_last_cuda_error() == 0


def test_query_support(lib):
    for D in (64, 128):
        for dt in (fa.FA_FP16, fa.FA_BF16):
            assert fa.fa_query_support(D, dt) == fa.FA_OK
    for D in (0, 32, 96, 256):
        assert fa.fa_query_support(D, fa.FA_BF16) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_query_support(128, 7) == fa.FA_ERR_UNSUPPORTED


# Fake, 256-byte aligned, far-apart addresses: the checks below return before any use.
Q, K, V, O, L = 0x10000000, 0x20000000, 0x30000000, 0x40000000, 0x50000000
GOOD = dict(B=1, H=2, Sq=512, Sk=512, D=64, layout=fa.FA_BSND, causal=0, scale=0.125, dtype=fa.FA_FP16)


def call(q=Q, k=K, v=V, o=O, lse=L, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd(q, k, v, o, lse, a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["layout"], a["causal"],
                     a["scale"], a["dtype"], None)


@pytest.mark.parametrize("kw", [dict(B=0), dict(H=0), dict(B=-1), dict(Sk=0), dict(Sq=-1), dict(D=0),
                                dict(layout=2), dict(layout=-1), dict(dtype=2),
                                dict(scale=float("nan")), dict(scale=float("inf"))])
def test_invalid_arguments(lib, kw):
    assert call(**kw) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("D", [32, 80, 96, 256])
def test_unsupported_head_dim(lib, D):
    assert call(D=D) == fa.FA_ERR_UNSUPPORTED


def test_oversized_lengths_unsupported(lib):
    assert call(Sq=1 << 31) == fa.FA_ERR_UNSUPPORTED
    assert call(Sk=1 << 31) == fa.FA_ERR_UNSUPPORTED


def test_empty_query_is_a_no_op(lib):
    assert call(Sq=0) == fa.FA_OK
    assert call(Sq=0, q=0, o=0, lse=0) == fa.FA_OK


@pytest.mark.parametrize("which", ["q", "k", "v", "o", "lse"])
def test_null_pointer(lib, which):
    assert call(**{which: 0}) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("which,off", [("q", 8), ("k", 2), ("v", 4), ("o", 8), ("lse", 2)])
def test_misaligned_pointer(lib, which, off):
    base = dict(q=Q, k=K, v=V, o=O, lse=L)[which]
    assert call(**{which: base + off}) == fa.FA_ERR_MISALIGNED


def test_lse_needs_only_4_byte_alignment(lib):
    # passes the alignment and alias checks; on a machine without a GPU it then fails in CUDA
    st = call(lse=L + 4)
    assert st not in (fa.FA_ERR_MISALIGNED, fa.FA_ERR_ALIAS, fa.FA_ERR_INVALID_ARG)


@pytest.mark.parametrize("o,lse", [(Q, L), (Q + 4096, L), (K, L), (V + 64, L), (O, Q), (O, O + 16), (O, V)])
def test_aliasing_outputs_rejected(lib, o, lse):
    assert call(o=o, lse=lse) == fa.FA_ERR_ALIAS


def test_python_wrapper_checks_shapes():
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 16, 2, 64, dtype=torch.float16)
    k = torch.zeros(1, 16, 3, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        fa.flash_attention_forward(q, k, k, layout="BSND")
    with pytest.raises(ValueError, match="head_num"):
        fa.flash_attention_forward(q, q, q, layout="BSND", head_num=8)
    with pytest.raises(TypeError):
        x = torch.zeros(1, 16, 2, 64, dtype=torch.float32)
        fa.flash_attention_forward(x, x, x, layout="BSND")
    with pytest.raises(ValueError, match="contiguous"):
        t = torch.zeros(1, 2, 16, 64, dtype=torch.float16).transpose(1, 2)
        fa.flash_attention_forward(t, t, t, layout="BSND")


WS = 0x60000000


def call_ws(ws=WS, ws_bytes=16, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_ws(a.get("q", Q), a.get("k", K), a.get("v", V), a.get("o", O), a.get("lse", L),
                        a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["layout"], a["causal"], a["scale"],
                        a["dtype"], ws, ws_bytes, None)


def test_workspace_size_is_small_constant(lib):
    assert 4 <= fa.fa_fwd_workspace_size() <= 256
    assert fa.fa_fwd_workspace_size() % 4 == 0


def test_workspace_validation(lib):
    assert call_ws(ws=0) == fa.FA_ERR_INVALID_ARG
    assert call_ws(ws_bytes=fa.fa_fwd_workspace_size() - 1) == fa.FA_ERR_INVALID_ARG
    assert call_ws(ws=WS + 4) == fa.FA_ERR_MISALIGNED
    assert call_ws(ws=Q + 64) == fa.FA_ERR_ALIAS
    assert call_ws(ws=L) == fa.FA_ERR_ALIAS
    assert call_ws(ws=0, Sq=0) == fa.FA_OK
    assert call_ws(D=96) == fa.FA_ERR_UNSUPPORTED


def test_dynamic_schedule_argument_errors_match_static(lib):
    for kw in (dict(B=0), dict(layout=3), dict(dtype=5), dict(scale=float("nan"))):
        assert call_ws(**kw) == call(**kw) == fa.FA_ERR_INVALID_ARG


def call_noalloc(q=Q, k=K, v=V, o=O, lse=L, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_noalloc(q, k, v, o, lse, a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["layout"], a["causal"],
                             a["scale"], a["dtype"], None)


NOALLOC_CASES = [dict(B=0), dict(H=0), dict(Sk=0), dict(Sq=-1), dict(D=0), dict(layout=2), dict(dtype=2),
                 dict(scale=float("nan")), dict(D=96), dict(D=256), dict(Sq=1 << 31), dict(Sk=1 << 31),
                 dict(B=1 << 30, Sq=0), dict(H=1 << 30, Sq=0), dict(Sq=0), dict(Sq=0, q=0, o=0, lse=0),
                 dict(q=0), dict(lse=0), dict(q=Q + 8), dict(o=O + 8), dict(lse=L + 2), dict(o=Q),
                 dict(o=O, lse=O + 16), dict(lse=V + 64)]


@pytest.mark.parametrize("kw", NOALLOC_CASES, ids=lambda kw: ",".join(f"{k}={v}" for k, v in kw.items()))
def test_noalloc_argument_errors_match_fa_fwd(lib, kw):
    """fa_fwd_noalloc answers every call that fails before the device exactly as fa_fwd does,
    in the same order (a size beyond the limits is refused even when Sq = 0)."""
    assert call_noalloc(**kw) == call(**kw)


def test_noalloc_reaches_device_checks(lib):
    # valid arguments: the call gets past the host checks to the device lookup, which fails on a
    # machine without a GPU (FA_ERR_CUDA) or on the fake pointers (FA_ERR_NOT_DEVICE_POINTER / CUDA)
    st = call_noalloc()
    assert st not in (fa.FA_OK, fa.FA_ERR_INVALID_ARG, fa.FA_ERR_MISALIGNED, fa.FA_ERR_ALIAS,
                      fa.FA_ERR_UNSUPPORTED), st
    assert call_noalloc(B=1 << 30, Sq=0) == fa.FA_ERR_UNSUPPORTED


def call_opts(opts=None, ws=None, ws_bytes=0, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_opts(a.get("q", Q), a.get("k", K), a.get("v", V), a.get("o", O), a.get("lse", L),
                          a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["layout"], a["causal"], a["scale"],
                          a["dtype"], opts, ws, ws_bytes, None)


def test_default_softmax_options(lib):
    o = fa.fa_fwd_default_options()
    assert (o.rescale_threshold_log2, o.bf16_headroom_log2, o.branch_counts) == (15.0, 8.0, None)


def test_softmax_options_validation(lib):
    """fa_fwd_opts: the settings' ranges, the counters' alignment and overlap; other arguments as fa_fwd."""
    def opts(t=15.0, h=8.0, counts=None):
        o = fa.FwdOptions()
        o.rescale_threshold_log2, o.bf16_headroom_log2, o.branch_counts = t, h, counts
        return o
    for bad in (opts(t=-1.0), opts(t=15.5), opts(t=float("nan")), opts(h=-0.5), opts(h=17.0),
                opts(h=float("inf"))):
        assert call_opts(bad) == fa.FA_ERR_INVALID_ARG
    assert call_opts(opts(counts=0x61000004)) == fa.FA_ERR_MISALIGNED
    assert call_opts(opts(counts=Q + 64)) == fa.FA_ERR_ALIAS
    assert call_opts(opts(counts=L)) == fa.FA_ERR_ALIAS
    assert call_opts(opts(), ws=WS, ws_bytes=4) == fa.FA_ERR_INVALID_ARG
    assert call_opts(opts(), ws=WS + 4, ws_bytes=16) == fa.FA_ERR_MISALIGNED
    assert call_opts(opts(counts=WS + 8), ws=WS, ws_bytes=16) == fa.FA_ERR_ALIAS
    for kw in (dict(B=0), dict(layout=3), dict(dtype=5), dict(scale=float("nan")), dict(D=96), dict(Sq=0),
               dict(q=0), dict(o=O + 8), dict(o=Q)):
        assert call_opts(None, **kw) == call_opts(opts(t=0.0, h=0.0), **kw) == call(**kw), kw
    # valid settings get past the host checks (the call fails later without a GPU)
    assert call_opts(opts(t=0.0, h=0.0)) not in (fa.FA_OK, fa.FA_ERR_INVALID_ARG, fa.FA_ERR_MISALIGNED,
                                                  fa.FA_ERR_ALIAS)


def call_heads(begin=0, count=2, ws=None, ws_bytes=0, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_heads(a.get("q", Q), a.get("k", K), a.get("v", V), a.get("o", O), a.get("lse", L),
                           a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["layout"], a["causal"], a["scale"],
                           a["dtype"], begin, count, ws, ws_bytes, None)


def test_head_range_validation(lib):
    """fa_fwd_heads: the range must lie in [0, B * H]; other arguments are checked as fa_fwd checks them."""
    for begin, count in ((-1, 1), (0, -1), (0, 3), (2, 1), (3, 0)):
        assert call_heads(begin, count) == fa.FA_ERR_INVALID_ARG, (begin, count)
    for kw in (dict(B=0), dict(layout=3), dict(dtype=5), dict(scale=float("nan")), dict(D=96), dict(Sq=0),
               dict(q=0), dict(o=O + 8), dict(o=Q)):
        assert call_heads(**kw) == call(**kw), kw
    assert call_heads(ws=WS, ws_bytes=4) == fa.FA_ERR_INVALID_ARG
    assert call_heads(ws=WS + 4, ws_bytes=16) == fa.FA_ERR_MISALIGNED
    assert call_heads(ws=Q + 64, ws_bytes=16) == fa.FA_ERR_ALIAS
    # an empty range is a no-op; a valid call gets past the host checks (it fails later without a GPU)
    assert call_heads(1, 0) == fa.FA_OK
    assert call_heads(1, 1) not in (fa.FA_OK, fa.FA_ERR_INVALID_ARG, fa.FA_ERR_MISALIGNED, fa.FA_ERR_ALIAS)


def call_selftest(limit_us=20000, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_selftest_wait_timeout(Q, K, V, O, L, a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["layout"],
                                       a["causal"], a["scale"], a["dtype"], limit_us, None)


def test_selftest_limit_range_and_argument_checks(lib):
    """The wait-timeout self-test takes a limit of 1 ms .. 1 s and validates like fa_fwd."""
    assert call_selftest(limit_us=999) == fa.FA_ERR_INVALID_ARG
    assert call_selftest(limit_us=1000001) == fa.FA_ERR_INVALID_ARG
    for kw in (dict(B=0), dict(layout=3), dict(dtype=5), dict(scale=float("nan"))):
        assert call_selftest(**kw) == call(**kw) == fa.FA_ERR_INVALID_ARG
    assert call_selftest(D=96) == fa.FA_ERR_UNSUPPORTED
    assert call_selftest(Sq=0) == fa.FA_OK


CUQ, CUK = 0x70000000, 0x70001000


def call_varlen(**kw):
    a = dict(q=Q, k=K, v=V, o=O, lse=L, cu_q=CUQ, cu_k=CUK, B=3, H=2, total_q=600, total_k=700, max_q=300,
             max_k=400, D=128, causal=1, scale=0.1, dtype=fa.FA_BF16, ws=None, ws_bytes=0)
    a.update(kw)
    return fa.fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu_q"], a["cu_k"], a["B"], a["H"],
                            a["total_q"], a["total_k"], a["max_q"], a["max_k"], a["D"], a["causal"], a["scale"],
                            a["dtype"], a["ws"], a["ws_bytes"], None)


def test_varlen_host_validation(lib):
    """Checks of the packed entry that return before any device call."""
    for kw in (dict(B=0), dict(H=0), dict(total_q=-1), dict(max_k=-1), dict(dtype=7), dict(scale=float("inf")),
               dict(max_q=601), dict(max_k=701), dict(max_k=0), dict(cu_q=0), dict(cu_k=0), dict(lse=0),
               dict(ws=WS, ws_bytes=4)):
        assert call_varlen(**kw) == fa.FA_ERR_INVALID_ARG, kw
    assert call_varlen(D=96) == fa.FA_ERR_UNSUPPORTED
    assert call_varlen(total_q=0, max_q=0) == fa.FA_OK
    assert call_varlen(max_q=0) == fa.FA_OK
    assert call_varlen(cu_q=CUQ + 2) == fa.FA_ERR_MISALIGNED
    assert call_varlen(q=Q + 8) == fa.FA_ERR_MISALIGNED
    assert call_varlen(ws=WS + 4, ws_bytes=16) == fa.FA_ERR_MISALIGNED
    assert call_varlen(o=CUQ) == fa.FA_ERR_ALIAS
    assert call_varlen(lse=Q + 64) == fa.FA_ERR_ALIAS
    assert call_varlen(ws=CUK, ws_bytes=16) == fa.FA_ERR_ALIAS


DQ, DK, DV, DO_, WSB = 0x71000000, 0x72000000, 0x73000000, 0x74000000, 0x75000000


def call_bwd(**kw):
    a = dict(q=Q, k=K, v=V, o=O, dout=DO_, lse=L, dq=DQ, dk=DK, dv=DV, B=1, H=2, Sq=512, Sk=512, D=128,
             layout=fa.FA_BHSD, causal=1, scale=0.1, dtype=fa.FA_BF16, ws=WSB, ws_bytes=1 << 20)
    a.update(kw)
    return fa.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"], a["B"], a["H"],
                     a["Sq"], a["Sk"], a["D"], a["layout"], a["causal"], a["scale"], a["dtype"], a["ws"],
                     a["ws_bytes"], None)


def test_bwd_workspace_size():
    assert fa.fa_bwd_workspace_size(1, 2, 512) == 2 * 2 * 512 * 4
    assert fa.fa_bwd_workspace_size(1, 2, 513) == 2 * 2 * 640 * 4     # each head padded to whole 128-row tiles
    assert fa.fa_bwd_workspace_size(0, 2, 512) == 0


def test_bwd_host_validation(lib):
    for kw in (dict(B=0), dict(Sk=0), dict(layout=5), dict(dtype=9), dict(scale=float("nan")), dict(q=0),
               dict(lse=0), dict(dq=0), dict(ws=0), dict(ws_bytes=100)):
        assert call_bwd(**kw) == fa.FA_ERR_INVALID_ARG, kw
    assert call_bwd(D=80) == fa.FA_ERR_UNSUPPORTED
    assert call_bwd(dq=DQ + 8) == fa.FA_ERR_MISALIGNED
    assert call_bwd(ws=WSB + 4) == fa.FA_ERR_MISALIGNED
    assert call_bwd(lse=L + 2) == fa.FA_ERR_MISALIGNED
    assert call_bwd(dq=Q) == fa.FA_ERR_ALIAS
    assert call_bwd(dk=DV) == fa.FA_ERR_ALIAS
    assert call_bwd(ws=DO_) == fa.FA_ERR_ALIAS


# fa_lse_merge: fake pointers far apart, sized for B=1, H=2, S=64, D=128
MP, MLP, MA, MLA, MO, MLO = (1 << 40, 2 << 40, 3 << 40, 4 << 40, 5 << 40, 6 << 40)


def call_merge(o_part=MP, lse_part=MLP, o_acc=MA, lse_acc=MLA, o_out=MO, lse_out=MLO, B=1, H=2, S=64, D=128,
               layout=fa.FA_BSND, dtype=fa.FA_BF16, flags=fa.FA_MERGE_ACCUMULATE | fa.FA_MERGE_FINAL):
    return fa.fa_lse_merge(o_part, lse_part, o_acc, lse_acc, o_out, lse_out, B, H, S, D, layout, dtype, flags,
                           None)


def test_merge_host_validation(lib):
    for kw in (dict(B=0), dict(H=-1), dict(S=-1), dict(layout=3), dict(dtype=7), dict(flags=4), dict(flags=-1),
               dict(o_part=0), dict(lse_part=0), dict(o_acc=0), dict(lse_acc=0), dict(o_out=0),
               dict(lse_out=0), dict(o_acc=0, flags=fa.FA_MERGE_ACCUMULATE), dict(o_acc=0, flags=0),
               dict(o_out=0, flags=fa.FA_MERGE_FINAL)):
        assert call_merge(**kw) == fa.FA_ERR_INVALID_ARG, kw
    assert call_merge(D=96) == fa.FA_ERR_UNSUPPORTED
    assert call_merge(S=0) == fa.FA_OK
    assert call_merge(o_part=MP + 8) == fa.FA_ERR_MISALIGNED
    assert call_merge(o_acc=MA + 4) == fa.FA_ERR_MISALIGNED
    assert call_merge(o_out=MO + 2) == fa.FA_ERR_MISALIGNED
    assert call_merge(lse_acc=MLA + 2) == fa.FA_ERR_MISALIGNED
    assert call_merge(o_out=MP) == fa.FA_ERR_ALIAS
    assert call_merge(lse_out=MA + 64) == fa.FA_ERR_ALIAS
    assert call_merge(o_acc=MP + 4096) == fa.FA_ERR_ALIAS
    assert call_merge(lse_acc=MA + 16) == fa.FA_ERR_ALIAS


def test_merge_optional_buffers_are_not_checked(lib):
    # a final copy (flags = FINAL) needs no running result; a first merge (flags = 0) needs no output:
    # with everything else valid the call reaches the device checks, which fail on fake pointers
    for kw in (dict(o_acc=0, lse_acc=0, flags=fa.FA_MERGE_FINAL), dict(o_out=0, lse_out=0, flags=0)):
        st = call_merge(**kw)
        assert st not in (fa.FA_ERR_INVALID_ARG, fa.FA_ERR_MISALIGNED, fa.FA_ERR_ALIAS), (kw, st)


def call_out_proj(o=MP, w=MA, y=MO, B=1, H=2, S=64, D=128, E=256, layout=fa.FA_BSND, dtype=fa.FA_BF16):
    return fa.fa_out_proj(o, w, y, B, H, S, D, E, layout, dtype, None)


def test_out_proj_host_validation(lib):
    for kw in (dict(B=0), dict(H=0), dict(S=-1), dict(E=0), dict(layout=2), dict(dtype=5), dict(o=0), dict(w=0),
               dict(y=0)):
        assert call_out_proj(**kw) == fa.FA_ERR_INVALID_ARG, kw
    assert call_out_proj(D=32) == fa.FA_ERR_UNSUPPORTED
    assert call_out_proj(E=48) == fa.FA_ERR_UNSUPPORTED          # not a multiple of 32
    assert call_out_proj(S=0) == fa.FA_OK
    assert call_out_proj(o=MP + 8) == fa.FA_ERR_MISALIGNED
    assert call_out_proj(y=MO + 2) == fa.FA_ERR_MISALIGNED
    assert call_out_proj(y=MP + 64) == fa.FA_ERR_ALIAS
    assert call_out_proj(w=MO + 1024) == fa.FA_ERR_ALIAS


def test_fwd_proj_host_validation(lib):
    def call(**kw):
        a = dict(q=Q, k=K, v=V, w=MA, o=O, lse=L, y=MO, B=1, H=2, Sq=64, Sk=64, D=128, E=256, layout=fa.FA_BSND,
                 causal=0, scale=0.125, dtype=fa.FA_BF16)
        a.update(kw)
        return fa.fa_fwd_proj(a["q"], a["k"], a["v"], a["w"], a["o"], a["lse"], a["y"], a["B"], a["H"], a["Sq"],
                              a["Sk"], a["D"], a["E"], a["layout"], a["causal"], a["scale"], a["dtype"], None, 0,
                              None)
    assert call(w=0) == fa.FA_ERR_INVALID_ARG
    assert call(y=0) == fa.FA_ERR_INVALID_ARG
    assert call(E=40) == fa.FA_ERR_UNSUPPORTED
    assert call(y=Q) == fa.FA_ERR_ALIAS
    assert call(w=O) == fa.FA_ERR_ALIAS
    assert call(scale=float("inf")) == fa.FA_ERR_INVALID_ARG


def test_bwd_atomic_workspace_and_validation(lib):
    # the per-row sums plus a [B * H, Sq_pad, D] fp32 accumulator
    assert fa.fa_bwd_atomic_workspace_size(1, 2, 513, 128) == 2 * 640 * (2 + 128) * 4
    assert fa.fa_bwd_atomic_workspace_size(1, 2, 0, 128) == 0

    def call(**kw):
        a = dict(D=128, ws_bytes=fa.fa_bwd_atomic_workspace_size(1, 2, 64, 128))
        a.update(kw)
        return fa.fa_bwd_atomic(Q, K, V, O, DO_, L, DQ, DK, DV, 1, 2, 64, 64, a["D"], fa.FA_BSND, 1, 0.125,
                                fa.FA_BF16, WSB, a["ws_bytes"], None)
    assert call(D=96) == fa.FA_ERR_UNSUPPORTED
    assert call(ws_bytes=fa.fa_bwd_workspace_size(1, 2, 64)) == fa.FA_ERR_INVALID_ARG   # too small for dQ
    # D = 64: its own accumulator size; a D = 128 workspace is large enough, a deterministic one is not
    assert fa.fa_bwd_atomic_workspace_size(1, 2, 64, 64) == 2 * 128 * (2 + 64) * 4
    assert call(D=64, ws_bytes=fa.fa_bwd_workspace_size(1, 2, 64)) == fa.FA_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- split-KV (fa_fwd_splitkv)

SKW = 0x70000000     # a 256-byte aligned fake workspace, far from the fake tensors


def call_split(ws=SKW, ws_bytes=None, nsplit=4, **kw):
    a = dict(GOOD)
    a.update(kw)
    if ws_bytes is None:
        ws_bytes = max(256, fa.fa_fwd_splitkv_workspace_size(a["B"], a["H"], max(a["Sq"], 0), a["D"], nsplit))
    return fa.fa_fwd_splitkv(Q, K, V, O, L, a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["layout"], a["scale"],
                             a["dtype"], nsplit, ws, ws_bytes, None)


def test_splitkv_workspace_size(lib):
    B, H, Sq, D = 2, 3, 300, 128
    for n in (1, 4, 64):
        rows = B * H * n * Sq
        assert fa.fa_fwd_splitkv_workspace_size(B, H, Sq, D, n) == 256 + (rows * 4 + 15) // 16 * 16 + rows * D * 4
    assert fa.fa_fwd_splitkv_workspace_size(B, H, Sq, 64, 8) < fa.fa_fwd_splitkv_workspace_size(B, H, Sq, 128, 8)
    for bad in (dict(nsplit=0), dict(nsplit=65), dict(D=96), dict(B=0), dict(H=-1), dict(Sq=-1)):
        a = dict(B=B, H=H, Sq=Sq, D=D, nsplit=4)
        a.update(bad)
        assert fa.fa_fwd_splitkv_workspace_size(a["B"], a["H"], a["Sq"], a["D"], a["nsplit"]) == 0, bad


def test_splitkv_host_validation(lib):
    for kw in (dict(B=0), dict(layout=3), dict(dtype=5), dict(scale=float("nan")), dict(nsplit=0),
               dict(nsplit=65), dict(ws=0), dict(ws_bytes=255)):
        assert call_split(**kw) == fa.FA_ERR_INVALID_ARG, kw
    # the workspace must hold nsplit splits' partials: one byte short is refused
    need = fa.fa_fwd_splitkv_workspace_size(GOOD["B"], GOOD["H"], GOOD["Sq"], GOOD["D"], 4)
    assert call_split(ws_bytes=need - 1) == fa.FA_ERR_INVALID_ARG
    assert call_split(ws=SKW + 16) == fa.FA_ERR_MISALIGNED
    assert call_split(ws=Q) == fa.FA_ERR_ALIAS
    assert call_split(D=96) == fa.FA_ERR_UNSUPPORTED
    assert call_split(Sq=0) == fa.FA_OK


def test_default_splits():
    assert fa.default_splits(1, 2, 512, 512) == 1            # 4 key tiles: too short to split
    assert fa.default_splits(1, 2, 512, 8192) == 8           # 64 tiles, 8 per range
    assert fa.default_splits(1, 8, 128, 65536) == 18         # 8 units: 148 // 8
    assert fa.default_splits(4, 8, 512, 32768) == 2          # 64 units
    assert fa.default_splits(2, 40, 8192, 8192) == 1         # already thousands of units
    assert fa.default_splits(1, 1, 1, 1000000) == 64         # capped at 64
