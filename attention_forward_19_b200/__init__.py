"""B200 (sm_100a) FlashAttention forward: Python binding of libfa_fwd.so.

The binding only marshals arguments: it reads pointers, shapes and the
current CUDA stream from torch tensors and calls the C ABI declared in
include/fa_fwd.h.  Every step of the computation runs in the library's CUDA
kernel.  There is no CPU fallback: if the library cannot be loaded, importing
the entry points raises.

    from attention_forward_19_b200 import flash_attention_forward
    o, lse = flash_attention_forward(q, k, v, layout="BHSD", causal=True)

The C entry points are also exposed under their own names (fa_fwd,
fa_device_status, fa_query_support, fa_status_string, fa_last_cuda_error,
fa_version) with the same arguments as in the header.
"""
import ctypes
import math
import os

from . import build as _build

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_NOT_DEVICE_POINTER = 3
FA_ERR_MISALIGNED = 4
FA_ERR_ALIAS = 5
FA_ERR_CUDA = 6
FA_ERR_TIMEOUT = 7

FA_BSND = 0
FA_BHSD = 1
FA_FP16 = 0
FA_BF16 = 1

FA_MERGE_ACCUMULATE = 1
FA_MERGE_FINAL = 2

LAYOUTS = {"BSND": FA_BSND, "BHSD": FA_BHSD}

# Names every public symbol of include/fa_fwd.h.
EXPORTED_SYMBOLS = ("fa_fwd", "fa_fwd_ws", "fa_fwd_workspace_size", "fa_fwd_opts", "fa_fwd_default_options",
                    "fa_fwd_heads", "fa_fwd_noalloc", "fa_fwd_varlen", "fa_fwd_splitkv",
                    "fa_fwd_splitkv_workspace_size",
                    "fa_bwd",
                    "fa_bwd_workspace_size", "fa_bwd_atomic",
                    "fa_bwd_atomic_workspace_size", "fa_lse_merge", "fa_fwd_ring_step", "fa_out_proj",
                    "fa_fwd_proj",
                    "fa_selftest_wait_timeout", "fa_device_status", "fa_query_support", "fa_status_string",
                    "fa_last_cuda_error", "fa_version")


class FwdOptions(ctypes.Structure):
    """The C fa_fwd_options: the lazy rescale's threshold and bf16 headroom (log2 units) and an
    optional device pointer to four 64-bit branch counters."""
    _fields_ = [("rescale_threshold_log2", ctypes.c_float), ("bf16_headroom_log2", ctypes.c_float),
                ("branch_counts", ctypes.c_void_p)]


class RingSegment(ctypes.Structure):
    """The C fa_ring_segment: query rows [row0, row0 + rows) against keys [key0, key0 + keys); a causal
    offset >= 0 makes key c visible from row r iff c <= r + offset (< 0: no mask); first / last say
    whether the rows have an earlier result to merge with and whether this result is final."""
    _fields_ = [("row0", ctypes.c_int64), ("key0", ctypes.c_int64), ("keys", ctypes.c_int64),
                ("causal_offset", ctypes.c_int64), ("first", ctypes.c_int32), ("last", ctypes.c_int32)]


class FaError(RuntimeError):
    """A non-zero fa_status returned by the library."""

    def __init__(self, status, where):
        self.status = status
        name = fa_status_string(status) if _LIB is not None else str(status)
        extra = ""
        if status == FA_ERR_CUDA and _LIB is not None:
            extra = f" (CUDA error {fa_last_cuda_error()})"
        super().__init__(f"{where}: {name}{extra}")


_LIB = None


def library_path():
    return _build.LIB


def load_library(path=None, rebuild_if_stale=True):
    """Loads libfa_fwd.so (compiling it first if missing or stale and nvcc is available)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if path is None:
        path = _build.LIB
        if rebuild_if_stale and os.path.exists(_build.NVCC):
            _build.build()
    if not os.path.exists(path):
        raise ImportError(f"the CUDA library {path} is missing; run python -m attention_forward_19_b200.build")
    lib = ctypes.CDLL(path)
    i64, vp, c_int, c_float = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.restype = c_int
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, c_float, c_int, vp]
    lib.fa_fwd_ws.restype = c_int
    lib.fa_fwd_ws.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, c_float, c_int, vp,
                              ctypes.c_size_t, vp]
    lib.fa_fwd_opts.restype = c_int
    lib.fa_fwd_opts.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, c_float, c_int,
                                ctypes.POINTER(FwdOptions), vp, ctypes.c_size_t, vp]
    lib.fa_fwd_default_options.restype = None
    lib.fa_fwd_default_options.argtypes = [ctypes.POINTER(FwdOptions)]
    lib.fa_fwd_heads.restype = c_int
    lib.fa_fwd_heads.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, c_float, c_int, i64, i64,
                                 vp, ctypes.c_size_t, vp]
    lib.fa_fwd_noalloc.restype = c_int
    lib.fa_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, c_float, c_int, vp]
    lib.fa_fwd_varlen.restype = c_int
    lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, c_int, c_float,
                                  c_int, vp, ctypes.c_size_t, vp]
    lib.fa_bwd.restype = c_int
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, c_float, c_int,
                           vp, ctypes.c_size_t, vp]
    lib.fa_lse_merge.restype = c_int
    lib.fa_lse_merge.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, c_int, c_int, c_int, vp]
    lib.fa_fwd_splitkv.restype = c_int
    lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_float, c_int, c_int, vp,
                                   ctypes.c_size_t, vp]
    lib.fa_fwd_splitkv_workspace_size.restype = ctypes.c_size_t
    lib.fa_fwd_splitkv_workspace_size.argtypes = [i64, i64, i64, i64, c_int]
    lib.fa_fwd_ring_step.restype = c_int
    lib.fa_fwd_ring_step.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.POINTER(RingSegment),
                                     c_int, c_int, c_float, c_int, vp, ctypes.c_size_t, vp]
    lib.fa_out_proj.restype = c_int
    lib.fa_out_proj.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, vp]
    lib.fa_fwd_proj.restype = c_int
    lib.fa_fwd_proj.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, c_int, c_int, c_float,
                                c_int, vp, ctypes.c_size_t, vp]
    lib.fa_bwd_atomic.restype = c_int
    lib.fa_bwd_atomic.argtypes = lib.fa_bwd.argtypes
    lib.fa_bwd_atomic_workspace_size.restype = ctypes.c_size_t
    lib.fa_bwd_atomic_workspace_size.argtypes = [i64, i64, i64, i64]
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_bwd_workspace_size.argtypes = [i64, i64, i64]
    lib.fa_selftest_wait_timeout.restype = c_int
    lib.fa_selftest_wait_timeout.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, c_float,
                                             c_int, ctypes.c_uint32, vp]
    lib.fa_fwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_fwd_workspace_size.argtypes = []
    lib.fa_device_status.restype = c_int
    lib.fa_device_status.argtypes = [vp]
    lib.fa_query_support.restype = c_int
    lib.fa_query_support.argtypes = [i64, c_int]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_status_string.argtypes = [c_int]
    lib.fa_last_cuda_error.restype = c_int
    lib.fa_last_cuda_error.argtypes = []
    lib.fa_version.restype = c_int
    lib.fa_version.argtypes = []
    _LIB = lib
    return lib


# ----------------------------------------------------------------------------- raw C entry points


def fa_fwd(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, stream):
    """The C fa_fwd with raw pointers (ints) and sizes; returns the fa_status code."""
    lib = load_library()
    return lib.fa_fwd(q, k, v, o, lse, int(B), int(H), int(Sq), int(Sk), int(D), int(layout),
                      int(bool(causal)), float(scale), int(dtype), stream)


def fa_fwd_ws(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, workspace, workspace_bytes,
              stream):
    """The C fa_fwd_ws (dynamic schedule) with raw pointers and sizes; returns the fa_status code."""
    lib = load_library()
    return lib.fa_fwd_ws(q, k, v, o, lse, int(B), int(H), int(Sq), int(Sk), int(D), int(layout),
                         int(bool(causal)), float(scale), int(dtype), workspace, int(workspace_bytes), stream)


def fa_fwd_default_options():
    """The C fa_fwd_default_options: a FwdOptions holding the defaults fa_fwd uses."""
    opts = FwdOptions()
    load_library().fa_fwd_default_options(ctypes.byref(opts))
    return opts


def fa_fwd_opts(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, opts, workspace, workspace_bytes,
                stream):
    """The C fa_fwd_opts (opts: a FwdOptions or None) with raw pointers; returns the fa_status code."""
    lib = load_library()
    return lib.fa_fwd_opts(q, k, v, o, lse, int(B), int(H), int(Sq), int(Sk), int(D), int(layout),
                           int(bool(causal)), float(scale), int(dtype), ctypes.byref(opts) if opts is not None else None,
                           workspace, int(workspace_bytes), stream)


def fa_fwd_heads(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, head_begin, head_count,
                 workspace, workspace_bytes, stream):
    """The C fa_fwd_heads (only the flattened heads [head_begin, head_begin + head_count) of the
    whole problem's tensors) with raw pointers and sizes; returns the fa_status code."""
    lib = load_library()
    return lib.fa_fwd_heads(q, k, v, o, lse, int(B), int(H), int(Sq), int(Sk), int(D), int(layout),
                            int(bool(causal)), float(scale), int(dtype), int(head_begin), int(head_count), workspace,
                            int(workspace_bytes), stream)


def fa_fwd_noalloc(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, stream):
    """The C fa_fwd_noalloc: the dynamic schedule with the library's fixed scratch, for callers
    that cannot allocate device memory; returns the fa_status code."""
    lib = load_library()
    return lib.fa_fwd_noalloc(q, k, v, o, lse, int(B), int(H), int(Sq), int(Sk), int(D), int(layout),
                              int(bool(causal)), float(scale), int(dtype), stream)


def fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, total_q, total_k, max_q, max_k, D, causal, scale, dtype,
                  workspace, workspace_bytes, stream):
    """The C fa_fwd_varlen (packed variable-length batch) with raw pointers; returns the fa_status code."""
    lib = load_library()
    return lib.fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, int(B), int(H), int(total_q), int(total_k), int(max_q),
                             int(max_k), int(D), int(bool(causal)), float(scale), int(dtype), workspace,
                             int(workspace_bytes), stream)


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, Sq, Sk, D, layout, causal, scale, dtype, workspace,
           workspace_bytes, stream):
    """The C fa_bwd (gradients) with raw pointers and sizes; returns the fa_status code."""
    lib = load_library()
    return lib.fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, int(B), int(H), int(Sq), int(Sk), int(D), int(layout),
                      int(bool(causal)), float(scale), int(dtype), workspace, int(workspace_bytes), stream)


def fa_lse_merge(o_part, lse_part, o_acc, lse_acc, o_out, lse_out, B, H, S, D, layout, dtype, flags, stream):
    """The C fa_lse_merge (merge of a partial attention result) with raw pointers; returns the fa_status code."""
    lib = load_library()
    return lib.fa_lse_merge(o_part, lse_part, o_acc, lse_acc, o_out, lse_out, int(B), int(H), int(S), int(D),
                            int(layout), int(dtype), int(flags), stream)


def fa_fwd_splitkv(q, k, v, o, lse, B, H, Sq, Sk, D, layout, scale, dtype, nsplit, workspace, workspace_bytes,
                   stream):
    """The C fa_fwd_splitkv with raw pointers and sizes; returns the fa_status code."""
    lib = load_library()
    return lib.fa_fwd_splitkv(q, k, v, o, lse, int(B), int(H), int(Sq), int(Sk), int(D), int(layout), float(scale),
                              int(dtype), int(nsplit), workspace, int(workspace_bytes), stream)


def fa_fwd_splitkv_workspace_size(B, H, Sq, D, nsplit):
    return load_library().fa_fwd_splitkv_workspace_size(int(B), int(H), int(Sq), int(D), int(nsplit))


def fa_fwd_ring_step(q, k, v, o, acc, lse, B, H, Sq, Sk, D, rows, segs, layout, scale, dtype, workspace,
                     workspace_bytes, stream):
    """The C fa_fwd_ring_step with raw pointers; segs is a sequence of (row0, key0, keys, causal_offset,
    first, last) tuples.  Returns the fa_status code."""
    lib = load_library()
    arr = (RingSegment * max(1, len(segs)))(*[RingSegment(*[int(x) for x in g]) for g in segs])
    return lib.fa_fwd_ring_step(q, k, v, o, acc, lse, int(B), int(H), int(Sq), int(Sk), int(D), int(rows), arr,
                                len(segs), int(layout), float(scale), int(dtype), workspace, int(workspace_bytes),
                                stream)


def fa_out_proj(o, w_o, y, B, H, S, D, E, layout, dtype, stream):
    """The C fa_out_proj (y = o w_o^T) with raw pointers and sizes; returns the fa_status code."""
    return load_library().fa_out_proj(o, w_o, y, int(B), int(H), int(S), int(D), int(E), int(layout), int(dtype),
                                      stream)


def fa_fwd_proj(q, k, v, w_o, o, lse, y, B, H, Sq, Sk, D, E, layout, causal, scale, dtype, workspace,
                workspace_bytes, stream):
    """The C fa_fwd_proj (attention, then y = o w_o^T) with raw pointers; returns the fa_status code."""
    return load_library().fa_fwd_proj(q, k, v, w_o, o, lse, y, int(B), int(H), int(Sq), int(Sk), int(D), int(E),
                                      int(layout), int(bool(causal)), float(scale), int(dtype), workspace,
                                      int(workspace_bytes), stream)


def fa_bwd_atomic(q, k, v, o, dout, lse, dq, dk, dv, B, H, Sq, Sk, D, layout, causal, scale, dtype, workspace,
                  workspace_bytes, stream):
    """The C fa_bwd_atomic (non-deterministic dQ accumulation) with raw pointers; returns the fa_status code."""
    lib = load_library()
    return lib.fa_bwd_atomic(q, k, v, o, dout, lse, dq, dk, dv, int(B), int(H), int(Sq), int(Sk), int(D),
                             int(layout), int(bool(causal)), float(scale), int(dtype), workspace,
                             int(workspace_bytes), stream)


def fa_bwd_atomic_workspace_size(B, H, Sq, D):
    return load_library().fa_bwd_atomic_workspace_size(int(B), int(H), int(Sq), int(D))


def fa_bwd_workspace_size(B, H, Sq):
    return load_library().fa_bwd_workspace_size(int(B), int(H), int(Sq))


def fa_selftest_wait_timeout(q, k, v, o, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, wait_limit_us,
                             stream):
    """The C fa_selftest_wait_timeout: a launch whose loads are withheld, so that every bounded
    wait runs out; returns the fa_status code of the launch."""
    lib = load_library()
    return lib.fa_selftest_wait_timeout(q, k, v, o, lse, int(B), int(H), int(Sq), int(Sk), int(D), int(layout),
                                        int(bool(causal)), float(scale), int(dtype), int(wait_limit_us), stream)


def fa_fwd_workspace_size():
    return load_library().fa_fwd_workspace_size()


def fa_device_status(stream=None):
    return load_library().fa_device_status(stream)


def fa_query_support(D, dtype):
    return load_library().fa_query_support(int(D), int(dtype))


def fa_status_string(status):
    return load_library().fa_status_string(int(status)).decode()


def fa_last_cuda_error():
    return load_library().fa_last_cuda_error()


def fa_version():
    return load_library().fa_version()


# ----------------------------------------------------------------------------- torch convenience


def _dtype_code(t):
    import torch
    if t.dtype == torch.float16:
        return FA_FP16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float16 or bfloat16")


def _dims(q, k, layout, head_num=None):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D")
    if layout == FA_BSND:
        B, Sq, H, D = q.shape
        Bk, Sk, Hk, Dk = k.shape
    else:
        B, H, Sq, D = q.shape
        Bk, Hk, Sk, Dk = k.shape
    if (Bk, Hk, Dk) != (B, H, D):
        raise ValueError(f"q {tuple(q.shape)} and k {tuple(k.shape)} do not match in layout "
                         f"{'BSND' if layout == FA_BSND else 'BHSD'}")
    if head_num is not None and head_num != H:
        raise ValueError(f"head_num mismatch: head_num={head_num} but the tensors hold {H} heads")
    return B, H, Sq, Sk, D


def flash_attention_forward(q, k, v, layout="BSND", causal=False, scale=None, head_num=None,
                            out=None, lse=None, stream=None, schedule="dynamic", workspace=None, heads=None,
                            softmax_options=None):
    """Attention forward on CUDA tensors through the C ABI.

    q: [B, Sq, H, D] (BSND) or [B, H, Sq, D] (BHSD); k, v likewise with Sk.
    scale=None uses 1/sqrt(D).  Returns (o, lse): o like q, lse fp32 [B, H, Sq].
    out / lse may be given to reuse buffers.  Runs on `stream` (default: the
    current torch stream) without synchronising.
    schedule="dynamic" calls fa_fwd_ws (work units handed out from a counter
    in `workspace`, a uint8 CUDA tensor of fa_fwd_workspace_size() bytes,
    allocated here when not given); "static" calls fa_fwd (no workspace).
    heads=(head_begin, head_count) calls fa_fwd_heads instead: only the
    flattened heads b * H + h in that range are computed, in place in the
    whole tensors; the other heads' rows of out and lse are left as they were.
    softmax_options (a dict with any of rescale_threshold_log2,
    bf16_headroom_log2, branch_counts -- a CUDA int64 tensor of 4 counters the
    kernel increments) calls fa_fwd_opts with those lazy-rescale settings.
    """
    import torch
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    B, H, Sq, Sk, D = _dims(q, k, lay, head_num)
    if v.shape != k.shape:
        raise ValueError(f"v {tuple(v.shape)} must have k's shape {tuple(k.shape)}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous in the stated layout")
        if t.dtype != q.dtype:
            raise TypeError("q, k, v must share one dtype")
    dt = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor like q")
    if lse.shape != (B, H, Sq) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor of shape [B, H, Sq]")
    if stream is None:
        stream = torch.cuda.current_stream(q.device) if q.is_cuda else None
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    if softmax_options is not None:
        if heads is not None:
            raise ValueError("softmax_options and heads cannot be combined")
        opts = fa_fwd_default_options()
        for key, val in softmax_options.items():
            if key == "branch_counts":
                if val.dtype != torch.int64 or val.numel() < 4 or not val.is_contiguous():
                    raise ValueError("branch_counts must be a contiguous int64 tensor of 4 counters")
                opts.branch_counts = val.data_ptr()
            elif key in ("rescale_threshold_log2", "bf16_headroom_log2"):
                setattr(opts, key, float(val))
            else:
                raise ValueError(f"unknown softmax option {key!r}")
        wptr, wbytes = None, 0
        if schedule == "dynamic":
            nbytes = fa_fwd_workspace_size()
            if workspace is None:
                workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
            wptr, wbytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
        elif schedule != "static":
            raise ValueError(f"schedule must be 'dynamic' or 'static', not {schedule!r}")
        st = fa_fwd_opts(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                         B, H, Sq, Sk, D, lay, causal, scale, dt, opts, wptr, wbytes, sptr)
        if st != FA_OK:
            raise FaError(st, "fa_fwd_opts")
        return out, lse
    if heads is not None:
        h0, hc = (int(x) for x in heads)
        wptr, wbytes = None, 0
        if schedule == "dynamic":
            nbytes = fa_fwd_workspace_size()
            if workspace is None:
                workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
            if workspace.numel() * workspace.element_size() < nbytes or not workspace.is_contiguous():
                raise ValueError(f"workspace must be a contiguous tensor of at least {nbytes} bytes")
            wptr, wbytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
        elif schedule != "static":
            raise ValueError(f"schedule must be 'dynamic' or 'static', not {schedule!r}")
        st = fa_fwd_heads(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                          B, H, Sq, Sk, D, lay, causal, scale, dt, h0, hc, wptr, wbytes, sptr)
        if st != FA_OK:
            raise FaError(st, "fa_fwd_heads")
        return out, lse
    if schedule == "static":
        st = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                    B, H, Sq, Sk, D, lay, causal, scale, dt, sptr)
        where = "fa_fwd"
    elif schedule == "dynamic":
        nbytes = fa_fwd_workspace_size()
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
        if workspace.numel() * workspace.element_size() < nbytes or not workspace.is_contiguous():
            raise ValueError(f"workspace must be a contiguous tensor of at least {nbytes} bytes")
        st = fa_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                       B, H, Sq, Sk, D, lay, causal, scale, dt, workspace.data_ptr(),
                       workspace.numel() * workspace.element_size(), sptr)
        where = "fa_fwd_ws"
    else:
        raise ValueError(f"schedule must be 'dynamic' or 'static', not {schedule!r}")
    if st != FA_OK:
        raise FaError(st, where)
    return out, lse


def flash_attention_varlen_forward(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q=None, max_seqlen_k=None,
                                   causal=False, scale=None, out=None, lse=None, stream=None, schedule="dynamic",
                                   workspace=None):
    """Attention forward over a packed batch of sequences of different lengths.

    q: [total_q, H, D]; k, v: [total_k, H, D]; cu_seqlens_q / cu_seqlens_k: int32
    CUDA tensors of B + 1 offsets (sequence b owns rows cu[b] .. cu[b+1]-1).
    max_seqlen_q / max_seqlen_k bound the lengths; when None they are read from
    the offsets (a device-to-host copy, which synchronises).  Returns (o, lse):
    o like q, lse fp32 [H, total_q].  Invalid offsets are reported by
    check_device_status().
    """
    import torch
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape:
        raise ValueError("q must be [total_q, H, D] and k, v [total_k, H, D]")
    total_q, H, D = q.shape
    total_k, Hk, Dk = k.shape
    if (Hk, Dk) != (H, D):
        raise ValueError(f"q {tuple(q.shape)} and k {tuple(k.shape)} differ in heads or head dim")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dtype != q.dtype:
            raise TypeError("q, k, v must share one dtype")
    for name, c in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if c.dtype != torch.int32 or c.dim() != 1 or not c.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 1-D int32 tensor")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must hold the same number (B + 1 >= 2) of offsets")
    B = cu_seqlens_q.numel() - 1
    if max_seqlen_q is None:
        max_seqlen_q = int((cu_seqlens_q[1:] - cu_seqlens_q[:-1]).max().item())
    if max_seqlen_k is None:
        max_seqlen_k = int((cu_seqlens_k[1:] - cu_seqlens_k[:-1]).max().item())
    dt = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor like q")
    if lse.shape != (H, total_q) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor of shape [H, total_q]")
    if stream is None:
        stream = torch.cuda.current_stream(q.device) if q.is_cuda else None
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    ws_ptr, ws_bytes = None, 0
    if schedule == "dynamic":
        nbytes = fa_fwd_workspace_size()
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
        if ws_bytes < nbytes or not workspace.is_contiguous():
            raise ValueError(f"workspace must be a contiguous tensor of at least {nbytes} bytes")
        ws_ptr = workspace.data_ptr()
    elif schedule != "static":
        raise ValueError(f"schedule must be 'dynamic' or 'static', not {schedule!r}")
    st = fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                       cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, H, total_q, total_k, max_seqlen_q,
                       max_seqlen_k, D, causal, scale, dt, ws_ptr, ws_bytes, sptr)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_varlen")
    return out, lse


def flash_attention_backward(q, k, v, o, lse, dout, layout="BSND", causal=False, scale=None, dq=None, dk=None,
                             dv=None, stream=None, workspace=None, deterministic=True):
    """Gradients (dq, dk, dv) of flash_attention_forward through the C ABI.

    q, k, v as for the forward; o and lse as the forward returned them; dout
    (dL/dO) like o.  Returns (dq, dk, dv) shaped like q, k, v.  `workspace`, a
    uint8 CUDA tensor of fa_bwd_workspace_size(B, H, Sq) bytes
    (fa_bwd_atomic_workspace_size(B, H, Sq, D) when deterministic=False), is
    allocated here when not given.  deterministic=False calls fa_bwd_atomic:
    one kernel per key tile, dQ added up in fp32 in any order.
    Runs on `stream` without synchronising.
    """
    import torch
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    B, H, Sq, Sk, D = _dims(q, k, lay)
    for name, t, like in (("v", v, k), ("o", o, q), ("dout", dout, q)):
        if t.shape != like.shape or t.dtype != q.dtype or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous tensor of shape {tuple(like.shape)} and q's dtype")
    for name, t in (("q", q), ("k", k)):
        if not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError(f"{name} must be contiguous and share q's dtype")
    if lse.shape != (B, H, Sq) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be the forward's contiguous fp32 [B, H, Sq] tensor")
    dt = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, like in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t.shape != like.shape or t.dtype != like.dtype or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous tensor like {name[1:]}")
    nbytes = fa_bwd_workspace_size(B, H, Sq) if deterministic else fa_bwd_atomic_workspace_size(B, H, Sq, D)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    if stream is None:
        stream = torch.cuda.current_stream(q.device) if q.is_cuda else None
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    fn = fa_bwd if deterministic else fa_bwd_atomic
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, Sq, Sk, D, lay, causal, scale, dt,
            workspace.data_ptr(), wbytes, sptr)
    if st != FA_OK:
        raise FaError(st, "fa_bwd" if deterministic else "fa_bwd_atomic")
    return dq, dk, dv


def lse_merge(o_part, lse_part, o_acc=None, lse_acc=None, out=None, lse_out=None, layout="BSND",
              accumulate=False, final=False, stream=None):
    """Merges a partial attention result (o_part, lse_part), normalised over one key block, into the
    running fp32 result (o_acc, lse_acc) through fa_lse_merge.

    o_part: 16-bit, [B, S, H, D] (BSND) or [B, H, S, D] (BHSD); lse_part fp32 [B, H, S].
    accumulate=False starts the running result from the partial; accumulate=True merges.  final=True
    writes the merged result to (out, lse_out) in o_part's dtype (allocated here when None) instead
    of updating (o_acc, lse_acc).  Returns (o_acc, lse_acc), or (out, lse_out) when final.
    """
    import torch
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    if o_part.dim() != 4 or not o_part.is_contiguous():
        raise ValueError("o_part must be a contiguous 4-D tensor")
    if lay == FA_BSND:
        B, S, H, D = o_part.shape
    else:
        B, H, S, D = o_part.shape
    dt = _dtype_code(o_part)
    if lse_part.shape != (B, H, S) or lse_part.dtype != torch.float32 or not lse_part.is_contiguous():
        raise ValueError("lse_part must be a contiguous fp32 tensor of shape [B, H, S]")
    need_acc = accumulate or not final
    if need_acc:
        if o_acc is None and not accumulate:
            o_acc = torch.empty(o_part.shape, dtype=torch.float32, device=o_part.device)
        if lse_acc is None and not accumulate:
            lse_acc = torch.empty((B, H, S), dtype=torch.float32, device=o_part.device)
        if o_acc is None or lse_acc is None:
            raise ValueError("accumulate=True needs the running result (o_acc, lse_acc)")
        if o_acc.shape != o_part.shape or o_acc.dtype != torch.float32 or not o_acc.is_contiguous():
            raise ValueError("o_acc must be a contiguous fp32 tensor shaped like o_part")
        if lse_acc.shape != (B, H, S) or lse_acc.dtype != torch.float32 or not lse_acc.is_contiguous():
            raise ValueError("lse_acc must be a contiguous fp32 tensor of shape [B, H, S]")
    if final:
        out = torch.empty_like(o_part) if out is None else out
        lse_out = torch.empty((B, H, S), dtype=torch.float32, device=o_part.device) if lse_out is None else lse_out
        if out.shape != o_part.shape or out.dtype != o_part.dtype or not out.is_contiguous():
            raise ValueError("out must be a contiguous tensor like o_part")
        if lse_out.shape != (B, H, S) or lse_out.dtype != torch.float32 or not lse_out.is_contiguous():
            raise ValueError("lse_out must be a contiguous fp32 tensor of shape [B, H, S]")
    if stream is None:
        stream = torch.cuda.current_stream(o_part.device) if o_part.is_cuda else None
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    flags = (FA_MERGE_ACCUMULATE if accumulate else 0) | (FA_MERGE_FINAL if final else 0)
    ptr = lambda t: t.data_ptr() if t is not None else None
    st = fa_lse_merge(o_part.data_ptr(), lse_part.data_ptr(), ptr(o_acc) if need_acc else None,
                      ptr(lse_acc) if need_acc else None, ptr(out) if final else None,
                      ptr(lse_out) if final else None, B, H, S, D, lay, dt, flags, sptr)
    if st != FA_OK:
        raise FaError(st, "fa_lse_merge")
    return (out, lse_out) if final else (o_acc, lse_acc)


def default_splits(B, H, Sq, Sk, sms=148):
    """A split count for flash_attention_forward_splitkv: enough key ranges to give every SM about one
    work unit (units of 256 query rows), each range at least 8 key tiles of 128 (a shorter range does not
    pay for the merge kernel: at 512 keys, c1, one pass takes 14.6 us and two ranges 17.9 us), at most
    64; 1 means the one-pass kernel is the better choice."""
    units = B * H * ((Sq + 255) // 256)
    return max(1, min(64, ((Sk + 127) // 128) // 8, sms // max(1, units)))


def flash_attention_forward_splitkv(q, k, v, layout="BSND", scale=None, nsplit=None, out=None, lse=None,
                                    workspace=None, stream=None):
    """Attention without a mask through fa_fwd_splitkv: the key range split into nsplit ranges (default
    default_splits(...)), each a work unit of its own, the partial results merged by a second kernel.
    Arguments and results as for flash_attention_forward (causal=False)."""
    import torch
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    B, H, Sq, Sk, D = _dims(q, k, lay)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if nsplit is None:
        nsplit = default_splits(B, H, Sq, Sk, torch.cuda.get_device_properties(q.device).multi_processor_count)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device) if lse is None else lse
    need = fa_fwd_splitkv_workspace_size(B, H, Sq, D, nsplit)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    st = fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, Sq, Sk, D,
                        lay, scale, _dtype_code(q), nsplit, workspace.data_ptr(), workspace.numel(), sptr)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_splitkv")
    return out, lse


def ring_step(q, k, v, segments, rows, out, lse, acc=None, layout="BSND", scale=None, workspace=None, stream=None):
    """One ring-attention step through fa_fwd_ring_step: every segment (row0, key0, keys, causal_offset,
    first, last) attends its query rows of q to its keys of k / v and merges the result into the running
    result of those rows (acc fp32 like q, lse fp32 [B, H, Sq]), or writes the final one to out / lse.

    q, out: [B, Sq, H, D] (BSND) or [B, H, Sq, D] (BHSD); k, v likewise with Sk rows; all contiguous CUDA
    tensors.  scale=None uses 1/sqrt(D).  Asynchronous on `stream` (default: the current torch stream)."""
    import torch
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    B, H, Sq, Sk, D = _dims(q, k, lay)
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if v.shape != k.shape or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("v must be shaped like k and out like q")
    if lse.shape != (B, H, Sq) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor of shape [B, H, Sq]")
    if acc is not None and (acc.shape != q.shape or acc.dtype != torch.float32 or not acc.is_contiguous()):
        raise ValueError("acc must be a contiguous fp32 tensor shaped like q")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if workspace is None:
        workspace = torch.empty(fa_fwd_workspace_size(), dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    st = fa_fwd_ring_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                          acc.data_ptr() if acc is not None else None, lse.data_ptr(), B, H, Sq, Sk, D, rows,
                          segments, lay, scale, _dtype_code(q), workspace.data_ptr(), workspace.numel(), sptr)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_ring_step")
    return out, lse


def _proj_dims(o, w_o, lay):
    if o.dim() != 4 or not o.is_contiguous():
        raise ValueError("o must be a contiguous 4-D tensor")
    if lay == FA_BSND:
        B, S, H, D = o.shape
    else:
        B, H, S, D = o.shape
    if w_o.dim() != 2 or w_o.shape[1] != H * D or not w_o.is_contiguous() or w_o.dtype != o.dtype:
        raise ValueError(f"w_o must be a contiguous [E, H * D = {H * D}] tensor of o's dtype")
    return B, H, S, D, w_o.shape[0]


def out_projection(o, w_o, layout="BSND", y=None, stream=None):
    """y = o w_o^T through fa_out_proj: o [B, S, H, D] (BSND) or [B, H, S, D] (BHSD), w_o [E, H * D]
    (a linear layer's weight).  Returns y [B, S, E] in o's dtype."""
    import torch
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    B, H, S, D, E = _proj_dims(o, w_o, lay)
    if y is None:
        y = torch.empty((B, S, E), dtype=o.dtype, device=o.device)
    if y.shape != (B, S, E) or y.dtype != o.dtype or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous [{B}, {S}, {E}] tensor of o's dtype")
    if stream is None:
        stream = torch.cuda.current_stream(o.device) if o.is_cuda else None
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    st = fa_out_proj(o.data_ptr(), w_o.data_ptr(), y.data_ptr(), B, H, S, D, E, lay, _dtype_code(o), sptr)
    if st != FA_OK:
        raise FaError(st, "fa_out_proj")
    return y


def flash_attention_forward_proj(q, k, v, w_o, layout="BSND", causal=False, scale=None, out=None, lse=None, y=None,
                                 stream=None, workspace=None):
    """Attention followed by its output projection (fa_fwd_proj): returns (y, o, lse) with
    y = o w_o^T [B, Sq, E], o and lse as flash_attention_forward returns them."""
    import torch
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    B, H, Sq, Sk, D = _dims(q, k, lay)
    if v.shape != k.shape:
        raise ValueError(f"v {tuple(v.shape)} must have k's shape {tuple(k.shape)}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError(f"{name} must be contiguous and share q's dtype")
    if w_o.dim() != 2 or w_o.shape[1] != H * D or not w_o.is_contiguous() or w_o.dtype != q.dtype:
        raise ValueError(f"w_o must be a contiguous [E, H * D = {H * D}] tensor of q's dtype")
    E = w_o.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device) if lse is None else lse
    y = torch.empty((B, Sq, E), dtype=q.dtype, device=q.device) if y is None else y
    if out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor like q")
    if lse.shape != (B, H, Sq) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor of shape [B, H, Sq]")
    if y.shape != (B, Sq, E) or y.dtype != q.dtype or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous [{B}, {Sq}, {E}] tensor of q's dtype")
    nbytes = fa_fwd_workspace_size()
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device) if q.is_cuda else None
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    st = fa_fwd_proj(q.data_ptr(), k.data_ptr(), v.data_ptr(), w_o.data_ptr(), out.data_ptr(), lse.data_ptr(),
                     y.data_ptr(), B, H, Sq, Sk, D, E, lay, causal, scale, _dtype_code(q), workspace.data_ptr(),
                     workspace.numel() * workspace.element_size(), sptr)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_proj")
    return y, out, lse


def check_device_status(stream=None):
    """Synchronises the stream and raises FaError if a kernel reported a wait timeout (or invalid
    sequence offsets of a variable-length batch)."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    st = fa_device_status(sptr)
    if st != FA_OK:
        raise FaError(st, "fa_device_status")
