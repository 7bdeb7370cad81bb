"""Python binding of the fp64 attention oracle (attn_oracle.c).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the package
smoke check and the benchmark's CPU-baseline / reference arm import this
module.  It shares nothing with the CUDA path.

The oracle computes, straight from the definition of the standard attention
on the pages (page "FlashAttention in ops-transformer on Ascend NPU",
section "why standard attention stalls"; page "FlashAttention: long-text
inference without running out of memory", section "the memory black hole"):

    O   = softmax(scale * Q K^T  [+ causal mask]) V
    LSE = M + ln(sum_j exp(s_j - M))      per query row (natural log)

with the causal mask aligned at the top-left corner (key j visible to query
i iff j <= i).  See attn_oracle.c for the details and the exact-decoding of
the 16-bit inputs.
"""
import ctypes
import os

import numpy as np

from . import build as _build

FP16, BF16, F64 = 0, 1, 2
BSND, BHSD = 0, 1
_LAYOUTS = {"BSND": BSND, "BHSD": BHSD}


def _as_u16_or_f64(x):
    """Returns (numpy array, dtype code) with the raw bits of a 16-bit tensor or fp64 data."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.float16:
            return x.view(torch.int16).numpy().view(np.uint16), FP16
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), BF16
        return x.to(torch.float64).numpy(), F64
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return x.view(np.uint16), FP16
    return np.ascontiguousarray(x, dtype=np.float64), F64


class Oracle:
    """Handle on one build of the oracle library (the normal one or a planted variant)."""

    def __init__(self, lib_path=None):
        if lib_path is None:
            lib_path = _build.build()
        self.lib_path = lib_path
        self._lib = ctypes.CDLL(lib_path)
        i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        c_int = ctypes.c_int
        f = self._lib.oracle_attn_fwd_rows
        f.restype = c_int
        f.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, dbl, c_int,
                      vp, i64, vp, vp, c_int]
        w = self._lib.oracle_attn_weights
        w.restype = c_int
        w.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, c_int, c_int, dbl, c_int, i64, vp]
        for name in ("oracle_fp16_to_f64", "oracle_bf16_to_f64"):
            g = getattr(self._lib, name)
            g.restype = dbl
            g.argtypes = [ctypes.c_uint16]
        self._lib.oracle_max_threads.restype = c_int
        self._lib.oracle_plant.restype = c_int

    @property
    def plant(self):
        return self._lib.oracle_plant()

    def max_threads(self):
        return self._lib.oracle_max_threads()

    def decode_fp16(self, bits):
        return self._lib.oracle_fp16_to_f64(int(bits))

    def decode_bf16(self, bits):
        return self._lib.oracle_bf16_to_f64(int(bits))

    @staticmethod
    def _dims(q, k, layout):
        if q.ndim != 4 or k.ndim != 4:
            raise ValueError("q, k, v must be 4-D")
        if layout == BSND:
            B, Sq, H, D = q.shape
            Sk = k.shape[1]
        else:
            B, H, Sq, D = q.shape
            Sk = k.shape[2]
        return B, H, Sq, Sk, D

    def fwd(self, q, k, v, *, layout="BHSD", causal=False, scale=None, rows=None, threads=0):
        """Attention forward in fp64.

        q, k, v: torch tensors (fp16 / bf16 / any float) or numpy arrays in the
        given layout ("BSND" = [B, S, H, D], "BHSD" = [B, H, S, D]).
        rows: optional 1-D array of flat row ids (b * H + h) * Sq + i.
        Returns (o, lse): without rows, o is [B, H, Sq, D] and lse [B, H, Sq]
        (head-major whatever the input layout); with rows, o is [n, D], lse [n].
        """
        lay = _LAYOUTS[layout] if isinstance(layout, str) else int(layout)
        qa, dt = _as_u16_or_f64(q)
        ka, dtk = _as_u16_or_f64(k)
        va, dtv = _as_u16_or_f64(v)
        if not (dt == dtk == dtv):
            raise ValueError("q, k, v must share one dtype")
        B, H, Sq, Sk, D = self._dims(qa, ka, lay)
        if scale is None:
            scale = 1.0 / np.sqrt(D)
        if rows is None:
            n = B * H * Sq
            rows_p = None
        else:
            rows = np.ascontiguousarray(rows, dtype=np.int64)
            n = rows.shape[0]
            rows_p = rows.ctypes.data
        o = np.empty((n, D), dtype=np.float64)
        lse = np.empty((n,), dtype=np.float64)
        rc = self._lib.oracle_attn_fwd_rows(
            qa.ctypes.data, ka.ctypes.data, va.ctypes.data, B, H, Sq, Sk, D, lay,
            int(bool(causal)), float(scale), dt, rows_p, n, o.ctypes.data, lse.ctypes.data,
            int(threads))
        if rc != 0:
            raise RuntimeError(f"oracle_attn_fwd_rows failed with code {rc}")
        if rows is None:
            return o.reshape(B, H, Sq, D), lse.reshape(B, H, Sq)
        return o, lse

    def fwd_varlen(self, q, k, v, cu_q, cu_k, *, causal=False, scale=None, rows=None, threads=0):
        """Attention forward over a packed batch of sequences of different lengths.

        q: [total_q, H, D], k, v: [total_k, H, D]; sequence b owns query rows
        cu_q[b] .. cu_q[b+1]-1 and key rows cu_k[b] .. cu_k[b+1]-1, and is the
        standard attention above on its own rows (causal: top-left aligned
        within the sequence).  This is the dense oracle applied to each
        sequence as a batch of one, in the packed [S, H, D] = BSND layout; it
        adds no arithmetic.  Returns (o [total_q, H, D], lse [H, total_q]),
        fp64; with rows (packed query row ids), o is [n, H, D] and lse [H, n]
        for those rows only.  A sequence with query rows but no keys raises
        ValueError (its softmax is over an empty set).
        """
        cu_q = [int(x) for x in cu_q]
        cu_k = [int(x) for x in cu_k]
        if len(cu_q) != len(cu_k) or len(cu_q) < 2:
            raise ValueError("cu_q and cu_k must hold the same number (B + 1 >= 2) of offsets")
        if q.ndim != 3 or k.ndim != 3:
            raise ValueError("q must be [total_q, H, D] and k, v [total_k, H, D]")
        total_q, H, D = q.shape
        want = np.arange(total_q) if rows is None else np.asarray(rows, dtype=np.int64)
        o = np.zeros((len(want), H, D), dtype=np.float64)
        lse = np.zeros((H, len(want)), dtype=np.float64)
        for b in range(len(cu_q) - 1):
            q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
            sel = np.nonzero((want >= q0) & (want < q1))[0]   # positions in the output
            if q1 == q0 or len(sel) == 0:
                continue
            if k1 == k0:
                raise ValueError(f"sequence {b} has query rows but no keys")
            local = want[sel] - q0
            flat = (np.arange(H)[:, None] * (q1 - q0) + local[None, :]).reshape(-1)   # (h * Sq_b + i)
            ob, lb = self.fwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], layout="BSND", causal=causal,
                              scale=scale, rows=flat, threads=threads)
            o[sel] = ob.reshape(H, len(sel), D).transpose(1, 0, 2)
            lse[:, sel] = lb.reshape(H, len(sel))
        return o, lse

    def weights(self, q, k, v, *, row, layout="BHSD", causal=False, scale=None):
        """Softmax weights (length Sk, zero where masked) of one flat query row."""
        lay = _LAYOUTS[layout] if isinstance(layout, str) else int(layout)
        qa, dt = _as_u16_or_f64(q)
        ka, _ = _as_u16_or_f64(k)
        va, _ = _as_u16_or_f64(v)
        B, H, Sq, Sk, D = self._dims(qa, ka, lay)
        if scale is None:
            scale = 1.0 / np.sqrt(D)
        w = np.empty((Sk,), dtype=np.float64)
        rc = self._lib.oracle_attn_weights(
            qa.ctypes.data, ka.ctypes.data, va.ctypes.data, B, H, Sq, Sk, D, lay,
            int(bool(causal)), float(scale), dt, int(row), w.ctypes.data)
        if rc != 0:
            raise RuntimeError(f"oracle_attn_weights failed with code {rc}")
        return w


_DEFAULT = None


def default():
    """The oracle built from attn_oracle.c without planted mistakes (built on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT


def build_planted(plant, out_dir):
    """Builds a planted-mistake variant into out_dir and returns an Oracle on it (tests only)."""
    out = os.path.join(out_dir, f"libattn_oracle_plant{plant}.so")
    _build.build(out=out, plant=plant, force=True)
    return Oracle(out)
