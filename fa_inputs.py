"""Seeded synthetic inputs for the attention forward pass.

This module is shared by the tests, the smoke check and the benchmark, and it
is the only thing the CUDA path's callers and the oracle's callers share.  It
holds no attention arithmetic: it only names the workloads and draws q, k, v.

Recipe: torch.Generator('cpu').manual_seed(seed); q, k, v are drawn in that
order as float32 standard normals of the layout's shape, multiplied by the
workload's standard deviation, and rounded to nearest into fp16 / bf16.  The
seed 42 is the one the accuracy check on the pages uses (page "ops-transformer
FlashAttention on Atlas 800", section "accuracy check"); workload n uses 42 + n.
"""
import math
from dataclasses import dataclass, replace

import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str          # "fp16" | "bf16"
    layout: str         # "BSND" ([B, S, H, D]) | "BHSD" ([B, H, S, D])
    B: int
    H: int
    Sq: int
    Sk: int
    D: int
    causal: bool
    scale: float
    qk_std: float = 1.0
    v_std: float = 1.0
    seed: int = 42
    # Structured inputs (both empty for the plain recipe).  If q_lead is given,
    # element 0 of query row i of every (batch, head) is set to
    # q_lead[i % len(q_lead)]; if k_lead is given, element 0 of key j is set to
    # k_lead[(j // 128) % len(k_lead)] (one value per block of 128 keys).  The
    # values replace the drawn ones before the rounding to the dtype.
    q_lead: tuple = ()
    k_lead: tuple = ()

    def q_shape(self):
        return (self.B, self.Sq, self.H, self.D) if self.layout == "BSND" else (self.B, self.H, self.Sq, self.D)

    def kv_shape(self):
        return (self.B, self.Sk, self.H, self.D) if self.layout == "BSND" else (self.B, self.H, self.Sk, self.D)

    def flops(self):
        """Attention-forward flops 4*B*H*Sq*Sk*D, halved when causal (the metric's convention)."""
        f = 4.0 * self.B * self.H * self.Sq * self.Sk * self.D
        return f / 2 if self.causal else f

    def with_(self, **kw):
        return replace(self, **kw)


# The five workloads the measurements are quoted on.
WORKLOADS = {
    "fp16_bsnd_b1_h2_s512_d64": Workload(
        "fp16_bsnd_b1_h2_s512_d64", "fp16", "BSND", 1, 2, 512, 512, 64, False, 1.0 / 8, seed=42),
    "fp16_bhsd_b8_h32_s4096_d128_causal": Workload(
        "fp16_bhsd_b8_h32_s4096_d128_causal", "fp16", "BHSD", 8, 32, 4096, 4096, 128, True,
        1.0 / math.sqrt(128), seed=43),
    "bf16_bhsd_b2_h40_s8192_d128_causal": Workload(
        "bf16_bhsd_b2_h40_s8192_d128_causal", "bf16", "BHSD", 2, 40, 8192, 8192, 128, True,
        1.0 / math.sqrt(128), seed=44),
    "bf16_bhsd_b1_h8_s65536_d128_causal": Workload(
        "bf16_bhsd_b1_h8_s65536_d128_causal", "bf16", "BHSD", 1, 8, 65536, 65536, 128, True,
        1.0 / math.sqrt(128), seed=45),
    "bf16_bsnd_b1_h32_s16000_d128_qk3": Workload(
        "bf16_bsnd_b1_h32_s16000_d128_qk3", "bf16", "BSND", 1, 32, 16000, 16000, 128, False,
        1.0 / math.sqrt(128), qk_std=3.0, seed=46),
}
WORKLOAD_ORDER = list(WORKLOADS)
BENCH_WORKLOAD = "bf16_bhsd_b2_h40_s8192_d128_causal"


def make_qkv(w: Workload, device="cpu"):
    """Draws q, k, v for workload w (see the module docstring for the recipe)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    dt = DTYPES[w.dtype]
    q = torch.randn(w.q_shape(), generator=g, dtype=torch.float32) * w.qk_std
    k = torch.randn(w.kv_shape(), generator=g, dtype=torch.float32) * w.qk_std
    v = (torch.randn(w.kv_shape(), generator=g, dtype=torch.float32) * w.v_std).to(dt)
    seq_dim = 1 if w.layout == "BSND" else 2
    if w.q_lead:
        lead = torch.tensor(w.q_lead, dtype=torch.float32)
        vals = lead[torch.arange(w.Sq) % len(w.q_lead)]
        shape = [1, 1, 1]
        shape[seq_dim] = w.Sq
        q[..., 0] = vals.reshape(shape)
    if w.k_lead:
        lead = torch.tensor(w.k_lead, dtype=torch.float32)
        vals = lead[(torch.arange(w.Sk) // 128) % len(w.k_lead)]
        shape = [1, 1, 1]
        shape[seq_dim] = w.Sk
        k[..., 0] = vals.reshape(shape)
    q, k = q.to(dt), k.to(dt)
    if device != "cpu":
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


def sample_rows(w: Workload, per_head_first=64, per_head_last=64, stride=97, max_rows=None):
    """Flat row ids (b * H + h) * Sq + i for a stratified sample of every head.

    Each head contributes its first rows, every stride-th row and its last rows,
    so that the first and last query tiles, the diagonal and the ragged tail
    are all represented.
    """
    rows = []
    for bh in range(w.B * w.H):
        picked = set(range(min(per_head_first, w.Sq)))
        picked.update(range(0, w.Sq, stride))
        picked.update(range(max(0, w.Sq - per_head_last), w.Sq))
        rows.extend(bh * w.Sq + i for i in sorted(picked))
    if max_rows is not None and len(rows) > max_rows:
        step = len(rows) / max_rows
        rows = [rows[int(j * step)] for j in range(max_rows)]
    return rows


# ----------------------------------------------------------------------------- packed variable-length batches

@dataclass(frozen=True)
class VarlenWorkload:
    """A packed batch of sequences: q [total_q, H, D], k / v [total_k, H, D].

    Lengths: `lengths` if given, else `nseq` query lengths drawn uniformly from
    [min_len, max_len] with the workload's seed (key length = query length).
    Values as for Workload: fp32 standard normals times the std, rounded."""
    name: str
    dtype: str
    H: int
    D: int
    causal: bool
    scale: float
    nseq: int = 0
    min_len: int = 1
    max_len: int = 1
    lengths: tuple = ()     # ((Sq, Sk), ...) overrides the drawn lengths
    qk_std: float = 1.0
    v_std: float = 1.0
    seed: int = 47

    def seq_lengths(self):
        if self.lengths:
            return [tuple(x) for x in self.lengths]
        g = torch.Generator(device="cpu")
        g.manual_seed(int(self.seed) + 1000)
        n = torch.randint(self.min_len, self.max_len + 1, (self.nseq,), generator=g).tolist()
        return [(a, a) for a in n]

    def offsets(self):
        """cu_seqlens_q, cu_seqlens_k as int32 CPU tensors of nseq + 1 offsets."""
        ls = self.seq_lengths()
        cq = [0]
        ck = [0]
        for a, b in ls:
            cq.append(cq[-1] + a)
            ck.append(ck[-1] + b)
        return torch.tensor(cq, dtype=torch.int32), torch.tensor(ck, dtype=torch.int32)

    def flops(self):
        """Sum over sequences of 4*H*Sq*Sk*D, halved when causal (the dense metric's convention)."""
        f = sum(4.0 * self.H * a * b * self.D for a, b in self.seq_lengths())
        return f / 2 if self.causal else f


VARLEN_WORKLOADS = {
    "bf16_varlen_n16_h32_d128_causal": VarlenWorkload(
        "bf16_varlen_n16_h32_d128_causal", "bf16", 32, 128, True, 1.0 / math.sqrt(128),
        nseq=16, min_len=128, max_len=8192, seed=47),
}


def make_varlen_qkv(w: VarlenWorkload, device="cpu"):
    """Draws packed q, k, v (recipe as make_qkv) and returns (q, k, v, cu_q, cu_k)."""
    cu_q, cu_k = w.offsets()
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    dt = DTYPES[w.dtype]
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = (torch.randn((tq, w.H, w.D), generator=g, dtype=torch.float32) * w.qk_std).to(dt)
    k = (torch.randn((tk, w.H, w.D), generator=g, dtype=torch.float32) * w.qk_std).to(dt)
    v = (torch.randn((tk, w.H, w.D), generator=g, dtype=torch.float32) * w.v_std).to(dt)
    if device != "cpu":
        q, k, v, cu_q, cu_k = (t.to(device) for t in (q, k, v, cu_q, cu_k))
    return q, k, v, cu_q, cu_k


def make_dout(w: Workload, device="cpu"):
    """Draws the output gradient dO for workload w: float32 standard normals of
    q's shape from seed + 500, rounded to the dtype (q, k, v are unchanged)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed) + 500)
    do = torch.randn(w.q_shape(), generator=g, dtype=torch.float32).to(DTYPES[w.dtype])
    return do.to(device) if device != "cpu" else do
