"""The attention output projection in fp64: Y = O W^T over all heads of a token.

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only the test suite, the package smoke
check and the benchmark may import it.  It shares no code with the CUDA path.

Page "catlass FlashAttention template tuning" (hwcomputing.csdn.net/6a0d4681),
section on graph fusion: the fused operator FusedAttnProj is FlashAttention
followed by the output MatMul.  Reading taken (the page names the operators,
not their shapes): the MatMul is the usual output projection of multi-head
attention, every token's head outputs concatenated head after head,
    Y[b, s, n] = sum_{h, d} O[b, s, h, d] * W[n, h * D + d],
with W in a linear layer's [E, H * D] layout.  The contraction is one numpy
matmul on the exact fp64 decoding of the 16-bit inputs.
"""
import torch


def _f64(x):
    return torch.as_tensor(x).detach().cpu().to(torch.float64).numpy()


def out_proj(o, w, layout="BSND"):
    """o: [B, S, H, D] (BSND) or [B, H, S, D] (BHSD); w: [E, H * D].  Returns Y [B, S, E] in fp64."""
    oa = _f64(o)
    if layout == "BHSD":
        oa = oa.transpose(0, 2, 1, 3)
    elif layout != "BSND":
        raise ValueError(f"layout must be 'BSND' or 'BHSD', not {layout!r}")
    B, S, H, D = oa.shape
    wa = _f64(w)
    if wa.shape[1] != H * D:
        raise ValueError(f"w has {wa.shape[1]} inputs, o has H * D = {H * D}")
    return oa.reshape(B, S, H * D) @ wa.T


def attention_out_proj(q, k, v, w, *, layout="BSND", causal=False, scale=None, orc=None):
    """The fused operator's result: attention from the fp64 oracle, then out_proj.  Returns (Y, O, LSE)
    with O head-major [B, H, S, D] and LSE [B, H, S]."""
    from . import attn as oracle_attn
    orc = oracle_attn.default() if orc is None else orc
    o, lse = orc.fwd(q, k, v, layout=layout, causal=causal, scale=scale)
    return out_proj(o, w, layout="BHSD"), o, lse
