"""fp64 CPU oracle for the attention backward pass (gradients of the forward).

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only the test suite, the package smoke
check and the benchmark may import it.  It shares no code with the CUDA path.

What it computes.  The forward of the pages is O = softmax(S) V with
S = scale * Q K^T (+ the top-left causal mask) per (batch, head).  Its
backward recomputes the attention weights from Q, K and the row's
log-sum-exp instead of storing them (page "FlashAttention in ops-transformer
on Ascend NPU" (ai6s.net/6a0d3bfb), section "how FA runs on the NPU",
recomputation; page "catlass FlashAttention template tuning"
(hwcomputing.csdn.net/6a0d4681), section on the backward and its
`deterministic` flag).  Given dO = dL/dO, the chain rule through
O = P V and P = softmax(S) gives, row by row:

    P    = exp(S - LSE)                      (the forward's weights)
    dV   = P^T dO
    dP   = dO V^T
    D_i  = sum_j P_ij dP_ij  = sum_d dO_id O_id
    dS   = P * (dP - D)                      (softmax Jacobian, elementwise)
    dQ   = scale * dS K
    dK   = scale * dS^T Q

Masked entries have P = 0 and so dS = 0.  Inputs are the same 16-bit tensors
the GPU gets, decoded exactly to fp64 (torch's own upcast); every step is a
plain dense fp64 matrix product on one (batch, head) at a time, so the full
score matrix is materialised (fine for the test sizes).  The LSE and O used
here are computed by this module from the definition, never taken from the
GPU.
"""
import numpy as np
import torch


def _bhsd(x, layout):
    """[B, S, H, D] (BSND) or [B, H, S, D] (BHSD) -> fp64 numpy [B, H, S, D]."""
    t = torch.as_tensor(x).to(torch.float64)
    if layout == "BSND":
        t = t.permute(0, 2, 1, 3)
    return t.contiguous().numpy()


def _mask(Sq, Sk, causal):
    """True where key j is visible to query i (top-left aligned when causal)."""
    if not causal:
        return np.ones((Sq, Sk), dtype=bool)
    return np.arange(Sk)[None, :] <= np.arange(Sq)[:, None]


def attention_fwd_bwd(q, k, v, do, *, layout="BHSD", causal=False, scale=None):
    """Returns (o, lse, dq, dk, dv) in fp64, all head-major [B, H, S, D] (lse [B, H, Sq])."""
    qa, ka, va, doa = (_bhsd(t, layout) for t in (q, k, v, do))
    B, H, Sq, D = qa.shape
    Sk = ka.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    vis = _mask(Sq, Sk, causal)
    o = np.zeros((B, H, Sq, D))
    lse = np.zeros((B, H, Sq))
    dq = np.zeros((B, H, Sq, D))
    dk = np.zeros((B, H, Sk, D))
    dv = np.zeros((B, H, Sk, D))
    for b in range(B):
        for h in range(H):
            s = scale * (qa[b, h] @ ka[b, h].T)
            s = np.where(vis, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            p = e / l
            o[b, h] = p @ va[b, h]
            lse[b, h] = (m + np.log(l))[:, 0]
            dv[b, h] = p.T @ doa[b, h]
            dp = doa[b, h] @ va[b, h].T
            d_row = (doa[b, h] * o[b, h]).sum(axis=1, keepdims=True)
            ds = p * (dp - d_row)
            dq[b, h] = scale * (ds @ ka[b, h])
            dk[b, h] = scale * (ds.T @ qa[b, h])
    return o, lse, dq, dk, dv


def softmax_backward_rows(dp, p):
    """dS for given dP and P row by row, as the explicit Jacobian product
    dS_i = J_i dP_i with J_i = diag(P_i) - P_i P_i^T (a pin for the closed form
    P * (dP - rowsum(P * dP)) used above)."""
    out = np.zeros_like(p)
    for i in range(p.shape[0]):
        jac = np.diag(p[i]) - np.outer(p[i], p[i])
        out[i] = jac @ dp[i]
    return out
