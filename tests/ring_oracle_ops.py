"""Block attention and the merge of partial results from the fp64 oracle, in
the shape attention_forward_19_b200.ring.BlockwiseStep composes a ring step
from.  The ring tests run the ring's host logic with these steps on the CPU
(test_ring_cpu.py) and compare fa_fwd_ring_step with them (test_ring_gpu.py).
"""
import torch


class OracleOps:
    """Block attention and merge from the oracle, in fp64 on the CPU."""

    acc_dtype = torch.float64
    lse_dtype = torch.float64

    def __init__(self, layout, scale):
        from oracle import attn as oracle_attn
        self.layout, self.scale, self.orc = layout, scale, oracle_attn.default()
        self.calls = []

    def _to_layout(self, o_bhsd):
        t = torch.from_numpy(o_bhsd)
        return t.permute(0, 2, 1, 3) if self.layout == "BSND" else t

    def _head_major(self, t):
        return (t.permute(0, 2, 1, 3) if self.layout == "BSND" else t).double().numpy()

    def block(self, q, k, v, diagonal, o, lse):
        self.calls.append(bool(diagonal))
        oo, ll = self.orc.fwd(q, k, v, layout=self.layout, causal=bool(diagonal), scale=self.scale)
        o.copy_(self._to_layout(oo))
        lse.copy_(torch.from_numpy(ll))

    def merge(self, o_part, lse_part, o_acc, lse_acc, o_out, lse_out, accumulate, final):
        from oracle.merge import merge_partials
        parts = [self._head_major(o_part)]
        lses = [lse_part.double().numpy()]
        if accumulate:
            parts.insert(0, self._head_major(o_acc))
            lses.insert(0, lse_acc.double().numpy())
        o, l = merge_partials(parts, lses)
        dst_o, dst_l = (o_out, lse_out) if final else (o_acc, lse_acc)
        dst_o.copy_(self._to_layout(o))
        dst_l.copy_(torch.from_numpy(l))
