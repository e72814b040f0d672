"""A CPU backend for the ring schedules of long_sequence_context_b200/ring.py
built on the fp64 oracle: lets the multi-rank schedule (which chunks meet at
which step, the merges, the dK/dV sums travelling with their K/V) be checked
on CPU ranks against the oracle's attention of the whole sequence.

TEST INFRASTRUCTURE: used by tests only.

Block backward: the gradient terms of one (q chunk, kv chunk) block given the
rows' final O and LSE -- P = exp(scale q.k - LSE) (masked j <= i on a DIAG
block), dV = P^T dO, dP = dO V^T, delta = rowsum(dO * O), dS = P (dP - delta),
dQ = scale dS K, dK = scale dS^T Q ("Megatron-LM source analysis: Context
Parallel", section 2: the backward mirrors the forward block by block).
"""
import numpy as np
import torch

from oracle import oracle as orc


class OracleBlocks:
    def __init__(self, scale):
        self.scale = scale

    def new_acc(self, q):
        return (torch.zeros(q.shape, dtype=torch.float64),
                torch.full(q.shape[:-1], float("-inf"), dtype=torch.float64))

    def fwd(self, q, k, v, diag):
        o, lse = orc.attn_fwd(q.numpy(), k.numpy(), v.numpy(), diag, self.scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(self, o_acc, lse_acc, o_part, lse_part):
        B, H, S, D = o_acc.shape
        o, l = orc.merge(o_acc.numpy().reshape(-1, D), lse_acc.numpy().reshape(-1),
                         o_part.numpy().reshape(-1, D), lse_part.numpy().reshape(-1))
        o_acc.copy_(torch.from_numpy(o.reshape(B, H, S, D)))
        lse_acc.copy_(torch.from_numpy(l.reshape(B, H, S)))

    def finalize(self, o_acc, dtype):
        return o_acc.clone()

    def zeros_f32(self, like):
        return torch.zeros(like.shape, dtype=torch.float64)

    def bwd_into(self, q, k, v, o, lse, do, diag, dq_acc, dk_acc, dv_acc):
        dq, dk, dv = self.bwd(q, k, v, o, lse, do, diag)
        dq_acc += dq
        dk_acc += dk
        dv_acc += dv

    def bwd(self, q, k, v, o, lse, do, diag):
        s = self.scale * torch.einsum("bhid,bhjd->bhij", q, k)
        p = torch.exp(s - lse[..., None])
        if diag:
            n = q.shape[2]
            p = p * torch.tril(torch.ones(n, n, dtype=p.dtype))
        dv = torch.einsum("bhij,bhid->bhjd", p, do)
        dp = torch.einsum("bhid,bhjd->bhij", do, v)
        delta = (do * o).sum(-1, keepdim=True)
        ds = p * (dp - delta)
        dq = self.scale * torch.einsum("bhij,bhjd->bhid", ds, k)
        dk = self.scale * torch.einsum("bhij,bhid->bhjd", ds, q)
        return dq, dk, dv

    def add(self, acc, x):
        acc += x

    def cast(self, acc, dtype):
        return acc.clone()
