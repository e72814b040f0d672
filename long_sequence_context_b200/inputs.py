"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws random tensors.  It is
the one piece shared by the CUDA path's callers and the oracle's callers, so
both see exactly the same (dtype-rounded) values.

Recipe: one CPU ``torch.Generator`` per workload, seeded with ``seed``; draw
fp32 standard normals in the order q, k, v, dO (each of shape [B, H, S, D]),
multiply q, k, v by ``qkv_scale``, then round to the workload dtype.
"""
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    cp_size: int
    causal: bool
    dtype: str  # "bf16" or "fp32"
    backward: bool
    qkv_scale: float = 1.0
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def scale(self) -> float:
        return 1.0 / (self.D ** 0.5)

    def flops_fwd(self) -> float:
        """Algorithmic forward FLOPs: 4*B*H*S^2*D, half of it when causal."""
        dense = 4.0 * self.B * self.H * self.S * self.S * self.D
        return dense / 2 if self.causal else dense

    def flops_bwd(self) -> float:
        """Backward = 2.5 x forward (five S^2*D matmuls against two)."""
        return 2.5 * self.flops_fwd()

    def describe(self) -> str:
        kind = "causal" if self.causal else "non-causal"
        split = "zigzag" if self.causal else "contiguous"
        return (f"{kind} attention B={self.B},H={self.H},S={self.S},D={self.D}, "
                f"cp_size={self.cp_size} {split}, {self.dtype}")


# The five workloads: the fp32 small case the oracle covers in full, then the
# bf16 cases.  Seeds are 1000 + position.
WORKLOADS = {
    "causal_b1h2s256d64_cp2_fp32": Workload("causal_b1h2s256d64_cp2_fp32", 1, 2, 256, 64, 2, True,
                                            "fp32", False, 1.0, 1000),
    "causal_b1h16s8192d128_cp4_bf16": Workload("causal_b1h16s8192d128_cp4_bf16", 1, 16, 8192, 128, 4,
                                               True, "bf16", False, 1.0, 1001),
    "causal_b1h32s32768d128_cp8_bf16": Workload("causal_b1h32s32768d128_cp8_bf16", 1, 32, 32768, 128,
                                                8, True, "bf16", True, 1.0, 1002),
    "noncausal_b2h32s16384d128_cp2_bf16": Workload("noncausal_b2h32s16384d128_cp2_bf16", 2, 32, 16384,
                                                   128, 2, False, "bf16", True, 1.0, 1003),
    "causal_b1h8s131072d128_cp16_bf16": Workload("causal_b1h8s131072d128_cp16_bf16", 1, 8, 131072,
                                                 128, 16, True, "bf16", True, 0.5, 1004),
}
WORKLOAD_ORDER = list(WORKLOADS)


def make_qkv(B, H, S, D, dtype=torch.bfloat16, seed=0, qkv_scale=1.0, with_dout=True):
    """Return CPU tensors (q, k, v, dout) of shape [B, H, S, D] in ``dtype``.

    dout is None when ``with_dout`` is False (it is still drawn, after v, so the
    q, k, v values do not depend on the flag)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, S, D)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    dout = torch.randn(shape, generator=g, dtype=torch.float32) if with_dout else None
    if qkv_scale != 1.0:
        q.mul_(qkv_scale)
        k.mul_(qkv_scale)
        v.mul_(qkv_scale)
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    if dout is not None:
        dout = dout.to(dtype)
    return q, k, v, dout


def workload_inputs(w: Workload, with_dout=None):
    if with_dout is None:
        with_dout = w.backward
    return make_qkv(w.B, w.H, w.S, w.D, w.torch_dtype, w.seed, w.qkv_scale, with_dout)


def make_layer_inputs(B, S, E, seed=0, dtype=torch.bfloat16):
    """CPU tensors for the attention layer: x [B,S,E], w_qkv [3E,E], b_qkv [3E],
    w_o [E,E], b_o [E], dy [B,S,E].  x and dy ~ N(0,1); weights and biases
    ~ U(-1/sqrt(E), 1/sqrt(E)) (the range nn.Linear initialises them in), drawn
    in that order from one seeded generator, then rounded to ``dtype``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    bound = E ** -0.5

    def uni(*shape):
        return (torch.rand(shape, generator=g, dtype=torch.float32) * 2 - 1) * bound

    x = torch.randn((B, S, E), generator=g, dtype=torch.float32)
    w_qkv, b_qkv, w_o, b_o = uni(3 * E, E), uni(3 * E), uni(E, E), uni(E)
    dy = torch.randn((B, S, E), generator=g, dtype=torch.float32)
    return tuple(t.to(dtype) for t in (x, w_qkv, b_qkv, w_o, b_o, dy))


def flops_layer(B, S, E, H, causal=True):
    """Algorithmic FLOPs of one layer (forward, backward): projections
    8*B*S*E^2 forward and twice that backward, plus the attention's counts."""
    D = E // H
    att = 4.0 * B * H * S * S * D * (0.5 if causal else 1.0)
    proj = 8.0 * B * S * E * E
    return proj + att, 2 * proj + 2.5 * att
