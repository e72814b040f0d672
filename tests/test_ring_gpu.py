"""The multi-rank ring (long_sequence_context_b200/ring.py) with the library's
kernels as the block backend, N virtual ranks driven in one process
(loopback: the ranks' exchanges are delivered in memory, one rank after
another -- no kernel waits on another rank).  Every rank's O, LSE, dQ, dK, dV
against the fp64 oracle of the whole sequence (bf16 tolerances) and against
the one-call cpattn_fwd / cpattn_bwd of the whole sequence."""
import numpy as np
import pytest
import torch

from long_sequence_context_b200 import cpattn as cp
from long_sequence_context_b200 import ring
from long_sequence_context_b200.inputs import make_qkv
from oracle import oracle as orc
from tests.util import assert_close, assert_lse_close, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,causal,S", [
    (2, True, 1024),    # chunks of 256: tcgen05 blocks
    (4, True, 1024),    # chunks of 128: DIAG blocks on the CUDA-core kernels
    (3, True, 1536),    # an odd ring: the dK/dV sums make three hops
    (2, False, 1024),
])
def test_loopback_ring_with_library_blocks(world, causal, S):
    B, H, D = 1, 2, 128
    scale = D ** -0.5
    q, k, v, do = make_qkv(B, H, S, D, torch.bfloat16, seed=31)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    be = ring.CudaBlocks(scale)
    loc = lambda x, r: ring.local_chunks(x, r, world, causal)
    fwd = ring.run_loopback([ring.fwd_schedule(r, world, loc(qd, r), loc(kd, r), loc(vd, r), causal, be)
                             for r in range(world)])
    bwd = ring.run_loopback([ring.bwd_schedule(r, world, loc(qd, r), loc(kd, r), loc(vd, r),
                                               [a for a, _ in fwd[r]], [b for _, b in fwd[r]],
                                               loc(dod, r), causal, be) for r in range(world)])
    cp.check_device_status()
    # the whole sequence: fp64 oracle and the one-call library path
    f = lambda t: np64(t)
    ro, rl = orc.attn_fwd(f(q), f(k), f(v), causal, scale)
    rdq, rdk, rdv = orc.attn_bwd(f(q), f(k), f(v), f(do), causal, scale)
    o1, l1 = cp.fwd(qd, kd, vd, world, causal, scale)
    g1 = cp.bwd(qd, kd, vd, o1, l1, dod, world, causal, scale)
    ref = {"o": torch.from_numpy(ro), "lse": torch.from_numpy(rl), "dq": torch.from_numpy(rdq),
           "dk": torch.from_numpy(rdk), "dv": torch.from_numpy(rdv)}
    one = {"o": o1, "lse": l1, "dq": g1[0], "dk": g1[1], "dv": g1[2]}
    for r in range(world):
        got = {"o": [a for a, _ in fwd[r]], "lse": [b for _, b in fwd[r]],
               "dq": bwd[r][0], "dk": bwd[r][1], "dv": bwd[r][2]}
        for name, chunks in got.items():
            want = ring.local_chunks(ref[name], r, world, causal)
            same = ring.local_chunks(one[name], r, world, causal)
            for g, w, s in zip(chunks, want, same):
                if name == "lse":
                    assert_lse_close(g, w.numpy())
                    assert_lse_close(g, np64(s))
                elif name == "o":  # fp32 block partials: one rounding
                    assert_close(g, w.numpy(), dtype=torch.bfloat16)
                    assert_close(g, np64(s), dtype=torch.bfloat16)
                else:  # fp32 sums of the block terms (cpattn_bwd_accumulate), one rounding
                    assert_close(g, w.numpy(), dtype=torch.bfloat16)
                    assert_close(g, np64(s), dtype=torch.bfloat16)


def test_accumulate_adds_into_fp32():
    import ctypes
    acc = torch.randn(1000, device="cuda")
    x = torch.randn(1000, device="cuda").to(torch.bfloat16)
    want = acc.double() + x.double()
    cp.accumulate_(acc, x)
    torch.cuda.synchronize()
    assert (acc.double() - want).abs().max().item() <= 1e-6
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert cp.lib.cpattn_accumulate(p(acc), p(x), 6, cp.BF16, None) == cp.ERR_SHAPE  # n % 4 != 0
