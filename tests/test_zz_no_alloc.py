"""cpattn_bwd_noalloc: the backward for callers that cannot allocate device
memory (allocator callbacks, processes whose memory pool belongs to another
framework, paths that cannot afford an allocation).  It must give what
cpattn_bwd gives with a caller-owned workspace, call after call, and refuse
shapes whose scratch would not fit the fixed array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own."""
import pytest
import torch

from long_sequence_context_b200.inputs import make_qkv
from tests.util import assert_close, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    from long_sequence_context_b200 import cpattn
    cpattn.set_path(0)
    return cpattn


@pytest.mark.parametrize("B,H,S,D,cp_size,causal,dtype", [
    (1, 4, 2048, 128, 4, True, torch.bfloat16),
    (1, 2, 1024, 64, 2, False, torch.bfloat16),
    (1, 2, 256, 64, 2, True, torch.float32),
])
def test_noalloc_matches_workspace_backward_twice(cp, B, H, S, D, cp_size, causal, dtype):
    q, k, v, dout = make_qkv(B, H, S, D, dtype, seed=900 + S + D)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = cp.fwd(qd, kd, vd, cp_size, causal)
    ref = cp.bwd(qd, kd, vd, o, lse, dod, cp_size, causal)
    assert cp.sync_status() == cp.OK
    # outputs preallocated, as a caller without an allocator would hold them
    outs = [torch.empty_like(qd) for _ in range(3)]
    for call in range(2):
        for t in outs:
            t.fill_(float("nan"))
        got = cp.bwd_noalloc(qd, kd, vd, o, lse, dod, cp_size, causal,
                             dq=outs[0], dk=outs[1], dv=outs[2])
        assert cp.sync_status() == cp.OK
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            assert_close(g.cpu(), np64(r.cpu()), dtype, f"call {call} {name}")
            # same kernels, same inputs, no atomics: the results are identical
            assert torch.equal(g, r), f"call {call} {name}: differs from cpattn_bwd"


def test_noalloc_rejects_shapes_beyond_the_scratch(cp):
    B, H, S, D = 2, 64, 131072, 128
    assert cp.bwd_workspace_bytes(B, H, S, D) > cp.NOALLOC_SCRATCH_BYTES
    t = torch.empty((1, 1, 1, 8), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(8, dtype=torch.float32, device="cuda")
    p = t.data_ptr()
    import ctypes
    vp = ctypes.c_void_p(p)
    st = cp.lib.cpattn_bwd_noalloc(vp, vp, vp, vp, ctypes.c_void_p(lse.data_ptr()), vp, vp, vp, vp,
                                   B, H, S, D, 8, 1, D ** -0.5, cp.BF16, None)
    assert st == cp.ERR_WORKSPACE
    st = cp.lib.cpattn_bwd_noalloc(vp, vp, vp, vp, ctypes.c_void_p(lse.data_ptr()), vp, vp, vp, vp,
                                   1, 1, 256, 96, 1, 1, 0.1, cp.BF16, None)
    assert st == cp.ERR_SHAPE
    assert cp.sync_status() == cp.OK
