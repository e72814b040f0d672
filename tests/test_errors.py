"""Failure detection on the GPU without faulting it: a bounded in-kernel wait is
made to run out (the forward's TMA warp is told to skip one K/V load), the
kernel gives up cleanly, the host reads CPATTN_ERR_TIMEOUT from the device
error word, and the next call on the same context is correct again."""
import numpy as np
import pytest
import torch

from long_sequence_context_b200.inputs import make_qkv
from oracle import oracle as orc
from tests.util import assert_close, assert_lse_close, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    from long_sequence_context_b200 import cpattn
    cpattn.set_path(0)
    return cpattn


def test_skipped_load_times_out_and_context_survives(cp):
    B, H, S, D, N = 1, 2, 1024, 128, 2
    q, k, v, _ = make_qkv(B, H, S, D, torch.bfloat16, seed=77, with_dout=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    assert cp.sync_status() == cp.OK
    cp.debug_stall(1)
    try:
        cp.fwd(qd, kd, vd, N, True)
        st = cp.sync_status()
    finally:
        cp.debug_stall(0)
    assert st == cp.ERR_TIMEOUT, cp.status_str(st)
    assert cp.sync_status() == cp.OK  # the error word was cleared
    o, lse = cp.fwd(qd, kd, vd, N, True)
    assert cp.sync_status() == cp.OK
    o_ref, lse_ref = orc.attn_fwd(np64(q), np64(k), np64(v), True, D ** -0.5)
    assert_close(o.cpu(), o_ref, torch.bfloat16, "O after recovery")
    assert_lse_close(lse.cpu(), lse_ref)


def test_bad_arguments_do_not_launch(cp):
    n0 = cp.launch_count()
    q = torch.zeros((1, 1, 102, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cp.CpattnError) as e:   # 102 rows are not 4 whole chunks
        cp.fwd(q, q, q, 2, True)
    assert e.value.status == cp.ERR_SHAPE
    q = torch.zeros((1, 1, 256, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(TypeError):
        cp.fwd(q, q, q, 2, True)
    assert cp.launch_count() == n0
