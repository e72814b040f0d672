"""GPU parity of the recompute backward against the fp64 oracle."""
import numpy as np
import pytest
import torch

from long_sequence_context_b200.inputs import WORKLOADS, make_qkv, workload_inputs
from oracle import oracle as orc
from tests.util import assert_close, np64, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    from long_sequence_context_b200 import cpattn
    cpattn.set_path(0)
    return cpattn


def run_fwd_bwd(cp, q, k, v, dout, cp_size, causal):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = cp.fwd(qd, kd, vd, cp_size, causal)
    dq, dk, dv = cp.bwd(qd, kd, vd, o, lse, dod, cp_size, causal)
    assert cp.sync_status() == cp.OK
    return dq.cpu(), dk.cpu(), dv.cpu()


SMALL = [
    (1, 2, 1024, 128, 2, True, torch.bfloat16),
    (1, 2, 1024, 64, 4, True, torch.bfloat16),
    (2, 1, 768, 128, 1, True, torch.bfloat16),
    (1, 2, 1024, 128, 2, False, torch.bfloat16),
    (1, 2, 256, 64, 2, True, torch.float32),
    (1, 1, 512, 128, 4, False, torch.float32),
]


@pytest.mark.parametrize("B,H,S,D,cp_size,causal,dtype", SMALL)
def test_bwd_vs_oracle(cp, B, H, S, D, cp_size, causal, dtype):
    q, k, v, dout = make_qkv(B, H, S, D, dtype, seed=100 + S + D)
    dq, dk, dv = run_fwd_bwd(cp, q, k, v, dout, cp_size, causal)
    rq, rk, rv = orc.attn_bwd(np64(q), np64(k), np64(v), np64(dout), causal, D ** -0.5)
    assert_close(dq, rq, dtype, "dQ")
    assert_close(dk, rk, dtype, "dK")
    assert_close(dv, rv, dtype, "dV")


@pytest.mark.parametrize("B,H,S,D,cp_size,causal,dtype", SMALL[:2])
def test_bwd_cuda_cores_vs_oracle(cp, B, H, S, D, cp_size, causal, dtype):
    q, k, v, dout = make_qkv(B, H, S, D, dtype, seed=200 + S)
    prev = cp.set_path(1)
    try:
        dq, dk, dv = run_fwd_bwd(cp, q, k, v, dout, cp_size, causal)
    finally:
        cp.set_path(prev)
    rq, rk, rv = orc.attn_bwd(np64(q), np64(k), np64(v), np64(dout), causal, D ** -0.5)
    assert_close(dq, rq, dtype, "dQ")
    assert_close(dk, rk, dtype, "dK")
    assert_close(dv, rv, dtype, "dV")


FULL = ["causal_b1h32s32768d128_cp8_bf16", "noncausal_b2h32s16384d128_cp2_bf16",
        "causal_b1h8s131072d128_cp16_bf16"]


@pytest.mark.parametrize("name", FULL)
def test_bwd_full_workload_sampled(cp, name):
    w = WORKLOADS[name]
    q, k, v, dout = workload_inputs(w)
    dq, dk, dv = run_fwd_bwd(cp, q, k, v, dout, w.cp_size, w.causal)
    n_chunks = 2 * w.cp_size if w.causal else w.cp_size
    # dQ on sampled rows of two heads; dK / dV on the last 32 key columns of one
    # head (rows that see them are few when causal; all rows otherwise)
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        args = [np64(t[sl]) for t in (q, k, v, dout)]
        rows = sample_rows(w.S, n_chunks, 48, seed=h)
        rq = orc.attn_bwd_dq_rows(*args, w.causal, w.scale, 0, 0, rows)
        assert_close(dq[b, h, rows], rq, torch.bfloat16, f"{name} dQ rows b{b} h{h}")
    b, h = 0, w.H // 2
    sl = (slice(b, b + 1), slice(h, h + 1))
    args = [np64(t[sl]) for t in (q, k, v, dout)]
    cols = np.arange(w.S - 32, w.S) if w.causal else np.array([0, 1, w.S // 2, w.S - 1])
    rk, rv = orc.attn_bwd_kv_cols(*args, w.causal, w.scale, 0, 0, cols)
    assert_close(dk[b, h, cols], rk, torch.bfloat16, f"{name} dK cols")
    assert_close(dv[b, h, cols], rv, torch.bfloat16, f"{name} dV cols")
    # identities that hold at any size: sum_j dK_j = 0, sum_j dV_j = sum_i dO_i
    dk_sum = np64(dk).sum(axis=2)
    dv_sum = np64(dv).sum(axis=2)
    do_sum = np64(dout).sum(axis=2)
    dk_abs = np.abs(np64(dk)).sum(axis=2)
    assert np.all(np.abs(dk_sum) <= 1e-2 * dk_abs + 1e-2), float(np.max(np.abs(dk_sum)))
    assert np.max(np.abs(dv_sum - do_sum)) <= 1e-2 * w.S ** 0.5, float(np.max(np.abs(dv_sum - do_sum)))
