"""GPU parity of the ring forward against the fp64 oracle.

Every call goes through the C ABI (via the ctypes binding).  Small shapes are
compared element by element; the full workloads on sampled rows of every
head plus one whole head."""
import numpy as np
import pytest
import torch

from long_sequence_context_b200.inputs import WORKLOADS, make_qkv, workload_inputs
from oracle import oracle as orc
from tests.util import assert_close, assert_lse_close, np64, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    from long_sequence_context_b200 import cpattn
    cpattn.set_path(0)
    return cpattn


def run_fwd(cp, q, k, v, cp_size, causal, scale=None):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = cp.fwd(qd, kd, vd, cp_size, causal, scale)
    assert cp.sync_status() == cp.OK
    return o.cpu(), lse.cpu()


def oracle_fwd(q, k, v, causal, scale, heads=None):
    return orc.attn_fwd(np64(q), np64(k), np64(v), causal, scale, heads)


# (B, H, S, D, cp_size, causal): several tiles, odd tile counts per chunk
# (a lone last Q tile), chunk of exactly one tile, both head sizes
SMALL = [
    (1, 2, 1024, 128, 2, True),
    (1, 2, 1024, 64, 4, True),
    (2, 2, 768, 128, 1, True),
    (1, 3, 2048, 128, 8, True),
    (1, 2, 1536, 64, 2, True),
    (1, 2, 1024, 128, 2, False),
    (2, 1, 384, 64, 3, False),
    (1, 1, 128, 128, 1, False),
    (1, 1, 256, 128, 1, True),
]


@pytest.mark.parametrize("B,H,S,D,cp_size,causal", SMALL)
def test_fwd_bf16_tensor_cores_vs_oracle(cp, B, H, S, D, cp_size, causal):
    q, k, v, _ = make_qkv(B, H, S, D, torch.bfloat16, seed=S + D + cp_size, with_dout=False)
    o, lse = run_fwd(cp, q, k, v, cp_size, causal)
    assert cp.last_path() == 0, "tcgen05 path expected"
    o_ref, lse_ref = oracle_fwd(q, k, v, causal, D ** -0.5)
    assert_close(o, o_ref, torch.bfloat16, "O")
    assert_lse_close(lse, lse_ref)


@pytest.mark.parametrize("B,H,S,D,cp_size,causal", SMALL[:5] + [(1, 2, 320, 64, 2, True)])
def test_fwd_bf16_cuda_cores_vs_oracle(cp, B, H, S, D, cp_size, causal):
    q, k, v, _ = make_qkv(B, H, S, D, torch.bfloat16, seed=7 + S, with_dout=False)
    prev = cp.set_path(1)
    try:
        o, lse = run_fwd(cp, q, k, v, cp_size, causal)
        assert cp.last_path() == 1
    finally:
        cp.set_path(prev)
    o_ref, lse_ref = oracle_fwd(q, k, v, causal, D ** -0.5)
    assert_close(o, o_ref, torch.bfloat16, "O")
    assert_lse_close(lse, lse_ref)


def test_fwd_fp32_small_workload(cp):
    w = WORKLOADS["causal_b1h2s256d64_cp2_fp32"]
    q, k, v, _ = workload_inputs(w)
    o, lse = run_fwd(cp, q, k, v, w.cp_size, w.causal)
    o_ref, lse_ref = oracle_fwd(q, k, v, w.causal, w.scale)
    assert_close(o, o_ref, torch.float32, "O")
    assert_lse_close(lse, lse_ref)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_steps_and_merge_equal_fused(cp, dtype):
    B, H, S, D, N = 1, 2, 1024, 128, 4
    q, k, v, _ = make_qkv(B, H, S, D, dtype, seed=11, with_dout=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o_acc = torch.zeros((B, H, S, D), dtype=torch.float32, device="cuda")
    lse_acc = torch.full((B, H, S), float("-inf"), dtype=torch.float32, device="cuda")
    for t in range(N):
        op, lp = cp.fwd_step(qd, kd, vd, N, t, True)
        op_ref, lp_ref = orc.ring_step(np64(q), np64(k), np64(v), N, True, D ** -0.5, t)
        assert_close(op.cpu(), op_ref, torch.float32 if dtype == torch.float32 else torch.bfloat16,
                     f"step {t} O")
        assert_lse_close(lp.cpu(), lp_ref, f"step {t} LSE")
        cp.merge_(o_acc, lse_acc, op, lp)
    o = cp.finalize(o_acc, dtype)
    assert cp.sync_status() == cp.OK
    o_ref, lse_ref = oracle_fwd(q, k, v, True, D ** -0.5)
    assert_close(o.cpu(), o_ref, dtype, "merged O")
    assert_lse_close(lse_acc.cpu(), lse_ref)
    o_f, lse_f = cp.fwd(qd, kd, vd, N, True)
    assert_close(o.cpu(), np64(o_f), dtype, "merged vs fused")


def test_fwd_agrees_across_cp_size(cp):
    B, H, S, D = 1, 2, 4096, 128
    q, k, v, _ = make_qkv(B, H, S, D, torch.bfloat16, seed=21, with_dout=False)
    o_ref, lse_ref = oracle_fwd(q, k, v, True, D ** -0.5)
    outs = []
    for n in (1, 2, 4, 8, 16):
        o, lse = run_fwd(cp, q, k, v, n, True)
        assert_close(o, o_ref, torch.bfloat16, f"cp={n}")
        assert_lse_close(lse, lse_ref, f"cp={n} lse")
        outs.append(np64(o))
    for x in outs[1:]:
        assert np.max(np.abs(x - outs[0])) <= 2e-2


def test_fwd_is_deterministic(cp):
    q, k, v, _ = make_qkv(1, 4, 2048, 128, torch.bfloat16, seed=31, with_dout=False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = cp.fwd(qd, kd, vd, 4, True)
    o2, l2 = cp.fwd(qd, kd, vd, 4, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_large_scores_rescale_path(cp):
    # scores with a wide range force the running-max rescale of O in TMEM
    B, H, S, D = 1, 2, 2048, 128
    q, k, v, _ = make_qkv(B, H, S, D, torch.float32, seed=41, with_dout=False)
    ramp = torch.linspace(0.2, 6.0, S).view(1, 1, S, 1)
    q = (q * 2.5).to(torch.bfloat16)
    k = (k * ramp).to(torch.bfloat16)
    v = v.to(torch.bfloat16)
    o, lse = run_fwd(cp, q, k, v, 4, True)
    o_ref, lse_ref = oracle_fwd(q, k, v, True, D ** -0.5)
    assert_close(o, o_ref, torch.bfloat16, "O")
    assert_lse_close(lse, lse_ref)


def test_output_guard_bands_untouched(cp):
    B, H, S, D = 1, 2, 1024, 128
    q, k, v, _ = make_qkv(B, H, S, D, torch.bfloat16, seed=51, with_dout=False)
    n = B * H * S * D
    pad = 4096
    obuf = torch.full((n + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((B * H * S + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    o = obuf[pad:pad + n].view(B, H, S, D)
    lse = lbuf[pad:pad + B * H * S].view(B, H, S)
    cp.fwd(q.cuda(), k.cuda(), v.cuda(), 2, True, out=o, lse=lse)
    assert cp.sync_status() == cp.OK
    assert torch.all(obuf[:pad] == 7.0) and torch.all(obuf[pad + n:] == 7.0)
    assert torch.all(lbuf[:pad] == 7.0) and torch.all(lbuf[pad + B * H * S:] == 7.0)


FULL = ["causal_b1h16s8192d128_cp4_bf16", "causal_b1h32s32768d128_cp8_bf16",
        "noncausal_b2h32s16384d128_cp2_bf16", "causal_b1h8s131072d128_cp16_bf16"]


@pytest.mark.parametrize("name", FULL)
def test_fwd_full_workload_sampled_rows(cp, name):
    w = WORKLOADS[name]
    q, k, v, _ = workload_inputs(w, with_dout=False)
    o, lse = run_fwd(cp, q, k, v, w.cp_size, w.causal)
    assert cp.last_path() == 0
    n_chunks = 2 * w.cp_size if w.causal else w.cp_size
    for b in range(w.B):
        for h in range(w.H):
            rows = sample_rows(w.S, n_chunks, 128, seed=1000 * b + h)
            o_ref, l_ref = orc.attn_fwd_rows(np64(q[b:b + 1, h:h + 1]), np64(k[b:b + 1, h:h + 1]),
                                             np64(v[b:b + 1, h:h + 1]), w.causal, w.scale, 0, 0, rows)
            assert_close(o[b, h, rows], o_ref, torch.bfloat16, f"{name} b{b} h{h} O rows")
            assert_lse_close(lse[b, h, rows], l_ref, f"{name} b{b} h{h} LSE rows")


def test_fwd_full_workload_whole_head(cp):
    w = WORKLOADS["causal_b1h16s8192d128_cp4_bf16"]
    q, k, v, _ = workload_inputs(w, with_dout=False)
    o, lse = run_fwd(cp, q, k, v, w.cp_size, w.causal)
    for h in (0, w.H // 2, w.H - 1):
        o_ref, l_ref = oracle_fwd(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], True, w.scale)
        assert_close(o[:, h:h + 1], o_ref, torch.bfloat16, f"head {h}")
        assert_lse_close(lse[:, h:h + 1], l_ref, f"head {h} lse")
