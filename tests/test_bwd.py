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


def early_and_late_keys(S, n_chunks, seed):
    """Key columns whose dK / dV sum over long ring walks: the first key of
    every chunk and 16 seeded keys from the first half of the sequence (every
    query row after them sees them, so their terms come from q tiles of every
    virtual rank at every ring step), plus the last 32 keys (a DIAG corner)."""
    c = S // n_chunks
    g = np.random.default_rng(1000 + seed)
    cols = {a * c for a in range(n_chunks)}
    cols |= {int(x) for x in g.integers(0, S // 2, size=16)}
    cols |= set(range(S - 32, S))
    return np.array(sorted(cols), dtype=np.int64)


@pytest.mark.parametrize("name", FULL)
def test_bwd_full_workload_sampled(cp, name):
    w = WORKLOADS[name]
    q, k, v, dout = workload_inputs(w)
    dq, dk, dv = run_fwd_bwd(cp, q, k, v, dout, w.cp_size, w.causal)
    n_chunks = 2 * w.cp_size if w.causal else w.cp_size
    # dQ on sampled rows of two heads; dK / dV of one head on early keys (long
    # walks over every ring step) and the last 32 keys when causal, on four keys
    # (each seen by every row) otherwise
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        args = [np64(t[sl]) for t in (q, k, v, dout)]
        rows = sample_rows(w.S, n_chunks, 48, seed=h)
        rq = orc.attn_bwd_dq_rows(*args, w.causal, w.scale, 0, 0, rows)
        assert_close(dq[b, h, rows], rq, torch.bfloat16, f"{name} dQ rows b{b} h{h}")
    b, h = 0, w.H // 2
    sl = (slice(b, b + 1), slice(h, h + 1))
    args = [np64(t[sl]) for t in (q, k, v, dout)]
    cols = early_and_late_keys(w.S, n_chunks, seed=h) if w.causal else np.array([0, 1, w.S // 2, w.S - 1])
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


ACC_CASES = [
    (1, 2, 1024, 128, 2, True, torch.bfloat16, 0),   # tcgen05 kernels
    (1, 2, 1024, 64, 2, False, torch.bfloat16, 0),
    (1, 2, 1024, 128, 4, True, torch.bfloat16, 1),   # CUDA-core kernels
    (1, 2, 256, 64, 2, True, torch.float32, 0),      # fp32: CUDA-core kernels (automatic)
]


@pytest.mark.parametrize("B,H,S,D,cp_size,causal,dtype,path", ACC_CASES)
def test_bwd_accumulate_adds_the_gradients_in_fp32(cp, B, H, S, D, cp_size, causal, dtype, path):
    """cpattn_bwd_accumulate adds dQ, dK, dV into fp32 sums: from zero, one
    rounding of the sum gives cpattn_bwd's output exactly; from a seeded start,
    two calls add twice the gradient (checked against the oracle)."""
    q, k, v, dout = make_qkv(B, H, S, D, dtype, seed=300 + S + D + path)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    prev = cp.set_path(path)
    try:
        o, lse = cp.fwd(qd, kd, vd, cp_size, causal)
        ref = cp.bwd(qd, kd, vd, o, lse, dod, cp_size, causal)
        zero = [torch.zeros(q.shape, dtype=torch.float32, device="cuda") for _ in range(3)]
        cp.bwd_accumulate_(qd, kd, vd, o, lse, dod, *zero, cp_size, causal)
        gen = torch.Generator().manual_seed(7)
        start = [torch.randn(q.shape, generator=gen, dtype=torch.float32) for _ in range(3)]
        acc = [t.cuda() for t in start]
        cp.bwd_accumulate_(qd, kd, vd, o, lse, dod, *acc, cp_size, causal)
        cp.bwd_accumulate_(qd, kd, vd, o, lse, dod, *acc, cp_size, causal)
        assert cp.sync_status() == cp.OK
        assert cp.last_path() == (1 if dtype == torch.float32 else path)
    finally:
        cp.set_path(prev)
    for name, z, r in zip(("dQ", "dK", "dV"), zero, ref):
        assert torch.equal(z.to(dtype), r), f"{name}: one rounding of the fp32 sum differs from cpattn_bwd"
    want = orc.attn_bwd(np64(q), np64(k), np64(v), np64(dout), causal, D ** -0.5)
    for name, a, s0, w_ in zip(("dQ", "dK", "dV"), acc, start, want):
        got = (np64(a.cpu()) - np64(s0)) / 2.0
        assert_close(got, w_, dtype, f"{name} (two accumulating calls)")


def test_bwd_accumulate_rejects_mismatched_accumulators(cp):
    q = torch.zeros((1, 1, 256, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 256), dtype=torch.float32, device="cuda")
    good = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    bf = torch.zeros(q.shape, dtype=torch.bfloat16, device="cuda")
    short = torch.zeros((1, 1, 128, 64), dtype=torch.float32, device="cuda")
    n0 = cp.launch_count()
    with pytest.raises(TypeError):
        cp.bwd_accumulate_(q, q, q, q, lse, q, bf, good, good.clone(), 1, True)
    with pytest.raises(ValueError):
        cp.bwd_accumulate_(q, q, q, q, lse, q, good, short, good.clone(), 1, True)
    with pytest.raises(ValueError):
        cp.bwd_accumulate_(q, q, q, q, lse, q, good, good, good.clone(), 1, True)
    assert cp.launch_count() == n0


# chunk lengths that are not multiples of 16 (CUDA-core kernels; any c is allowed)
ODD = [
    (1, 2, 96, 64, 2, True, torch.float32),     # c = 24
    (1, 1, 28, 64, 2, True, torch.float32),     # c = 7
    (1, 1, 6, 64, 3, True, torch.float32),      # c = 1
    (1, 2, 40, 128, 5, False, torch.float32),   # c = 8, non-causal
    (1, 2, 200, 64, 4, True, torch.bfloat16),   # c = 25
    (2, 1, 120, 128, 3, False, torch.bfloat16), # c = 40
]


@pytest.mark.parametrize("B,H,S,D,cp_size,causal,dtype", ODD)
def test_any_chunk_length_fwd_bwd_vs_oracle(cp, B, H, S, D, cp_size, causal, dtype):
    from tests.util import assert_lse_close
    q, k, v, dout = make_qkv(B, H, S, D, dtype, seed=500 + S + cp_size)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = cp.fwd(qd, kd, vd, cp_size, causal)
    dq, dk, dv = cp.bwd(qd, kd, vd, o, lse, dod, cp_size, causal)
    assert cp.sync_status() == cp.OK
    assert cp.last_path() == 1
    ro, rl = orc.attn_fwd(np64(q), np64(k), np64(v), causal, D ** -0.5)
    assert_close(o.cpu(), ro, dtype, "O")
    assert_lse_close(lse.cpu(), rl)
    rq, rk, rv = orc.attn_bwd(np64(q), np64(k), np64(v), np64(dout), causal, D ** -0.5)
    assert_close(dq.cpu(), rq, dtype, "dQ")
    assert_close(dk.cpu(), rk, dtype, "dK")
    assert_close(dv.cpu(), rv, dtype, "dV")
    # the per-step partials merged equal the fused result
    o_acc = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    l_acc = torch.full(q.shape[:-1], float("-inf"), dtype=torch.float32, device="cuda")
    for t in range(cp_size):
        op, lp = cp.fwd_step(qd, kd, vd, cp_size, t, causal)
        cp.merge_(o_acc, l_acc, op, lp)
    assert cp.sync_status() == cp.OK
    assert_close(o_acc.cpu(), ro, dtype, "O from steps + merge")


TWO_SM_CASES = [
    (1, 2, 1024, 128, 2, True),    # 2 tiles per chunk: one pair per chunk
    (1, 4, 4096, 128, 4, True),    # 4 tiles per chunk, 4 heads (head groups of 4)
    (2, 2, 2048, 128, 2, False),
    (1, 3, 1024, 128, 2, True),    # 3 heads: head groups of 1
]


@pytest.mark.parametrize("B,H,S,D,cp_size,causal", TWO_SM_CASES)
def test_two_sm_dq_matches_one_sm_dq(cp, B, H, S, D, cp_size, causal):
    """The two-SM dQ kernel (a cluster of two CTAs per pair of Q tiles,
    cta_group::2 MMAs) against the one-SM dQ kernel on the same inputs: the
    same products in the same order per output row, so the fp32 sums, and
    hence the bf16 dQ, can differ at most by the tensor core's internal
    summation order -- one bf16 rounding step (2^-8 relative) of an element,
    plus 2^-8 of the row's largest entry for sums near a rounding boundary of
    a cancelling row.  dK and dV come from the same kernel on both paths."""
    q, k, v, dout = make_qkv(B, H, S, D, torch.bfloat16, seed=400 + S + H)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = cp.fwd(qd, kd, vd, cp_size, causal)
    dq2, dk2, dv2 = cp.bwd(qd, kd, vd, o, lse, dod, cp_size, causal)
    prev = cp.set_path(2)
    try:
        dq1, dk1, dv1 = cp.bwd(qd, kd, vd, o, lse, dod, cp_size, causal)
        assert cp.sync_status() == cp.OK
        assert cp.last_path() == 0
    finally:
        cp.set_path(prev)
    assert torch.equal(dk2, dk1) and torch.equal(dv2, dv1)
    a, b = dq2.float(), dq1.float()
    rowmax = b.abs().amax(dim=-1, keepdim=True)
    bound = 2.0 ** -8 * (b.abs() + rowmax) + 1e-30
    assert bool(((a - b).abs() <= bound).all()), float((a - b).abs().max())
    rq, _, _ = orc.attn_bwd(np64(q), np64(k), np64(v), np64(dout), causal, D ** -0.5)
    assert_close(dq2.cpu(), rq, torch.bfloat16, "dQ (two SMs)")


@pytest.mark.parametrize("groups", [2, 4])
def test_head_group_calls_match_one_call(cp, groups):
    # Heads are independent problems: calling the forward and the backward on
    # head-slice views (as the end-to-end benchmark does, to overlap its copies)
    # gives every output bit for bit as one call on all heads.
    B, H, S, D, cps = 1, 4, 2048, 128, 2
    q, k, v, dout = make_qkv(B, H, S, D, torch.bfloat16, seed=321)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, dout))
    o, lse = cp.fwd(qd, kd, vd, cps, True)
    dq, dk, dv = cp.bwd(qd, kd, vd, o, lse, dod, cps, True)
    og, lg = torch.full_like(o, float("nan")), torch.full_like(lse, float("nan"))
    gq, gk, gv = (torch.full_like(t, float("nan")) for t in (dq, dk, dv))
    ws = torch.empty(cp.bwd_workspace_bytes(B, H, S, D), dtype=torch.uint8, device=qd.device)
    for c in range(groups):
        h = slice(c * H // groups, (c + 1) * H // groups)
        cp.fwd(qd[:, h], kd[:, h], vd[:, h], cps, True, out=og[:, h], lse=lg[:, h])
        cp.bwd(qd[:, h], kd[:, h], vd[:, h], og[:, h], lg[:, h], dod[:, h], cps, True, workspace=ws,
               dq=gq[:, h], dk=gk[:, h], dv=gv[:, h])
    assert cp.sync_status() == cp.OK
    for name, a, b in (("O", o, og), ("LSE", lse, lg), ("dQ", dq, gq), ("dK", dk, gk), ("dV", dv, gv)):
        assert torch.equal(a, b), name
