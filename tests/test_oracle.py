"""Pins for the fp64 oracle: each check ties it to something other than itself
(a library routine, a closed form, finite differences, the pages' worked
example, or an exhaustive invariant), so that a dropped term, a wrong sign or
index, or a transposed operand fails at least one of them."""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import oracle as orc
from oracle import plan as oplan

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


def sdpa64(q, k, v, causal, scale):
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    return F.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=causal, scale=scale).numpy()


# ---------------------------------------------------------------- forward --

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("S,D", [(1, 4), (7, 8), (37, 16), (128, 64)])
def test_fwd_matches_torch_sdpa_fp64(causal, S, D):
    B, H = 2, 3
    q, k, v = (rnd((B, H, S, D), s) for s in (1, 2, 3))
    scale = 1.0 / math.sqrt(D)
    o, lse = orc.attn_fwd(q, k, v, causal, scale)
    ref = sdpa64(q, k, v, causal, scale)
    assert np.max(np.abs(o - ref)) < 1e-10


def test_fwd_scale_is_applied():
    S, D = 9, 4
    q, k, v = (rnd((1, 1, S, D), s) for s in (4, 5, 6))
    o, _ = orc.attn_fwd(q, k, v, True, 0.37)
    assert np.max(np.abs(o - sdpa64(q, k, v, True, 0.37))) < 1e-10
    o2, _ = orc.attn_fwd(q, k, v, True, 1.0)
    assert np.max(np.abs(o - o2)) > 1e-3  # the scale matters


def test_closed_form_single_position():
    q, k, v = (rnd((1, 1, 1, 8), s) for s in (7, 8, 9))
    scale = 0.3
    o, lse = orc.attn_fwd(q, k, v, True, scale)
    assert np.allclose(o[0, 0, 0], v[0, 0, 0], atol=1e-14)
    assert abs(lse[0, 0, 0] - scale * float(q[0, 0, 0] @ k[0, 0, 0])) < 1e-14


def test_closed_form_zero_queries_causal():
    # q == 0: every allowed score is 0, so LSE_i = log(i+1), O_i = mean(v_0..v_i)
    S, D = 50, 8
    q = np.zeros((1, 1, S, D))
    k, v = rnd((1, 1, S, D), 10), rnd((1, 1, S, D), 11)
    o, lse = orc.attn_fwd(q, k, v, True, 0.5)
    idx = np.arange(S)
    assert np.max(np.abs(lse[0, 0] - np.log(idx + 1))) < 1e-13
    mean = np.cumsum(v[0, 0], axis=0) / (idx[:, None] + 1)
    assert np.max(np.abs(o[0, 0] - mean)) < 1e-13
    o_nc, lse_nc = orc.attn_fwd(q, k, v, False, 0.5)
    assert np.max(np.abs(lse_nc[0, 0] - np.log(S))) < 1e-13
    assert np.max(np.abs(o_nc[0, 0] - v[0, 0].mean(axis=0))) < 1e-13


def test_closed_form_equal_keys():
    # all keys equal to u: s_ij = scale q_i.u for every j, so
    # LSE_i = scale q_i.u + log(#allowed) and O_i = mean of the allowed v
    S, D = 33, 16
    q, v = rnd((1, 1, S, D), 12), rnd((1, 1, S, D), 13)
    u = rnd((D,), 14)
    k = np.broadcast_to(u, (1, 1, S, D)).copy()
    scale = 0.25
    o, lse = orc.attn_fwd(q, k, v, True, scale)
    idx = np.arange(S)
    want = scale * (q[0, 0] @ u) + np.log(idx + 1)
    assert np.max(np.abs(lse[0, 0] - want)) < 1e-12
    mean = np.cumsum(v[0, 0], axis=0) / (idx[:, None] + 1)
    assert np.max(np.abs(o[0, 0] - mean)) < 1e-12


def test_closed_form_two_keys():
    D = 4
    q, k, v = (rnd((1, 1, 2, D), s) for s in (15, 16, 17))
    scale = 0.9
    o, lse = orc.attn_fwd(q, k, v, False, scale)
    a = scale * q[0, 0, 1] @ k[0, 0, 0]
    b = scale * q[0, 0, 1] @ k[0, 0, 1]
    assert abs(lse[0, 0, 1] - math.log(math.exp(a) + math.exp(b))) < 1e-13
    pa = math.exp(a) / (math.exp(a) + math.exp(b))
    assert np.max(np.abs(o[0, 0, 1] - (pa * v[0, 0, 0] + (1 - pa) * v[0, 0, 1]))) < 1e-13


def test_large_scale_selects_argmax():
    S, D = 16, 8
    q, k, v = (rnd((1, 1, S, D), s) for s in (18, 19, 20))
    o, _ = orc.attn_fwd(q, k, v, True, 1e4)
    for i in range(S):
        j = int(np.argmax(q[0, 0, i] @ k[0, 0, : i + 1].T))
        assert np.max(np.abs(o[0, 0, i] - v[0, 0, j])) < 1e-8


def test_softmax_rows_sum_to_one():
    # with v = 1 every output entry is sum_j P_ij
    S, D = 64, 8
    q, k = rnd((1, 1, S, D), 21, 3.0), rnd((1, 1, S, D), 22, 3.0)
    v = np.ones((1, 1, S, D))
    for causal in (True, False):
        o, _ = orc.attn_fwd(q, k, v, causal, 1.0)
        assert np.max(np.abs(o - 1.0)) < 1e-12


def test_brute_force_tiny():
    # no max-subtraction, dense matrix form, exhaustive over S <= 16
    for S in (1, 2, 5, 16):
        D = 8
        q, k, v = (rnd((S, D), 30 + s) for s in range(3))
        for causal in (True, False):
            o, lse = orc.attn_fwd(q, k, v, causal, 0.4)
            E = np.exp(0.4 * q @ k.T)
            if causal:
                E = np.tril(E)
            Z = E.sum(axis=1)
            assert np.max(np.abs(o[0, 0] - (E / Z[:, None]) @ v)) < 1e-12
            assert np.max(np.abs(lse[0, 0] - np.log(Z))) < 1e-12


def test_rows_variant_matches_full():
    S, D = 96, 16
    q, k, v = (rnd((1, 2, S, D), s) for s in (40, 41, 42))
    o, lse = orc.attn_fwd(q, k, v, True, 0.25)
    rows = [0, 5, 63, 95]
    orow, lrow = orc.attn_fwd_rows(q, k, v, True, 0.25, 0, 1, rows)
    assert np.max(np.abs(orow - o[0, 1, rows])) < 1e-14
    assert np.max(np.abs(lrow - lse[0, 1, rows])) < 1e-14


# --------------------------------------------------------------- backward --

def _loss(q, k, v, dout, causal, scale):
    o, _ = orc.attn_fwd(q, k, v, causal, scale)
    return float(np.sum(o * dout))


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_finite_differences(causal):
    S, D = 12, 6
    q, k, v, dout = (rnd((1, 1, S, D), s) for s in (50, 51, 52, 53))
    scale = 0.45
    dq, dk, dv = orc.attn_bwd(q, k, v, dout, causal, scale)
    h = 1e-6
    g = np.random.default_rng(54)
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            i, d = int(g.integers(S)), int(g.integers(D))
            xp, xm = x.copy(), x.copy()
            xp[0, 0, i, d] += h
            xm[0, 0, i, d] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd = (_loss(args_p["q"], args_p["k"], args_p["v"], dout, causal, scale)
                  - _loss(args_m["q"], args_m["k"], args_m["v"], dout, causal, scale)) / (2 * h)
            an = grad[0, 0, i, d]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, i, d, fd, an)


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_matches_torch_autograd_fp64(causal):
    B, H, S, D = 1, 2, 40, 16
    q, k, v, dout = (rnd((B, H, S, D), s) for s in (60, 61, 62, 63))
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = orc.attn_bwd(q, k, v, dout, causal, scale)
    tq, tk, tv = (torch.from_numpy(a).requires_grad_() for a in (q, k, v))
    out = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    out.backward(torch.from_numpy(dout))
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.max(np.abs(mine - ref.numpy())) < 1e-10


def test_bwd_sum_identities():
    # sum_j dS_ij = 0 for every row, hence sum_j dK_j = 0; sum_j P_ij = 1,
    # hence sum_j dV_j = sum_i dO_i
    S, D = 64, 8
    q, k, v, dout = (rnd((1, 1, S, D), s) for s in (70, 71, 72, 73))
    for causal in (True, False):
        dq, dk, dv = orc.attn_bwd(q, k, v, dout, causal, 0.3)
        assert np.max(np.abs(dk[0, 0].sum(axis=0))) < 1e-12
        assert np.max(np.abs(dv[0, 0].sum(axis=0) - dout[0, 0].sum(axis=0))) < 1e-12


def test_bwd_partial_variants_match_full():
    S, D = 80, 8
    q, k, v, dout = (rnd((1, 1, S, D), s) for s in (80, 81, 82, 83))
    for causal in (True, False):
        dq, dk, dv = orc.attn_bwd(q, k, v, dout, causal, 0.35)
        rows = [0, 17, 79]
        assert np.max(np.abs(orc.attn_bwd_dq_rows(q, k, v, dout, causal, 0.35, 0, 0, rows)
                             - dq[0, 0, rows])) < 1e-14
        cols = [3, 40, 79]
        dkc, dvc = orc.attn_bwd_kv_cols(q, k, v, dout, causal, 0.35, 0, 0, cols)
        assert np.max(np.abs(dkc - dk[0, 0, cols])) < 1e-14
        assert np.max(np.abs(dvc - dv[0, 0, cols])) < 1e-14


# ------------------------------------------------------------------- ring --

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("cp", [1, 2, 4, 8, 16])
def test_ring_equals_unsplit(causal, cp):
    S, D = 256, 16
    q, k, v = (rnd((1, 2, S, D), s) for s in (90, 91, 92))
    scale = 1.0 / math.sqrt(D)
    o_ref, lse_ref = orc.attn_fwd(q, k, v, causal, scale)
    o, lse = orc.ring_fwd(q, k, v, cp, causal, scale)
    assert np.max(np.abs(o - o_ref)) < 1e-12
    assert np.max(np.abs(lse - lse_ref)) < 1e-12


@pytest.mark.parametrize("causal", [True, False])
def test_ring_steps_merge_to_unsplit(causal):
    S, D, cp = 128, 8, 4
    q, k, v = (rnd((1, 1, S, D), s) for s in (93, 94, 95))
    o_ref, lse_ref = orc.attn_fwd(q, k, v, causal, 0.3)
    o_acc = np.zeros((S, D))
    lse_acc = np.full(S, -np.inf)
    for t in range(cp):
        op, lp = orc.ring_step(q, k, v, cp, causal, 0.3, t)
        o_acc, lse_acc = orc.merge(o_acc, lse_acc, op[0, 0], lp[0, 0])
    assert np.max(np.abs(o_acc - o_ref[0, 0])) < 1e-12
    assert np.max(np.abs(lse_acc - lse_ref[0, 0])) < 1e-12


def test_ring_step_zero_is_local_chunks():
    # step 0 uses each rank's own K/V: for causal zigzag, rows of chunk a see
    # only keys of chunks owned by the same rank that are not after a
    S, D, cp = 64, 4, 2
    c = S // (2 * cp)
    q, k, v = (rnd((1, 1, S, D), s) for s in (96, 97, 98))
    op, lp = orc.ring_step(q, k, v, cp, True, 0.5, 0)
    for i in (0, c - 1, c, 2 * c + 3, S - 1):
        a = i // c
        r = oplan.chunk_owner(a, cp, True)
        keys = [j for b in oplan.owned_chunks(r, cp, True) for j in range(b * c, (b + 1) * c)
                if j <= i]
        s = 0.5 * q[0, 0, i] @ k[0, 0, keys].T
        assert abs(lp[0, 0, i] - np.log(np.sum(np.exp(s)))) < 1e-12


def test_merge_identities():
    D = 4
    oa, ob = rnd((3, D), 100), rnd((3, D), 101)
    la, lb = np.array([0.3, -np.inf, 1.0]), np.array([-np.inf, 0.2, 1.0])
    o, l = orc.merge(oa, la, ob, lb)
    assert np.allclose(o[0], oa[0]) and l[0] == 0.3       # empty partial
    assert np.allclose(o[1], ob[1]) and l[1] == 0.2       # empty accumulator
    assert abs(l[2] - (1.0 + math.log(2.0))) < 1e-15      # equal weights
    assert np.max(np.abs(o[2] - 0.5 * (oa[2] + ob[2]))) < 1e-15
    both = orc.merge(np.zeros((1, D)), np.array([-np.inf]), np.zeros((1, D)), np.array([-np.inf]))
    assert both[1][0] == -np.inf and np.all(both[0] == 0)


# ------------------------------------------------------------------- plan --

def read_golden_zigzag():
    rows = []
    with open(os.path.join(GOLDEN, "zigzag_cp4.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


def test_plan_golden_zigzag_cp4():
    for r, a, b in read_golden_zigzag():
        assert oplan.owned_chunks(r, 4, True) == [a, b]


@pytest.mark.parametrize("cp", [1, 2, 3, 4, 8, 16])
def test_plan_invariants(cp):
    S = 2 * cp * 4
    rows = oplan.plan_rows(S, cp, True)
    assert len(rows) == cp * cp * 4
    seen = {}
    per_rank = {r: [0, 0] for r in range(cp)}
    for r, t, a, b, src, kind in rows:
        assert src == (r - t) % cp
        assert a in oplan.owned_chunks(r, cp, True)
        assert b in oplan.owned_chunks(src, cp, True)
        if kind != oplan.SKIP:
            assert (a, b) not in seen
            seen[(a, b)] = kind
            per_rank[r][kind - 1] += 1
    assert set(seen) == {(a, b) for a in range(2 * cp) for b in range(2 * cp) if a >= b}
    for r in range(cp):
        assert per_rank[r] == [2 * cp - 1, 2]  # balanced: 2N-1 FULL + 2 DIAG
    chunks = sorted(c for r in range(cp) for c in oplan.owned_chunks(r, cp, True))
    assert chunks == list(range(2 * cp))


def test_plan_noncausal_contiguous():
    rows = oplan.plan_rows(64, 4, False)
    assert len(rows) == 16
    assert all(kind == oplan.FULL for *_, kind in rows)
    assert sorted((a, b) for _, _, a, b, _, _ in rows) == [(a, b) for a in range(4) for b in range(4)]


def _plan_pins_fail(monkeypatch, **planted):
    """True when at least one of the plan pins above fails with `planted`
    functions swapped into the plan oracle (on the CPU, for this test only)."""
    for name, fn in planted.items():
        monkeypatch.setattr(oplan, name, fn)
    checks = [test_plan_golden_zigzag_cp4, test_plan_noncausal_contiguous] + \
             [lambda cp=cp: test_plan_invariants(cp) for cp in (1, 2, 3, 4, 8, 16)]
    failed = 0
    for check in checks:
        try:
            check()
        except AssertionError:
            failed += 1
    return failed > 0


@pytest.mark.parametrize("mistake", ["zigzag_off_by_one", "contiguous_when_causal", "diag_as_full",
                                     "ring_reads_ahead", "skip_as_full"])
def test_plan_pins_catch_planted_mistakes(monkeypatch, mistake):
    """Plausible mistakes planted in the plan oracle: each must make at least
    one of the plan pins (golden example, invariants) fail."""
    own, kind, rows = oplan.owned_chunks, oplan.block_kind, oplan.plan_rows
    if mistake == "zigzag_off_by_one":       # rank r owns {r, 2N-2-r}
        planted = {"owned_chunks": lambda r, n, c: [r, 2 * n - 2 - r] if c else [r]}
    elif mistake == "contiguous_when_causal":  # rank r owns {2r, 2r+1}
        planted = {"owned_chunks": lambda r, n, c: [2 * r, 2 * r + 1] if c else [r]}
    elif mistake == "diag_as_full":          # the diagonal block left unmasked
        planted = {"block_kind": lambda a, b, c: oplan.FULL if (c and a == b) else kind(a, b, c)}
    elif mistake == "skip_as_full":          # a future block computed
        planted = {"block_kind": lambda a, b, c: oplan.FULL if c else kind(a, b, c)}
    else:                                    # step t reads rank (r + t) mod N, src field kept
        def ahead(S, n, c):
            out = []
            for r, t, a, b, src, k in rows(S, n, c):
                s2 = (r + t) % n
                b2 = own(s2, n, c)[own(src, n, c).index(b)]
                out.append((r, t, a, b2, src, kind(a, b2, c)))
            return out
        planted = {"plan_rows": ahead}
    assert _plan_pins_fail(monkeypatch, **planted)
