"""FP8 (e4m3) path on the GPU: the per-tensor maximum and the quantiser
against the oracle's encoder (bit for bit), and the e4m3 ring forward against
the fp64 oracle attention of the dequantised inputs.

Tolerance of the forward (derived from the format, fixed before the kernel
first ran).  The inputs are compared as the values the codes stand for, so the
only rounding the method adds is that of P: the kernel rounds 2^6 * P to e4m3
(3 mantissa bits, round to nearest even): relative error <= 2^-4 in the
normal range, absolute <= 2^-10 * 2^-6 = 2^-16 (in units of P) below it.  With
the kernel's running maximum m_k <= m*_i (the row's true maximum score), the
row sum l = exp(LSE_i - m_k) >= exp(LSE_i - m*_i), so for every element

  |O - O_ref| <= 2^-4 * sum_j p_ij |v_jd|              (normal-range P)
               + 2^-16 * sum_{j in A_i} |v_jd| * exp(m*_i - LSE_i)   (subnormal P)
               + 2^-8 |O_ref|                          (bf16 output, fp32 sums)
               + 2^-10 * (sum_j p_ij |v_jd| + 1)       (score rounding, ex2, slack)

where sum_j p_ij |v_jd| is the oracle's attention of |v| (same q, k).  LSE
uses the unrounded P: the usual 1e-3."""
import numpy as np
import pytest
import torch

from long_sequence_context_b200.inputs import WORKLOADS, make_qkv, workload_inputs
from oracle import fp8
from oracle import oracle as orc
from tests.util import assert_lse_close, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    from long_sequence_context_b200 import cpattn
    cpattn.set_path(0)
    return cpattn


def _f32(t):
    return t.float().cpu().numpy()


def oracle_quantized(x, transpose=False, heads=None):
    """codes and dequantised fp64 values of x [B, H, S, D] by the oracle (of the
    heads listed, with the scale of the whole tensor)."""
    xf = _f32(x)
    amax = np.abs(xf).max()
    if heads is not None:
        xf = xf[:, heads]
    codes, s, amax = fp8.quantize(xf, amax)
    deq = fp8.dequantize(codes, s)
    if transpose:
        codes = np.ascontiguousarray(np.swapaxes(codes, 2, 3))
    return codes, deq, amax


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_amax_is_exact(cp, dtype):
    q, k, v, _ = make_qkv(2, 3, 512, 64, dtype, seed=61)
    for t in (q, k, v):
        a = cp.amax(t.cuda())
        torch.cuda.synchronize()
        assert a.item() == np.float32(np.abs(_f32(t)).max())


@pytest.mark.parametrize("B,H,S,D,dtype", [(1, 2, 1024, 128, torch.bfloat16), (2, 3, 256, 64, torch.bfloat16),
                                           (1, 4, 8192, 128, torch.bfloat16), (1, 2, 512, 128, torch.float32)])
def test_quantize_matches_oracle_codes_bitwise(cp, B, H, S, D, dtype):
    q, _, v, _ = make_qkv(B, H, S, D, dtype, seed=62 + S)
    for x, transpose in ((q, False), (v, True)):
        xd = x.cuda()
        a = cp.amax(xd)
        got = cp.quantize_e4m3(xd, a, transpose=transpose)
        want, _, _ = oracle_quantized(x, transpose)
        torch.cuda.synchronize()
        got = got.cpu().numpy()
        assert got.shape == want.shape
        n_bad = int((got != want).sum())
        assert n_bad == 0, f"{n_bad} codes differ (transpose={transpose})"


def fp8_bound(qd, kd, vd, causal, scale, o_ref, lse_ref, b, h, rows):
    """Per-element bound of the module docstring for the given rows of head (b, h)."""
    sl = (slice(b, b + 1), slice(h, h + 1))
    a_abs, _ = orc.attn_fwd_rows(qd[sl], kd[sl], np.abs(vd[sl]), causal, scale, 0, 0, rows)
    m_star = fp8.row_max_scores(qd[b, h], kd[b, h], causal, scale, rows)
    cum = np.cumsum(np.abs(vd[b, h]), axis=0)
    csum = cum[rows] if causal else np.broadcast_to(cum[-1], (len(rows), vd.shape[-1]))
    sub = csum * np.exp(m_star - lse_ref)[:, None]
    return ((2.0 ** -4 + 2.0 ** -10) * a_abs + 2.0 ** -16 * sub + 2.0 ** -8 * np.abs(o_ref)
            + 2.0 ** -10)


def check_rows(cp, o, lse, qd, kd, vd, causal, scale, heads, rows_of):
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    for b, h in heads:
        rows = rows_of(b, h)
        sl = (slice(b, b + 1), slice(h, h + 1))
        o_ref, l_ref = orc.attn_fwd_rows(qd[sl], kd[sl], vd[sl], causal, scale, 0, 0, rows)
        assert_lse_close(lse[b, h, rows], l_ref, f"lse b{b} h{h}")
        bound = fp8_bound(qd, kd, vd, causal, scale, o_ref, l_ref, b, h, rows)
        err = np.abs(o[b, h, rows] - o_ref)
        assert np.all(np.isfinite(o[b, h, rows]))
        n_bad = int((err > bound).sum())
        worst = float(np.max(err / bound))
        assert n_bad == 0, f"b{b} h{h}: {n_bad} elements above the bound (worst err/bound {worst:.2f})"


@pytest.mark.parametrize("B,H,S,cp_size,causal", [
    (1, 2, 1024, 2, True),
    (1, 2, 2048, 4, True),
    (2, 1, 1024, 2, False),
    (1, 1, 768, 3, False),
])
def test_fwd_fp8_vs_oracle_every_row(cp, B, H, S, cp_size, causal):
    D = 128
    scale = D ** -0.5
    q, k, v, _ = make_qkv(B, H, S, D, torch.bfloat16, seed=70 + S + cp_size)
    q8, k8, vt8, a3 = cp.quantize_qkv_e4m3(q.cuda(), k.cuda(), v.cuda())
    o, lse = cp.fwd_fp8(q8, k8, vt8, a3, cp_size, causal, scale)
    assert cp.sync_status() == cp.OK
    (_, qd, _), (_, kd, _), (_, vd, _) = (oracle_quantized(t) for t in (q, k, v))
    heads = [(b, h) for b in range(B) for h in range(H)]
    check_rows(cp, o, lse, qd, kd, vd, causal, scale, heads, lambda b, h: np.arange(S))


def test_fwd_fp8_full_workload_sampled_rows(cp):
    """The S = 32768, H = 32, cp 8 causal workload in e4m3: 128 sampled rows
    (first / last of every chunk plus seeded rows) of four heads."""
    w = WORKLOADS["causal_b1h32s32768d128_cp8_bf16"]
    q, k, v, _ = workload_inputs(w, with_dout=False)
    q8, k8, vt8, a3 = cp.quantize_qkv_e4m3(q.cuda(), k.cuda(), v.cuda())
    o, lse = cp.fwd_fp8(q8, k8, vt8, a3, w.cp_size, w.causal, w.scale)
    assert cp.sync_status() == cp.OK
    hs = [0, 11, 22, 31]
    (_, qd, _), (_, kd, _), (_, vd, _) = (oracle_quantized(t, heads=hs) for t in (q, k, v))
    n_chunks = 2 * w.cp_size
    check_rows(cp, o[:, hs], lse[:, hs], qd, kd, vd, w.causal, w.scale,
               [(0, i) for i in range(len(hs))],
               lambda b, i: sample_rows(w.S, n_chunks, 128, seed=hs[i]))


def test_fwd_fp8_rejects_unsupported_shapes(cp):
    z = torch.zeros((1, 1, 256, 64), dtype=torch.uint8, device="cuda")
    zt = torch.zeros((1, 1, 64, 256), dtype=torch.uint8, device="cuda")
    a3 = torch.ones(3, dtype=torch.float32, device="cuda")
    with pytest.raises(cp.CpattnError) as e:     # D = 64
        cp.fwd_fp8(z, z, zt, a3, 1, True)
    assert e.value.status == cp.ERR_SHAPE
    z = torch.zeros((1, 1, 256, 128), dtype=torch.uint8, device="cuda")
    zt = torch.zeros((1, 1, 128, 256), dtype=torch.uint8, device="cuda")
    with pytest.raises(cp.CpattnError) as e:     # chunk of 64 rows
        cp.fwd_fp8(z, z, zt, a3, 2, True)
    assert e.value.status == cp.ERR_SHAPE
    assert cp.sync_status() == cp.OK


def test_fp8_all_zero_values_and_tiny_inputs(cp):
    """An all-zero V (max|v| = 0: scale 1, every code 0) gives O = 0 exactly;
    inputs a million times smaller than N(0, 1) quantise to the same codes as
    the unit-scale ones (the per-tensor scale absorbs the magnitude) and give
    the oracle's result within the same bound."""
    B, H, S, D, cp_size = 1, 2, 1024, 128, 2
    q, k, v, _ = make_qkv(B, H, S, D, torch.bfloat16, seed=81)
    zero = torch.zeros_like(v).cuda()
    q8, k8, vt8, a3 = cp.quantize_qkv_e4m3(q.cuda(), k.cuda(), zero)
    o, lse = cp.fwd_fp8(q8, k8, vt8, a3, cp_size, True)
    assert cp.sync_status() == cp.OK
    assert a3[2].item() == 0.0
    assert int(vt8.count_nonzero().item()) == 0
    assert torch.count_nonzero(o).item() == 0 and torch.isfinite(lse).all()
    tiny = [(t.float() * 1e-6).to(torch.bfloat16) for t in (q, k, v)]
    q8t, k8t, vt8t, a3t = cp.quantize_qkv_e4m3(*(t.cuda() for t in tiny))
    want, _, _ = oracle_quantized(tiny[0])
    assert np.array_equal(q8t.cpu().numpy(), want)
    o, lse = cp.fwd_fp8(q8t, k8t, vt8t, a3t, cp_size, True, scale=D ** -0.5 * 1e12)
    assert cp.sync_status() == cp.OK
    (_, qd, _), (_, kd, _), (_, vd, _) = (oracle_quantized(t) for t in tiny)
    check_rows(cp, o.float() * 1e6, lse, qd, kd, vd * 1e6, True, D ** -0.5 * 1e12, [(0, 0), (0, 1)],
               lambda b, h: np.arange(S))
