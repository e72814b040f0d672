"""The layer's projection GEMM (cpattn_gemm, tcgen05) against an fp64 product
of the same bf16 values.

Bound per element: the result is rounded once to bf16 (relative 2^-9) after an
fp32 accumulation whose error is far below that, so
|C - ref| <= 2^-8 |ref| + 2^-16 sum_k |a_k||b_k|,
the second term covering elements whose exact value nearly cancels."""
import pytest
import torch

from long_sequence_context_b200 import cpattn as cp

pytestmark = pytest.mark.gpu


def _ref(a, b, bias, a_t, b_t):
    A = a.double().T if a_t else a.double()
    Bm = b.double() if b_t else b.double().T
    c = A @ Bm
    mag = A.abs() @ Bm.abs()
    if bias is not None:
        c = c + bias.double()
        mag = mag + bias.double().abs()
    return c, mag


def _check(c, ref, mag, what):
    err = (c.double().cpu() - ref).abs()
    bound = 2.0 ** -8 * ref.abs() + 2.0 ** -16 * mag
    assert torch.isfinite(c).all(), what
    bad = (err > bound).sum().item()
    assert bad == 0, f"{what}: {bad} elements outside the bound, max err {err.max().item():.3e}"


@pytest.mark.parametrize("a_t,b_t", [(0, 0), (0, 1), (1, 1), (1, 0)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (296, 520, 200), (4096, 2560, 256)])
def test_gemm_layouts_match_fp64(M, N, K, a_t, b_t):
    g = torch.Generator().manual_seed(M + N + K + 2 * a_t + b_t)
    a = torch.randn((K, M) if a_t else (M, K), generator=g).to(torch.bfloat16)
    b = torch.randn((K, N) if b_t else (N, K), generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g).to(torch.bfloat16) if (a_t, b_t) == (0, 0) else None
    c = cp.gemm(a.cuda(), b.cuda(), None if bias is None else bias.cuda(), a_t=bool(a_t), b_t=bool(b_t))
    cp.check_device_status()
    ref, mag = _ref(a, b, bias, a_t, b_t)
    _check(c, ref, mag, f"M{M} N{N} K{K} a_t{a_t} b_t{b_t}")


def test_gemm_repeat_is_bitwise_identical():
    g = torch.Generator().manual_seed(3)
    a = torch.randn(1024, 512, generator=g).to(torch.bfloat16).cuda()
    b = torch.randn(768, 512, generator=g).to(torch.bfloat16).cuda()
    c1 = cp.gemm(a, b)
    c2 = cp.gemm(a, b)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)


def test_gemm_rejects_unsupported_sizes():
    import ctypes
    t = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    assert cp.lib.cpattn_gemm(p, p, None, p, 100, 64, 64, 0, 0, None) == cp.ERR_SHAPE
    assert cp.lib.cpattn_gemm(p, p, None, p, 64, 64, 0, 0, 0, None) == cp.ERR_SHAPE
    assert cp.lib.cpattn_gemm(p, p, None, p, 64, 64, 64, 2, 0, None) == cp.ERR_ARG
    assert cp.lib.cpattn_gemm(ctypes.c_void_p(t.data_ptr() + 2), p, None, p, 64, 64, 64, 0, 0,
                              None) == cp.ERR_ALIGN
    assert cp.sync_status() == cp.OK
