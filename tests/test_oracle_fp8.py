"""Pins of the fp8 (e4m3) oracle (oracle/fp8.py) against things other than
itself: values the format definition fixes, torch's own float8_e4m3fn
conversion (an independent library routine), brute force, and the oracle's
LSE."""
import numpy as np
import pytest
import torch

from oracle import fp8
from oracle import oracle as orc


def test_decode_known_codes():
    assert fp8.decode_code(0x00) == 0.0
    assert fp8.decode_code(0x01) == 2.0 ** -9          # smallest subnormal
    assert fp8.decode_code(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert fp8.decode_code(0x08) == 2.0 ** -6          # smallest normal
    assert fp8.decode_code(0x38) == 1.0
    assert fp8.decode_code(0x3C) == 1.5
    assert fp8.decode_code(0x7E) == 448.0              # largest finite
    assert np.isnan(fp8.decode_code(0x7F)) and np.isnan(fp8.decode_code(0xFF))
    assert fp8.decode_code(0xB8) == -1.0
    assert fp8.decode_code(0x80) == 0.0 and np.signbit(fp8.decode_code(0x80))


def test_decode_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(ref) & np.isnan(fp8.DECODE)
    assert np.array_equal(np.isnan(ref), np.isnan(fp8.DECODE))
    assert np.all((ref == fp8.DECODE) | both_nan)


def test_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = fp8.decode(codes)
    got = fp8.encode(vals)
    # +0 / -0 keep their sign bit
    assert np.array_equal(got, codes)


def test_encode_midpoints_go_to_the_even_code():
    v = fp8.DECODE[:0x7F]
    mids = (v[:-1] + v[1:]) / 2
    got = fp8.encode(mids)
    lo = np.arange(0x7E)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want.astype(np.uint8))
    # a hair either side of a midpoint goes to the nearer value
    eps = 1e-9
    assert np.array_equal(fp8.encode(mids - eps * v[1:]), lo.astype(np.uint8))
    assert np.array_equal(fp8.encode(mids + eps * v[1:]), (lo + 1).astype(np.uint8))


def test_encode_saturates():
    assert fp8.encode(np.array([1e6, -1e6, 448.0, 463.9, 470.0]))[:5].tolist() == \
        [0x7E, 0xFE, 0x7E, 0x7E, 0x7E]
    assert fp8.encode(np.array([np.nan]))[0] == 0x7F


def test_encode_matches_torch_on_random_values():
    g = torch.Generator().manual_seed(4)
    x = (torch.randn(200000, generator=g, dtype=torch.float32) * 60).clamp(-440, 440)
    x = torch.cat([x, torch.randn(20000, generator=g) * 1e-3])   # subnormal range
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.encode(x.numpy()), ref)


def test_quantize_scale_and_bounds():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(4, 1000, generator=g).to(torch.bfloat16).float().numpy()
    codes, s, amax = fp8.quantize(x)
    assert amax == np.float32(np.abs(x).max())
    assert s == np.float32(448.0) / amax
    xq = fp8.dequantize(codes, s)
    # the largest element maps to (about) 448: relative error of RNE is <= 2^-4
    assert np.all(np.abs(xq - x) <= 2.0 ** -4 * np.abs(x) + 2.0 ** -10 / s)
    assert np.abs(fp8.decode(codes)).max() <= 448.0
    zero = fp8.quantize(np.zeros(8, dtype=np.float32))
    assert zero[1] == 1.0 and np.all(zero[0] == 0)


@pytest.mark.parametrize("causal", [True, False])
def test_row_max_scores_brackets_the_oracle_lse(causal):
    # LSE_i = m_i + log sum_j exp(s_ij - m_i) with 1 <= sum <= n_i
    g = torch.Generator().manual_seed(6)
    S, D = 64, 16
    q, k, v = (torch.randn(S, D, generator=g, dtype=torch.float64).numpy() for _ in range(3))
    _, lse = orc.attn_fwd(q[None, None], k[None, None], v[None, None], causal, 0.3)
    rows = np.arange(S)
    m = fp8.row_max_scores(q, k, causal, 0.3, rows)
    n = rows + 1 if causal else np.full(S, S)
    assert np.all(lse[0, 0] >= m - 1e-12)
    assert np.all(lse[0, 0] <= m + np.log(n) + 1e-12)
    # one key: the maximum is that score and LSE equals it
    assert abs(m[0] - 0.3 * q[0] @ k[0]) < 1e-12 if causal else True
