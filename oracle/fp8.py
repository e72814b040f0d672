"""FP8 (e4m3) side of the oracle.  TEST INFRASTRUCTURE ONLY: imported by
tests/ and bench.py's CPU-baseline leg, never by the product package.

Source of the method: "Megatron-LM source analysis: Context Parallel"
(mieleap.com), section 4: context parallelism combined with FP8 attention
inputs (the --fp8 flag) to save memory.  The pages do not fix the format or
the scaling, so this follows the plainest reading, stated here:

  * format: e4m3 in its "fn" variant -- 1 sign bit, 4 exponent bits (bias 7),
    3 mantissa bits, subnormals, no infinities, largest finite 448, the one
    code 0x7F / 0xFF is NaN;
  * per-tensor scaling: s = 448 / max|x| (fp32 arithmetic), code =
    round-to-nearest-even(fp32(x * s)) saturated to +-448; the value the code
    stands for is decode(code) / s;
  * attention on fp8 inputs is the attention of those dequantised values: the
    oracle is the fp64 attention (oracle.attn_fwd) of them.

Every function is written from the format's definition (a table of all 256
codes; encoding = the nearest table value, ties to the even code), not from
any conversion routine.
"""
import numpy as np

E4M3_MAX = 448.0


def decode_code(c: int) -> float:
    """Value of one e4m3 code (0..255) by the format definition."""
    sign = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 0xF
    m = c & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6          # subnormal: 0.m x 2^(1 - 7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)   # normal: 1.m x 2^(e - 7)


DECODE = np.array([decode_code(c) for c in range(256)], dtype=np.float64)

# non-negative finite values in increasing order, with their codes (0x00..0x7E)
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = DECODE[:0x7F]
assert np.all(np.diff(_POS_VALUES) > 0)


def encode(x) -> np.ndarray:
    """e4m3 codes of x (any float array): the nearest finite value, ties to the
    code with an even mantissa, saturated to +-448; NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_POS_VALUES, a, side="left")      # first value >= a
    hi = np.minimum(hi, len(_POS_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((_POS_CODES[hi] & 1) == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    code = np.where(a == _POS_VALUES[hi], _POS_CODES[hi], code)
    code = code | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def decode(codes) -> np.ndarray:
    return DECODE[np.asarray(codes, dtype=np.int64)]


def scale_of(amax) -> np.float32:
    """Per-tensor scale s = 448 / amax in fp32 (1 when the tensor is all zero)."""
    amax = np.float32(amax)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(E4M3_MAX) / amax


def quantize(x, amax=None):
    """(codes, s, amax) for a tensor x of bf16- or fp32-representable values:
    amax = max|x| (or the given maximum of the whole tensor x is a part of),
    s = 448 / amax (fp32), codes = encode(fp32(x * s))."""
    x32 = np.asarray(x, dtype=np.float32)
    if amax is None:
        amax = np.max(np.abs(x32)) if x32.size else 0.0
    amax = np.float32(amax)
    s = scale_of(amax)
    codes = encode((x32 * s).astype(np.float32))
    return codes, s, amax


def dequantize(codes, s) -> np.ndarray:
    """The values the codes stand for: decode(code) / s, in fp64."""
    return decode(codes) / np.float64(s)


def row_max_scores(q, k, causal, scale, rows):
    """max_{j in A_i} scale * q_i . k_j for the given rows of one head
    ([S, D] fp64 q, k): the largest score each row sees (the definition)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    out = np.empty(len(rows))
    for n, i in enumerate(rows):
        kk = k[: i + 1] if causal else k
        out[n] = np.max(scale * (kk @ q[i]))
    return out
