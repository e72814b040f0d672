"""Shared helpers for the parity tests: tolerances, comparisons against the
oracle, and the row / column samples used at full workload sizes."""
import numpy as np
import torch

# error bars: bf16 outputs max-abs 2e-2 and mean-abs 2e-3, fp32 outputs 1e-4,
# LSE 1e-3 (natural-log units)
BF16_MAX, BF16_MEAN = 2e-2, 2e-3
FP32_MAX = 1e-4
LSE_MAX = 1e-3


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got, want, dtype, what=""):
    got = np64(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - want)
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    if dtype == torch.float32:
        assert mx <= FP32_MAX, f"{what}: max-abs {mx:.3e} > {FP32_MAX}"
    else:
        assert mx <= BF16_MAX and mean <= BF16_MEAN, \
            f"{what}: max-abs {mx:.3e} (bar {BF16_MAX}), mean-abs {mean:.3e} (bar {BF16_MEAN})"
    return mx, mean


def assert_lse_close(got, want, what="lse"):
    got = np64(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    both_inf = np.isneginf(got) & np.isneginf(want)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    err = np.abs(np.where(both_inf, 0.0, got - want))
    mx = float(err.max(initial=0.0))
    assert mx <= LSE_MAX, f"{what}: max-abs {mx:.3e} > {LSE_MAX}"
    return mx


def sample_rows(S, n_chunks, n_total=128, seed=0):
    """First and last row of every chunk plus seeded random rows."""
    c = S // n_chunks
    rows = set()
    for a in range(n_chunks):
        rows.add(a * c)
        rows.add(a * c + c - 1)
    g = np.random.default_rng(seed)
    while len(rows) < min(n_total, S):
        rows.add(int(g.integers(S)))
    return np.array(sorted(rows), dtype=np.int64)
