"""GPU parity of the standalone log-sum-exp merge and the finalisation."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from tests.util import FP32_MAX, assert_lse_close, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cp():
    from long_sequence_context_b200 import cpattn
    return cpattn


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("rows", [1, 7, 1000, 4099])
def test_merge_matches_oracle(cp, D, rows):
    g = torch.Generator().manual_seed(rows + D)
    oa = torch.randn(rows, D, generator=g)
    ob = torch.randn(rows, D, generator=g)
    la = torch.randn(rows, generator=g) * 3
    lb = torch.randn(rows, generator=g) * 3
    # empty sides: -inf LSE (an empty side's O is ignored)
    la[::5] = float("-inf")
    lb[::7] = float("-inf")
    oa_ref, la_ref = orc.merge(np.where(np.isneginf(np64(la))[:, None], 0.0, np64(oa)), np64(la),
                               np64(ob), np64(lb))
    oa_d, la_d = oa.cuda(), la.cuda()
    cp.merge_(oa_d, la_d, ob.cuda(), lb.cuda())
    assert cp.sync_status() == cp.OK
    got = np64(oa_d)
    both_empty = np.isneginf(np64(la)) & np.isneginf(np64(lb))
    want = np.where(both_empty[:, None], np64(oa), oa_ref)
    assert np.max(np.abs(got - want)) <= FP32_MAX
    assert_lse_close(la_d.cpu(), la_ref)


def test_finalize_rounds_to_nearest_even(cp):
    x = torch.randn(513, 128, generator=torch.Generator().manual_seed(3))
    y = cp.finalize(x.cuda(), torch.bfloat16)
    assert torch.equal(y.cpu(), x.to(torch.bfloat16))
    z = cp.finalize(x.cuda(), torch.float32)
    assert torch.equal(z.cpu(), x)
