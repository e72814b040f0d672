"""Attention layer (projections + head reshapes + ring attention) on the GPU
against the fp64 layer oracle (oracle/layer.py).

Tolerance.  The layer's outputs pass through several bf16 roundings (q/k/v,
O, the merged heads, dO, dQ/dK/dV, the outputs themselves: relative 2^-9
each) and the weight and bias gradients are sums over B*S rows, so the check
is relative to the reference's scale: max |err| <= 2e-2 * max |ref| and
||err||_F <= 1e-2 * ||ref||_F for every output (the error of rounding the
reference itself to bf16 is ~2e-3 in the second measure).
"""
import numpy as np
import pytest
import torch

from long_sequence_context_b200 import cpattn as cp
from long_sequence_context_b200.inputs import make_layer_inputs
from oracle import layer as olayer

pytestmark = pytest.mark.gpu


def assert_rel(got, want, name, max_rel=2e-2, fro_rel=1e-2):
    got = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - want)
    scale_max, scale_fro = np.abs(want).max(), np.linalg.norm(want)
    assert np.isfinite(got).all(), name
    assert err.max() <= max_rel * scale_max, f"{name}: max err {err.max():.3e} vs max |ref| {scale_max:.3e}"
    assert np.linalg.norm(err) <= fro_rel * scale_fro, \
        f"{name}: rel Frobenius err {np.linalg.norm(err) / scale_fro:.3e}"


@pytest.mark.parametrize("B,S,E,H,cp_size,causal", [
    (1, 1024, 256, 2, 2, True),    # D = 128, tcgen05 attention
    (2, 512, 256, 4, 1, False),    # D = 64, non-causal
    (1, 96, 128, 1, 3, True),      # chunk 16 rows: CUDA-core attention
])
def test_layer_fwd_bwd_matches_oracle(B, S, E, H, cp_size, causal):
    x, w_qkv, b_qkv, w_o, b_o, dy = make_layer_inputs(B, S, E, seed=11)
    scale = (E // H) ** -0.5
    dev = [t.cuda() for t in (x, w_qkv, b_qkv, w_o, b_o, dy)]
    y, saved = cp.layer_fwd(*dev[:5], H, cp_size, causal, scale)
    grads = cp.layer_bwd(dev[0], dev[1], dev[3], saved, dev[5], H, cp_size, causal, scale)
    cp.check_device_status()
    ref = olayer.layer_bwd(*(t.double().numpy() for t in (x, w_qkv, b_qkv, w_o, b_o, dy)),
                           H, causal, scale)
    assert_rel(y, ref["y"], "y")
    for name, g in zip(("dx", "dw_qkv", "db_qkv", "dw_o", "db_o"), grads):
        assert_rel(g, ref[name], name)


def test_layer_saved_attention_matches_the_attention_call():
    # the q, k, v, o, lse the layer saves are those of its own projections, and
    # o / lse equal a direct cpattn_fwd on them (bitwise: same kernels, inputs)
    B, S, E, H = 1, 512, 256, 2
    x, w_qkv, b_qkv, w_o, b_o, _ = (t.cuda() for t in make_layer_inputs(B, S, E, seed=5))
    _, (q, k, v, o, lse) = cp.layer_fwd(x, w_qkv, b_qkv, w_o, b_o, H, 2, True)
    o2, lse2 = cp.fwd(q, k, v, 2, True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    qkv = (x.double() @ w_qkv.double().T + b_qkv.double()).view(B, S, 3, H, E // H)
    ref_q = qkv[:, :, 0].transpose(1, 2)
    assert (q.double() - ref_q).abs().max().item() <= 2e-2 * ref_q.abs().max().item()


def test_layer_rejects_bad_arguments():
    x, w_qkv, b_qkv, w_o, b_o, _ = (t.cuda() for t in make_layer_inputs(1, 64, 96, seed=1))
    with pytest.raises(cp.CpattnError) as e:   # D = 96 / 1 is not 64 or 128
        cp.layer_fwd(x, w_qkv, b_qkv, w_o, b_o, 1, 1, True)
    assert e.value.status == cp.ERR_SHAPE
    x, w_qkv, b_qkv, w_o, b_o, _ = (t.cuda() for t in make_layer_inputs(1, 100, 128, seed=1))
    with pytest.raises(cp.CpattnError) as e:   # B * S = 100 rows: the GEMMs take multiples of 8
        cp.layer_fwd(x, w_qkv, b_qkv, w_o, b_o, 1, 2, True)
    assert e.value.status == cp.ERR_SHAPE
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    x, w_qkv, b_qkv, w_o, b_o, _ = (t.cuda() for t in make_layer_inputs(1, 64, 128, seed=1))
    with pytest.raises(cp.CpattnError) as e:
        cp.layer_fwd(x, w_qkv, b_qkv, w_o, b_o, 1, 1, True, workspace=small)
    assert e.value.status == cp.ERR_WORKSPACE
