"""Pins of the attention-layer oracle (oracle/layer.py), CPU only.

The layer oracle composes the attention oracle with the projections and head
reshapes of "Configuring RingAttention+FlashAttention for CP", section 3 code.
It is pinned here against an independent formulation: torch's own nn.Linear
arithmetic (F.linear), view/transpose head reshapes and
F.scaled_dot_product_attention, differentiated by torch autograd in fp64 --
a plausible slip in the oracle (a transposed weight, the q/k/v stacking order,
a missing bias gradient, a head reshape in the wrong order) fails one of them.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from long_sequence_context_b200.inputs import make_layer_inputs
from oracle import layer as olayer


def torch_layer(x, w_qkv, b_qkv, w_o, b_o, H, causal, scale):
    B, S, E = x.shape
    D = E // H
    wq, wk, wv = w_qkv[:E], w_qkv[E:2 * E], w_qkv[2 * E:]
    bq, bk, bv = b_qkv[:E], b_qkv[E:2 * E], b_qkv[2 * E:]

    def heads(t):
        return t.view(B, S, H, D).transpose(1, 2)

    q, k, v = heads(F.linear(x, wq, bq)), heads(F.linear(x, wk, bk)), heads(F.linear(x, wv, bv))
    o = F.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=scale)
    return F.linear(o.transpose(1, 2).reshape(B, S, E), w_o, b_o)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,S,E,H", [(2, 16, 16, 2), (1, 12, 24, 3)])
def test_layer_oracle_matches_torch_autograd(B, S, E, H, causal):
    x, w_qkv, b_qkv, w_o, b_o, dy = (t.double() for t in make_layer_inputs(B, S, E, seed=7))
    scale = (E // H) ** -0.5
    got = olayer.layer_bwd(x.numpy(), w_qkv.numpy(), b_qkv.numpy(), w_o.numpy(), b_o.numpy(),
                           dy.numpy(), H, causal, scale)
    params = [t.clone().requires_grad_(True) for t in (x, w_qkv, b_qkv, w_o, b_o)]
    y = torch_layer(*params, H, causal, scale)
    (y * dy).sum().backward()
    want = {"y": y.detach(), "dx": params[0].grad, "dw_qkv": params[1].grad,
            "db_qkv": params[2].grad, "dw_o": params[3].grad, "db_o": params[4].grad}
    for name, ref in want.items():
        np.testing.assert_allclose(got[name], ref.numpy(), rtol=0, atol=1e-10, err_msg=name)


def test_layer_with_identity_projections_is_the_attention():
    # Wqkv = [I; I; I], Wo = I, zero biases: y = merge(attention(split(x) x3))
    B, S, E, H = 1, 10, 8, 2
    x = make_layer_inputs(B, S, E, seed=3)[0].double().numpy()
    eye = np.eye(E)
    y, _ = olayer.layer_fwd(x, np.concatenate([eye, eye, eye]), np.zeros(3 * E), eye, np.zeros(E),
                            H, True, 0.5)
    xs = olayer.split_heads(x, H)
    # the attention of one head written out for this check: softmax over j <= i
    want = np.zeros_like(xs)
    for h in range(H):
        s = 0.5 * xs[0, h] @ xs[0, h].T
        s = np.where(np.tril(np.ones((S, S), bool)), s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        want[0, h] = (p / p.sum(axis=1, keepdims=True)) @ xs[0, h]
    np.testing.assert_allclose(y, olayer.merge_heads(want), rtol=0, atol=1e-12)


def test_head_reshapes_are_inverse_and_match_view_transpose():
    t = np.arange(2 * 5 * 12, dtype=np.float64).reshape(2, 5, 12)
    h = olayer.split_heads(t, 3)
    ref = torch.from_numpy(t).view(2, 5, 3, 4).transpose(1, 2).numpy()
    assert np.array_equal(h, ref)
    assert np.array_equal(olayer.merge_heads(h), t)
