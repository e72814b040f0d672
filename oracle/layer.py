"""fp64 oracle of the attention layer around the ring attention.

TEST INFRASTRUCTURE ONLY.  Imported by tests/ and by bench.py's CPU-baseline
leg; never by the product package.

What it computes, from the exact (bf16-rounded) inputs upcast to fp64, with no
intermediate rounding ("Configuring RingAttention+FlashAttention for CP",
section 3 code: q/k/v_proj and out_proj are nn.Linear(E, E) with bias, the
heads are q.view(B, S, H, D).transpose(1, 2), the ring attention's output is
transposed back and projected):

    [q | k | v] = x Wqkv^T + bqkv          (Wqkv = the three weights stacked)
    q, k, v     -> [B, H, S, D]            (split_heads)
    O, LSE      = attention(q, k, v)        (oracle.attn_fwd: the definition)
    Om          = merge_heads(O)            [B, S, E]
    y           = Om Wo^T + bo

and the gradients of L = sum(y * dy) by the chain rule, with the attention's
own gradient from oracle.attn_bwd:

    dWo = sum_rows dy^T Om,  dbo = sum_rows dy,  dOm = dy Wo
    dq, dk, dv = attention backward of split_heads(dOm)
    dQKV = [merge(dq) | merge(dk) | merge(dv)]
    dWqkv = sum_rows dQKV^T x,  dbqkv = sum_rows dQKV,  dx = dQKV Wqkv

Matrix products use numpy's matmul / einsum as library primitives.
"""
import numpy as np

from . import oracle


def split_heads(t, H):
    """[B, S, E] -> [B, H, S, D]"""
    B, S, E = t.shape
    return np.ascontiguousarray(t.reshape(B, S, H, E // H).transpose(0, 2, 1, 3))


def merge_heads(t):
    """[B, H, S, D] -> [B, S, E]"""
    B, H, S, D = t.shape
    return np.ascontiguousarray(t.transpose(0, 2, 1, 3).reshape(B, S, H * D))


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def layer_fwd(x, w_qkv, b_qkv, w_o, b_o, H, causal, scale):
    """Returns (y [B,S,E], saved dict with q, k, v, o, lse, om)."""
    x, w_qkv, b_qkv, w_o, b_o = map(_f64, (x, w_qkv, b_qkv, w_o, b_o))
    E = x.shape[-1]
    qkv = x @ w_qkv.T + b_qkv
    q = split_heads(qkv[..., :E], H)
    k = split_heads(qkv[..., E:2 * E], H)
    v = split_heads(qkv[..., 2 * E:], H)
    o, lse = oracle.attn_fwd(q, k, v, causal, scale)
    om = merge_heads(o)
    y = om @ w_o.T + b_o
    return y, {"q": q, "k": k, "v": v, "o": o, "lse": lse, "om": om}


def layer_bwd(x, w_qkv, b_qkv, w_o, b_o, dy, H, causal, scale):
    """Returns dict with dx, dw_qkv, db_qkv, dw_o, db_o (and the forward's y)."""
    x, w_qkv, w_o, dy = map(_f64, (x, w_qkv, w_o, dy))
    y, c = layer_fwd(x, w_qkv, b_qkv, w_o, b_o, H, causal, scale)
    rows = lambda t: t.reshape(-1, t.shape[-1])
    dw_o = rows(dy).T @ rows(c["om"])
    db_o = dy.sum(axis=(0, 1))
    dom = dy @ w_o
    dq, dk, dv = oracle.attn_bwd(c["q"], c["k"], c["v"], split_heads(dom, H), causal, scale)
    dqkv = np.concatenate([merge_heads(dq), merge_heads(dk), merge_heads(dv)], axis=-1)
    dw_qkv = rows(dqkv).T @ rows(x)
    db_qkv = dqkv.sum(axis=(0, 1))
    dx = dqkv @ w_qkv
    return {"y": y, "dx": dx, "dw_qkv": dw_qkv, "db_qkv": db_qkv, "dw_o": dw_o, "db_o": db_o}
