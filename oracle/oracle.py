"""Python front of the fp64 CPU oracle (oracle.c, built by oracle/build.py).

TEST INFRASTRUCTURE ONLY.  Imported by tests/, __graft_entry__.smoke() and
bench.py's CPU-baseline / reference leg; never by the product package.

Every function takes numpy arrays of shape [B, H, S, D] (or one head [S, D])
holding the exact (bf16- or fp32-rounded) input values, upcasts them to fp64
and loops over (batch, head) slices, optionally only a subset of heads.
What each C routine computes, and the passages it follows, is stated at the top
of oracle.c.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_L = ctypes.POINTER(ctypes.c_long)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        for name, argtypes in {
            "oracle_attn_fwd": [_D, _D, _D, ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                ctypes.c_double, _D, _D],
            "oracle_attn_fwd_rows": [_D, _D, _D, ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                     ctypes.c_double, _L, ctypes.c_long, _D, _D],
            "oracle_attn_bwd": [_D, _D, _D, _D, ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                ctypes.c_double, _D, _D, _D],
            "oracle_attn_bwd_dq_rows": [_D, _D, _D, _D, ctypes.c_long, ctypes.c_long,
                                        ctypes.c_int, ctypes.c_double, _L, ctypes.c_long, _D],
            "oracle_attn_bwd_kv_cols": [_D, _D, _D, _D, ctypes.c_long, ctypes.c_long,
                                        ctypes.c_int, ctypes.c_double, _L, ctypes.c_long, _D, _D],
            "oracle_ring_fwd": [_D, _D, _D, ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                ctypes.c_int, ctypes.c_double, _D, _D],
            "oracle_ring_step": [_D, _D, _D, ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                 ctypes.c_int, ctypes.c_double, ctypes.c_int, _D, _D],
            "oracle_merge": [_D, _D, _D, _D, ctypes.c_long, ctypes.c_long],
        }.items():
            fn = getattr(L, name)
            fn.argtypes = argtypes
            fn.restype = ctypes.c_int
        L.oracle_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def threads() -> int:
    return int(lib().oracle_threads())


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return a.ctypes.data_as(_D)


def _as4(x):
    x = _f64(x)
    if x.ndim == 2:
        x = x[None, None]
    assert x.ndim == 4
    return x


def _heads(B, H, heads):
    if heads is None:
        return [(b, h) for b in range(B) for h in range(H)]
    return [(b, h) for b in range(B) for h in heads]


def attn_fwd(q, k, v, causal, scale, heads=None):
    """O, LSE of full attention. Returns (o [B,H,S,D] or [B,len(heads),S,D], lse)."""
    q, k, v = _as4(q), _as4(k), _as4(v)
    B, H, S, D = q.shape
    hs = _heads(B, H, heads)
    nh = H if heads is None else len(heads)
    o = np.zeros((B, nh, S, D))
    lse = np.zeros((B, nh, S))
    for idx, (b, h) in enumerate(hs):
        hh = idx % nh
        ob = np.zeros((S, D))
        lb = np.zeros(S)
        rc = lib().oracle_attn_fwd(_p(_f64(q[b, h])), _p(_f64(k[b, h])), _p(_f64(v[b, h])), S, D,
                                   int(causal), float(scale), _p(ob), _p(lb))
        assert rc == 0
        o[b, hh], lse[b, hh] = ob, lb
    return o, lse


def attn_fwd_rows(q, k, v, causal, scale, b, h, rows):
    """O and LSE of the given rows of head (b, h)."""
    q, k, v = _as4(q), _as4(k), _as4(v)
    S, D = q.shape[2], q.shape[3]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.zeros((len(rows), D))
    lse = np.zeros(len(rows))
    rc = lib().oracle_attn_fwd_rows(_p(_f64(q[b, h])), _p(_f64(k[b, h])), _p(_f64(v[b, h])), S,
                                    D, int(causal), float(scale),
                                    rows.ctypes.data_as(_L), len(rows), _p(o), _p(lse))
    assert rc == 0
    return o, lse


def attn_bwd(q, k, v, dout, causal, scale, heads=None):
    """dQ, dK, dV of L = sum(O * dO)."""
    q, k, v, dout = _as4(q), _as4(k), _as4(v), _as4(dout)
    B, H, S, D = q.shape
    nh = H if heads is None else len(heads)
    dq = np.zeros((B, nh, S, D))
    dk = np.zeros((B, nh, S, D))
    dv = np.zeros((B, nh, S, D))
    for idx, (b, h) in enumerate(_heads(B, H, heads)):
        hh = idx % nh
        a, bb, c = np.zeros((S, D)), np.zeros((S, D)), np.zeros((S, D))
        rc = lib().oracle_attn_bwd(_p(_f64(q[b, h])), _p(_f64(k[b, h])), _p(_f64(v[b, h])),
                                   _p(_f64(dout[b, h])), S, D, int(causal), float(scale),
                                   _p(a), _p(bb), _p(c))
        assert rc == 0
        dq[b, hh], dk[b, hh], dv[b, hh] = a, bb, c
    return dq, dk, dv


def attn_bwd_dq_rows(q, k, v, dout, causal, scale, b, h, rows):
    q, k, v, dout = _as4(q), _as4(k), _as4(v), _as4(dout)
    S, D = q.shape[2], q.shape[3]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    dq = np.zeros((len(rows), D))
    rc = lib().oracle_attn_bwd_dq_rows(_p(_f64(q[b, h])), _p(_f64(k[b, h])), _p(_f64(v[b, h])),
                                       _p(_f64(dout[b, h])), S, D, int(causal), float(scale),
                                       rows.ctypes.data_as(_L), len(rows), _p(dq))
    assert rc == 0
    return dq


def attn_bwd_kv_cols(q, k, v, dout, causal, scale, b, h, cols):
    q, k, v, dout = _as4(q), _as4(k), _as4(v), _as4(dout)
    S, D = q.shape[2], q.shape[3]
    cols = np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
    dk = np.zeros((len(cols), D))
    dv = np.zeros((len(cols), D))
    rc = lib().oracle_attn_bwd_kv_cols(_p(_f64(q[b, h])), _p(_f64(k[b, h])), _p(_f64(v[b, h])),
                                       _p(_f64(dout[b, h])), S, D, int(causal), float(scale),
                                       cols.ctypes.data_as(_L), len(cols), _p(dk), _p(dv))
    assert rc == 0
    return dk, dv


def ring_fwd(q, k, v, cp_size, causal, scale, heads=None):
    """O, LSE by the zigzag ring with log-sum-exp merging (restated step by step)."""
    q, k, v = _as4(q), _as4(k), _as4(v)
    B, H, S, D = q.shape
    nh = H if heads is None else len(heads)
    o = np.zeros((B, nh, S, D))
    lse = np.zeros((B, nh, S))
    for idx, (b, h) in enumerate(_heads(B, H, heads)):
        hh = idx % nh
        ob, lb = np.zeros((S, D)), np.zeros(S)
        rc = lib().oracle_ring_fwd(_p(_f64(q[b, h])), _p(_f64(k[b, h])), _p(_f64(v[b, h])), S, D,
                                   int(cp_size), int(causal), float(scale), _p(ob), _p(lb))
        assert rc == 0, rc
        o[b, hh], lse[b, hh] = ob, lb
    return o, lse


def ring_step(q, k, v, cp_size, causal, scale, step, heads=None):
    """Partial (O, LSE) of every row at one ring step (LSE = -inf where all blocks SKIP)."""
    q, k, v = _as4(q), _as4(k), _as4(v)
    B, H, S, D = q.shape
    nh = H if heads is None else len(heads)
    o = np.zeros((B, nh, S, D))
    lse = np.zeros((B, nh, S))
    for idx, (b, h) in enumerate(_heads(B, H, heads)):
        hh = idx % nh
        ob, lb = np.zeros((S, D)), np.zeros(S)
        rc = lib().oracle_ring_step(_p(_f64(q[b, h])), _p(_f64(k[b, h])), _p(_f64(v[b, h])), S,
                                    D, int(cp_size), int(causal), float(scale), int(step),
                                    _p(ob), _p(lb))
        assert rc == 0, rc
        o[b, hh], lse[b, hh] = ob, lb
    return o, lse


def merge(o_acc, lse_acc, o_part, lse_part):
    """Log-sum-exp merge of two partial results, rows x D (returns new arrays)."""
    o_acc = _f64(o_acc).copy()
    lse_acc = _f64(lse_acc).copy()
    o_part = _f64(o_part)
    lse_part = _f64(lse_part)
    D = o_acc.shape[-1]
    rows = lse_acc.size
    rc = lib().oracle_merge(_p(o_acc), _p(lse_acc), _p(o_part), _p(lse_part), rows, D)
    assert rc == 0
    return o_acc, lse_acc
