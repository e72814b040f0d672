"""The Python binding checks every tensor argument before it calls the C ABI.

The ABI sees plain pointers and cannot tell a buffer's size, so a tensor of
the wrong shape, dtype or device would be read or written out of bounds on the
GPU.  These tests run on the CPU: each call gets CPU tensors with exactly one
argument wrong and must raise a shape / dtype error naming that argument --
not the later "must be a CUDA tensor" error, and without any launch."""
import pytest
import torch

from long_sequence_context_b200 import cpattn as cp

B, H, S, D = 1, 2, 256, 64


def _t(shape=(B, H, S, D), dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def _bad(name, good):
    """A tensor like `good` with one more row (or a second dtype for 'dtype:')."""
    shape = list(good.shape)
    shape[-1 if len(shape) < 3 else 2] += 16
    return torch.zeros(shape, dtype=good.dtype)


def _expect_rejected(fn, name):
    n0 = cp.launch_count()
    with pytest.raises((ValueError, TypeError)) as e:
        fn()
    msg = str(e.value)
    assert name in msg and "CUDA tensor" not in msg, msg
    assert cp.launch_count() == n0


def _bwd_args():
    return dict(q=_t(), k=_t(), v=_t(), o=_t(), lse=_t((B, H, S), torch.float32), dout=_t())


@pytest.mark.parametrize("name", ["k", "v", "o", "lse", "dout"])
def test_bwd_rejects_each_input(name):
    a = _bwd_args()
    a[name] = _bad(name, a[name])
    _expect_rejected(lambda: cp.bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], 2), name)


@pytest.mark.parametrize("name", ["dq", "dk", "dv"])
def test_bwd_rejects_each_output(name):
    a = _bwd_args()
    out = {name: _bad(name, a["q"])}
    _expect_rejected(lambda: cp.bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], 2, **out), name)


@pytest.mark.parametrize("name", ["dq", "dk", "dv"])
def test_bwd_rejects_output_dtype(name):
    a = _bwd_args()
    out = {name: _t(dtype=torch.float32)}
    _expect_rejected(lambda: cp.bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], 2, **out), name)


@pytest.mark.parametrize("name", ["dq_acc", "dk_acc", "dv_acc"])
def test_bwd_accumulate_rejects_each_accumulator(name):
    a = _bwd_args()
    acc = {n: _t(dtype=torch.float32) for n in ("dq_acc", "dk_acc", "dv_acc")}
    acc[name] = _bad(name, acc[name])
    _expect_rejected(lambda: cp.bwd_accumulate_(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"],
                                                acc["dq_acc"], acc["dk_acc"], acc["dv_acc"], 2), name)


@pytest.mark.parametrize("name", ["k", "v", "dout", "o"])
def test_bwd_noalloc_rejects_each_input(name):
    a = _bwd_args()
    a[name] = _bad(name, a[name])
    _expect_rejected(lambda: cp.bwd_noalloc(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], 2), name)


@pytest.mark.parametrize("name", ["k", "v"])
def test_fwd_rejects_mismatched_inputs(name):
    a = _bwd_args()
    a[name] = _bad(name, a[name])
    _expect_rejected(lambda: cp.fwd(a["q"], a["k"], a["v"], 2), name)
    _expect_rejected(lambda: cp.fwd_step(a["q"], a["k"], a["v"], 2, 0), name)


def test_fwd_rejects_wrong_outputs():
    a = _bwd_args()
    _expect_rejected(lambda: cp.fwd(a["q"], a["k"], a["v"], 2, out=_bad("out", a["q"])), "out")
    _expect_rejected(lambda: cp.fwd(a["q"], a["k"], a["v"], 2, lse=_t((B, H, S + 16), torch.float32)), "lse")
    _expect_rejected(lambda: cp.fwd(a["q"], a["k"], a["v"], 2, lse=_t((B, H, S), torch.bfloat16)), "lse")


def test_fwd_rejects_dtype_mismatch():
    a = _bwd_args()
    _expect_rejected(lambda: cp.fwd(a["q"], _t(dtype=torch.float32), a["v"], 2), "k")


@pytest.mark.parametrize("name", ["lse_acc", "o_part", "lse_part"])
def test_merge_rejects_each_operand(name):
    ops = dict(o_acc=_t((64, D), torch.float32), lse_acc=_t((64,), torch.float32),
               o_part=_t((64, D), torch.float32), lse_part=_t((64,), torch.float32))
    ops[name] = _bad(name, ops[name])
    _expect_rejected(lambda: cp.merge_(ops["o_acc"], ops["lse_acc"], ops["o_part"], ops["lse_part"]), name)


def test_accumulate_rejects_mismatch():
    _expect_rejected(lambda: cp.accumulate_(_t((64,), torch.float32), _t((80,))), "x")
    _expect_rejected(lambda: cp.accumulate_(_t((64,), torch.bfloat16), _t((64,))), "acc")


def test_layer_bwd_rejects_wrong_lse():
    E = H * D
    x = _t((B, S, E))
    saved = (_t(), _t(), _t(), _t(), _t((B, H, S + 16), torch.float32))
    _expect_rejected(lambda: cp.layer_bwd(x, _t((3 * E, E)), _t((E, E)), saved, x, H, 2), "lse")


def test_well_formed_cpu_call_reaches_the_device_check():
    # with every shape right, the only complaint left is the device
    a = _bwd_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        cp.bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], 2)
