"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, the host planner equals the plan oracle exactly, and
argument errors come back as status codes before any GPU work."""
import ctypes
import os
import re

import pytest

from oracle import plan as oplan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cpattn.h")


@pytest.fixture(scope="module")
def cp():
    from long_sequence_context_b200 import build
    build.build()
    from long_sequence_context_b200 import cpattn
    return cpattn


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cpattn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("cpattn_plan", "cpattn_fwd", "cpattn_fwd_step", "cpattn_merge", "cpattn_bwd",
              "cpattn_bwd_workspace_bytes", "cpattn_finalize", "cpattn_sync_status"):
        assert n in names


def test_library_exports_every_declared_symbol(cp):
    lib = ctypes.CDLL(cp.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert sorted(cp.EXPORTS) == declared_functions()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("cp_size", [1, 2, 3, 4, 8, 16])
def test_plan_equals_plan_oracle(cp, cp_size, causal):
    S = (2 if causal else 1) * cp_size * 128
    assert cp.plan(S, cp_size, causal) == oplan.plan_rows(S, cp_size, causal)


def test_plan_golden_cp4(cp):
    rows = cp.plan(8 * 64, 4, True)
    owned = {}
    for r, t, a, b, src, kind in rows:
        if t == 0:
            owned.setdefault(r, set()).add(a)
    assert owned == {0: {0, 7}, 1: {1, 6}, 2: {2, 5}, 3: {3, 4}}


def test_plan_errors(cp):
    n = ctypes.c_int(-1)
    assert cp.lib.cpattn_plan(100, 4, 1, None, 0, ctypes.byref(n)) == cp.ERR_SHAPE
    assert cp.lib.cpattn_plan(128, 4, 1, None, 0, ctypes.byref(n)) == cp.ERR_ARG
    assert n.value == 64
    buf = (ctypes.c_int32 * 6)()
    assert cp.lib.cpattn_plan(128, 4, 1, buf, 1, ctypes.byref(n)) == cp.ERR_ARG
    assert cp.lib.cpattn_plan(128, 0, 1, buf, 1, ctypes.byref(n)) == cp.ERR_SHAPE


def _fwd_status(cp, S=256, D=128, cp_size=2, causal=1, scale=0.1, dtype=0, ptr=256, B=1, H=1):
    p = ctypes.c_void_p(ptr)
    return cp.lib.cpattn_fwd(p, p, p, p, p, B, H, S, D, cp_size, causal, scale, dtype, None)


def test_argument_errors_are_reported_before_launch(cp):
    assert _fwd_status(cp, S=102) == cp.ERR_SHAPE          # not a multiple of 2*cp_size
    assert _fwd_status(cp, S=2 * 2 * 8 + 2) == cp.ERR_SHAPE  # 34 rows: not 4 whole chunks
    assert _fwd_status(cp, D=96) == cp.ERR_SHAPE
    assert _fwd_status(cp, cp_size=0) == cp.ERR_SHAPE
    assert _fwd_status(cp, B=0) == cp.ERR_SHAPE
    assert _fwd_status(cp, dtype=7) == cp.ERR_DTYPE
    assert _fwd_status(cp, scale=0.0) == cp.ERR_ARG
    assert _fwd_status(cp, scale=float("nan")) == cp.ERR_ARG
    assert _fwd_status(cp, ptr=0) == cp.ERR_ARG
    assert _fwd_status(cp, ptr=258) == cp.ERR_ALIGN
    p = ctypes.c_void_p(256)
    assert cp.lib.cpattn_fwd_step(p, p, p, p, p, 1, 1, 256, 128, 2, 1, 0.1, 2, 0, None) == cp.ERR_ARG
    assert cp.lib.cpattn_merge(p, p, p, p, -1, 128, None) == cp.ERR_SHAPE
    assert cp.lib.cpattn_merge(p, p, p, p, 0, 128, None) == cp.OK
    assert cp.lib.cpattn_finalize(p, p, 10, 128, 5, None) == cp.ERR_DTYPE
    # backward: workspace checks
    need = cp.bwd_workspace_bytes(1, 1, 256, 128)
    assert need >= 2 * 256 * 4
    args = [p] * 9 + [1, 1, 256, 128, 2, 1, 0.1]
    assert cp.lib.cpattn_bwd(*args, None, need, 0, None) == cp.ERR_WORKSPACE
    assert cp.lib.cpattn_bwd(*args, p, need - 1, 0, None) == cp.ERR_WORKSPACE
    assert cp.lib.cpattn_bwd(*args, ctypes.c_void_p(256 + 16), need, 0, None) == cp.ERR_ALIGN
    assert cp.bwd_workspace_bytes(1, 1, 256, 96) == 0


def test_layer_argument_errors_are_reported_before_launch(cp):
    p = ctypes.c_void_p(256)
    B, S, E, H = 1, 256, 256, 2
    need = cp.layer_workspace_bytes(B, S, E, H)
    assert need > 0 and cp.layer_workspace_bytes(B, S, 96, 1) == 0 and cp.layer_workspace_bytes(B, S, 256, 3) == 0

    def fwd(ptr=p, S=S, E=E, H=H, cp_size=2, scale=0.1, ws=p, ws_bytes=need):
        return cp.lib.cpattn_layer_fwd(*([ptr] + [p] * 10), B, S, E, H, cp_size, 1, scale, ws, ws_bytes, None)

    def bwd(ptr=p, S=S, E=E, H=H, cp_size=2, ws_bytes=need):
        return cp.lib.cpattn_layer_bwd(*([ptr] + [p] * 13), B, S, E, H, cp_size, 1, 0.1, p, ws_bytes, None)

    assert fwd(E=96, H=1) == cp.ERR_SHAPE          # D = 96
    assert fwd(E=256, H=3) == cp.ERR_SHAPE         # E not a multiple of H
    assert fwd(ptr=None) == cp.ERR_ARG
    assert fwd(ptr=ctypes.c_void_p(258)) == cp.ERR_ALIGN
    assert fwd(scale=0.0) == cp.ERR_ARG
    assert fwd(ws=None) == cp.ERR_WORKSPACE
    assert fwd(ws_bytes=need - 1) == cp.ERR_WORKSPACE
    assert fwd(S=100, ws_bytes=cp.layer_workspace_bytes(B, 100, E, H)) == cp.ERR_SHAPE  # B*S % 8 != 0
    assert bwd(ptr=None) == cp.ERR_ARG
    assert bwd(ws_bytes=need - 1) == cp.ERR_WORKSPACE
    assert bwd(cp_size=0) == cp.ERR_SHAPE


def test_accumulate_argument_errors(cp):
    p = ctypes.c_void_p(256)
    assert cp.lib.cpattn_accumulate(p, p, 6, 0, None) == cp.ERR_SHAPE
    assert cp.lib.cpattn_accumulate(p, p, -4, 0, None) == cp.ERR_SHAPE
    assert cp.lib.cpattn_accumulate(p, p, 8, 7, None) == cp.ERR_DTYPE
    assert cp.lib.cpattn_accumulate(None, p, 8, 0, None) == cp.ERR_ARG
    assert cp.lib.cpattn_accumulate(p, ctypes.c_void_p(258), 8, 0, None) == cp.ERR_ALIGN
    assert cp.lib.cpattn_accumulate(p, p, 0, 0, None) == cp.OK


def test_status_strings(cp):
    for s in range(8):
        assert cp.status_str(s)
    assert cp.status_str(99) == "unknown status"


def test_set_path_roundtrip(cp):
    prev = cp.set_path(1)
    assert cp.set_path(prev) == 1


def test_set_path_values(cp):
    """0 automatic, 1 CUDA cores, 2 tcgen05 on one SM each; anything else is 0."""
    prev = cp.set_path(2)
    try:
        assert cp.set_path(7) == 2
        assert cp.set_path(1) == 0
        assert cp.set_path(-3) == 1
        assert cp.set_path(0) == 0
    finally:
        cp.set_path(prev)
