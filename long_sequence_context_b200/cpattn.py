"""Python binding of libcpattn.so (the C ABI declared in include/cpattn.h).

Argument marshalling only: every function checks device / dtype / contiguity,
passes raw device pointers and the current CUDA stream to the library, and
turns a non-zero status into an exception.  All arithmetic runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback.  If the shared
library has not been built, importing this module raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcpattn.so")

OK, ERR_ARG, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(8)
BF16, FP32 = 0, 1
SKIP, FULL, DIAG = 0, 1, 2
PLAN_FIELDS = 6

# every symbol include/cpattn.h declares
EXPORTS = ["cpattn_plan", "cpattn_fwd", "cpattn_fwd_step", "cpattn_merge", "cpattn_finalize",
           "cpattn_bwd_workspace_bytes", "cpattn_bwd", "cpattn_sync_status",
           "cpattn_status_str", "cpattn_launch_count", "cpattn_set_path", "cpattn_last_path",
           "cpattn_debug_stall", "cpattn_profile", "cpattn_profile_read", "cpattn_bwd_noalloc",
           "cpattn_layer_workspace_bytes", "cpattn_layer_fwd", "cpattn_layer_bwd",
           "cpattn_accumulate", "cpattn_bwd_accumulate", "cpattn_gemm", "cpattn_amax",
           "cpattn_quantize_e4m3", "cpattn_fwd_fp8"]

# size of the library's fixed scratch array behind bwd_noalloc
NOALLOC_SCRATCH_BYTES = 64 << 20


class CpattnError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m long_sequence_context_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, l, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_long, ctypes.c_size_t
    sigs = {
        "cpattn_plan": ([i, i, i, vp, i, ctypes.POINTER(ctypes.c_int)], i),
        "cpattn_fwd": ([vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp], i),
        "cpattn_fwd_step": ([vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp], i),
        "cpattn_merge": ([vp, vp, vp, vp, l, i, vp], i),
        "cpattn_finalize": ([vp, vp, l, i, i, vp], i),
        "cpattn_bwd_workspace_bytes": ([i, i, i, i], sz),
        "cpattn_bwd": ([vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, sz, i, vp], i),
        "cpattn_bwd_accumulate": ([vp] * 9 + [i, i, i, i, i, i, f, vp, sz, i, vp], i),
        "cpattn_sync_status": ([vp], i),
        "cpattn_status_str": ([i], ctypes.c_char_p),
        "cpattn_launch_count": ([], ctypes.c_longlong),
        "cpattn_set_path": ([i], i),
        "cpattn_last_path": ([], i),
        "cpattn_debug_stall": ([i], i),
        "cpattn_bwd_noalloc": ([vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp], i),
        "cpattn_profile": ([i], i),
        "cpattn_profile_read": ([i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)], i),
        "cpattn_layer_workspace_bytes": ([i, i, i, i], sz),
        "cpattn_accumulate": ([vp, vp, l, i, vp], i),
        "cpattn_layer_fwd": ([vp] * 11 + [i] * 6 + [f, vp, sz, vp], i),
        "cpattn_gemm": ([vp, vp, vp, vp, i, i, i, i, i, vp], i),
        "cpattn_amax": ([vp, l, i, vp, vp], i),
        "cpattn_quantize_e4m3": ([vp, i, i, i, i, i, vp, vp, vp], i),
        "cpattn_fwd_fp8": ([vp] * 6 + [i] * 6 + [f, vp], i),
        "cpattn_layer_bwd": ([vp] * 14 + [i] * 6 + [f, vp, sz, vp], i),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


lib = _load()


def status_str(status: int) -> str:
    return lib.cpattn_status_str(int(status)).decode()


def _check(status, where):
    if status != OK:
        raise CpattnError(status, where)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _expect(t, name: str, shape, dtype, like=None):
    """Shape / dtype / device check of one tensor argument.  The C ABI sees
    plain pointers, so a wrong-sized buffer would be read or written out of
    bounds on the device: every tensor is checked here before any call."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if like is not None and t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, expected {like.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _qkv(q, k, v):
    """Checks q, k, v ([B, H, S, D], one dtype, one device); returns the shape."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a [B, H, S, D] tensor")
    _dtype_code(q)
    for t, n in ((k, "k"), (v, "v")):
        _expect(t, n, q.shape, q.dtype, q)
    _expect(q, "q", q.shape, q.dtype)
    return tuple(q.shape)


def plan(S: int, cp_size: int, causal: bool):
    """Ring schedule rows (r, t, q_chunk, kv_chunk, src_rank, kind); host only."""
    n = ctypes.c_int(0)
    st = lib.cpattn_plan(S, cp_size, int(causal), None, 0, ctypes.byref(n))
    if st not in (OK, ERR_ARG) or n.value == 0:
        _check(st if st != OK else ERR_SHAPE, "cpattn_plan")
    buf = (ctypes.c_int32 * (n.value * PLAN_FIELDS))()
    _check(lib.cpattn_plan(S, cp_size, int(causal), buf, n.value, ctypes.byref(n)), "cpattn_plan")
    flat = list(buf)
    return [tuple(flat[r * PLAN_FIELDS:(r + 1) * PLAN_FIELDS]) for r in range(n.value)]


def fwd(q, k, v, cp_size: int, causal: bool = True, scale=None, out=None, lse=None, stream=None):
    """Ring forward: returns (o, lse) with o like q and lse fp32 [B, H, S]."""
    B, H, S, D = _qkv(q, k, v)
    scale = float(scale if scale is not None else D ** -0.5)
    if out is not None:
        _expect(out, "out", q.shape, q.dtype, q)
    if lse is not None:
        _expect(lse, "lse", (B, H, S), torch.float32, q)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, S), dtype=torch.float32, device=q.device) if lse is None else lse
    st = lib.cpattn_fwd(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse_t, "lse"),
                        B, H, S, D, cp_size, int(causal), scale, _dtype_code(q), _stream(stream))
    _check(st, "cpattn_fwd")
    return o, lse_t


def fwd_step(q, k, v, cp_size: int, step: int, causal: bool = True, scale=None, stream=None):
    """One ring step for every virtual rank: fp32 partial (o_part, lse_part)."""
    B, H, S, D = _qkv(q, k, v)
    scale = float(scale if scale is not None else D ** -0.5)
    o = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    st = lib.cpattn_fwd_step(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o_part"),
                             _dev(lse, "lse_part"), B, H, S, D, cp_size, int(causal), scale, step,
                             _dtype_code(q), _stream(stream))
    _check(st, "cpattn_fwd_step")
    return o, lse


def merge_(o_acc, lse_acc, o_part, lse_part, stream=None):
    """In-place log-sum-exp merge of (o_part, lse_part) into (o_acc, lse_acc):
    o tensors [..., D] fp32, lse tensors the same leading shape, fp32."""
    if not isinstance(o_acc, torch.Tensor) or o_acc.dim() < 1:
        raise ValueError("o_acc must be a [..., D] tensor")
    D = o_acc.shape[-1]
    lead = tuple(o_acc.shape[:-1])
    _expect(o_acc, "o_acc", o_acc.shape, torch.float32)
    _expect(lse_acc, "lse_acc", lead, torch.float32, o_acc)
    _expect(o_part, "o_part", o_acc.shape, torch.float32, o_acc)
    _expect(lse_part, "lse_part", lead, torch.float32, o_acc)
    rows = lse_acc.numel()
    st = lib.cpattn_merge(_dev(o_acc, "o_acc"), _dev(lse_acc, "lse_acc"), _dev(o_part, "o_part"),
                          _dev(lse_part, "lse_part"), rows, D, _stream(stream))
    _check(st, "cpattn_merge")
    return o_acc, lse_acc


def finalize(o_acc, dtype=torch.bfloat16, stream=None):
    """fp32 [..., D] -> a new tensor of `dtype` (round to nearest even)."""
    if not isinstance(o_acc, torch.Tensor) or o_acc.dim() < 1:
        raise ValueError("o_acc must be a [..., D] tensor")
    _expect(o_acc, "o_acc", o_acc.shape, torch.float32)
    D = o_acc.shape[-1]
    o = torch.empty(o_acc.shape, dtype=dtype, device=o_acc.device)
    st = lib.cpattn_finalize(_dev(o_acc, "o_acc"), _dev(o, "o"), o_acc.numel() // D, D,
                             _dtype_code(o), _stream(stream))
    _check(st, "cpattn_finalize")
    return o


def bwd_workspace_bytes(B, H, S, D) -> int:
    return int(lib.cpattn_bwd_workspace_bytes(B, H, S, D))


def _bwd_args(q, k, v, o, lse, dout):
    B, H, S, D = _qkv(q, k, v)
    _expect(o, "o", q.shape, q.dtype, q)
    _expect(dout, "dout", q.shape, q.dtype, q)
    _expect(lse, "lse", (B, H, S), torch.float32, q)
    return B, H, S, D


def _workspace(workspace, need, q):
    if workspace is None:
        return torch.empty(need, dtype=torch.uint8, device=q.device)
    if not isinstance(workspace, torch.Tensor) or workspace.device != q.device:
        raise ValueError(f"workspace must be a tensor on {q.device}")
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace holds {workspace.numel() * workspace.element_size()} bytes, "
                         f"{need} needed")
    return workspace


def bwd(q, k, v, o, lse, dout, cp_size: int, causal: bool = True, scale=None, workspace=None,
        dq=None, dk=None, dv=None, stream=None):
    """Recompute backward: returns (dq, dk, dv) like q."""
    B, H, S, D = _bwd_args(q, k, v, o, lse, dout)
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        if t is not None:
            _expect(t, n, q.shape, q.dtype, q)
    scale = float(scale if scale is not None else D ** -0.5)
    workspace = _workspace(workspace, bwd_workspace_bytes(B, H, S, D), q)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    st = lib.cpattn_bwd(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"),
                        _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"),
                        B, H, S, D, cp_size, int(causal), scale,
                        ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size(),
                        _dtype_code(q), _stream(stream))
    _check(st, "cpattn_bwd")
    return dq, dk, dv


def bwd_accumulate_(q, k, v, o, lse, dout, dq_acc, dk_acc, dv_acc, cp_size: int,
                    causal: bool = True, scale=None, workspace=None, stream=None):
    """Recompute backward whose gradients are added, in fp32, into the fp32
    accumulators dq_acc, dk_acc, dv_acc (each shaped like q).  Returns them."""
    B, H, S, D = _bwd_args(q, k, v, o, lse, dout)
    for t, n in ((dq_acc, "dq_acc"), (dk_acc, "dk_acc"), (dv_acc, "dv_acc")):
        _expect(t, n, q.shape, torch.float32, q)
    if len({dq_acc.data_ptr(), dk_acc.data_ptr(), dv_acc.data_ptr()}) != 3:
        raise ValueError("dq_acc, dk_acc, dv_acc must be distinct tensors")
    scale = float(scale if scale is not None else D ** -0.5)
    workspace = _workspace(workspace, bwd_workspace_bytes(B, H, S, D), q)
    st = lib.cpattn_bwd_accumulate(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"),
        _dev(dout, "dout"), _dev(dq_acc, "dq_acc"), _dev(dk_acc, "dk_acc"), _dev(dv_acc, "dv_acc"),
        B, H, S, D, cp_size, int(causal), scale, ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), _dtype_code(q), _stream(stream))
    _check(st, "cpattn_bwd_accumulate")
    return dq_acc, dk_acc, dv_acc


def bwd_noalloc(q, k, v, o, lse, dout, cp_size: int, causal: bool = True, scale=None,
                dq=None, dk=None, dv=None, stream=None):
    """Backward without a caller workspace: the library's fixed device scratch
    array stands in for it (see cpattn_bwd_noalloc in include/cpattn.h).  For
    callers that cannot allocate device memory, pass preallocated dq/dk/dv;
    calls that may overlap on the GPU must be serialised by the caller."""
    B, H, S, D = _bwd_args(q, k, v, o, lse, dout)
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        if t is not None:
            _expect(t, n, q.shape, q.dtype, q)
    scale = float(scale if scale is not None else D ** -0.5)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    st = lib.cpattn_bwd_noalloc(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"),
                                _dev(lse, "lse"), _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"),
                                _dev(dv, "dv"), B, H, S, D, cp_size, int(causal), scale,
                                _dtype_code(q), _stream(stream))
    _check(st, "cpattn_bwd_noalloc")
    return dq, dk, dv


def accumulate_(acc, x, stream=None):
    """acc += x (acc fp32, x bf16 or fp32, same shape)."""
    _expect(acc, "acc", acc.shape, torch.float32)
    if not isinstance(x, torch.Tensor):
        raise TypeError("x must be a torch.Tensor")
    _dtype_code(x)
    _expect(x, "x", acc.shape, x.dtype, acc)
    _check(lib.cpattn_accumulate(_dev(acc, "acc"), _dev(x, "x"), acc.numel(), _dtype_code(x),
                                 _stream(stream)), "cpattn_accumulate")
    return acc


def gemm(a, b, bias=None, a_t: bool = False, b_t: bool = False, out=None, stream=None):
    """C = op(a) op(b) (+ bias) on the library's tcgen05 GEMM, bf16, fp32 accumulation.
    a: [M, K] (a_t: [K, M], used transposed); b: [N, K] as an nn.Linear weight
    (C = a b^T), or with b_t: [K, N] (C = a b).  bias: [N] or None."""
    for t, n in ((a, "a"), (b, "b")):
        if not isinstance(t, torch.Tensor) or t.dim() != 2:
            raise ValueError(f"{n} must be a 2-D tensor")
    M, K = (a.shape[1], a.shape[0]) if a_t else (a.shape[0], a.shape[1])
    N = b.shape[1] if b_t else b.shape[0]
    kb = b.shape[0] if b_t else b.shape[1]
    if kb != K:
        raise ValueError(f"inner dimensions differ: a gives K={K}, b gives {kb}")
    _expect(a, "a", a.shape, torch.bfloat16)
    _expect(b, "b", b.shape, torch.bfloat16, a)
    if bias is not None:
        _expect(bias, "bias", (N,), torch.bfloat16, a)
    if out is not None:
        _expect(out, "out", (M, N), torch.bfloat16, a)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=a.device) if out is None else out
    _check(lib.cpattn_gemm(_dev(a, "a"), _dev(b, "b"),
                           _dev(bias, "bias") if bias is not None else None, _dev(c, "out"),
                           M, N, K, int(a_t), int(b_t), _stream(stream)), "cpattn_gemm")
    return c


def amax(x, out=None, stream=None):
    """max |x| as a one-element fp32 device tensor (or into `out`)."""
    if not isinstance(x, torch.Tensor):
        raise TypeError("x must be a torch.Tensor")
    _dtype_code(x)
    _expect(x, "x", x.shape, x.dtype)
    if out is not None:
        _expect(out, "out", (1,), torch.float32, x)
    a = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    _check(lib.cpattn_amax(_dev(x, "x"), x.numel(), _dtype_code(x), _dev(a, "amax"), _stream(stream)),
           "cpattn_amax")
    return a


def quantize_e4m3(x, amax_t, transpose: bool = False, stream=None):
    """e4m3 codes (uint8) of x [B, H, S, D] with s = 448 / amax_t (device fp32
    scalar, e.g. from amax()): [B, H, S, D], or [B, H, D, S] with transpose."""
    if not isinstance(x, torch.Tensor) or x.dim() != 4:
        raise ValueError("x must be a [B, H, S, D] tensor")
    _dtype_code(x)
    _expect(x, "x", x.shape, x.dtype)
    if not isinstance(amax_t, torch.Tensor) or amax_t.numel() < 1 or amax_t.dtype != torch.float32 \
            or amax_t.device != x.device:
        raise ValueError("amax_t must be a float32 tensor on x's device")
    B, H, S, D = x.shape
    shape = (B, H, D, S) if transpose else (B, H, S, D)
    out = torch.empty(shape, dtype=torch.uint8, device=x.device)
    _check(lib.cpattn_quantize_e4m3(_dev(x, "x"), _dtype_code(x), B * H, S, D, int(transpose),
                                    ctypes.c_void_p(amax_t.data_ptr()), _dev(out, "out"),
                                    _stream(stream)), "cpattn_quantize_e4m3")
    return out


def quantize_qkv_e4m3(q, k, v, stream=None):
    """(q8, k8, vt8, amax3): per-tensor e4m3 codes of q, k and of V transposed
    per head, and the device float[3] of max|q|, max|k|, max|v|."""
    B, H, S, D = _qkv(q, k, v)
    a3 = torch.empty(3, dtype=torch.float32, device=q.device)
    for i, t in enumerate((q, k, v)):
        amax(t, out=a3[i:i + 1], stream=stream)
    q8 = quantize_e4m3(q, a3[0:1], stream=stream)
    k8 = quantize_e4m3(k, a3[1:2], stream=stream)
    vt8 = quantize_e4m3(v, a3[2:3], transpose=True, stream=stream)
    return q8, k8, vt8, a3


def fwd_fp8(q8, k8, vt8, amax3, cp_size: int, causal: bool = True, scale=None, out=None, lse=None,
            stream=None):
    """Ring forward on e4m3 inputs (see quantize_qkv_e4m3): returns (o bf16, lse fp32)."""
    if not isinstance(q8, torch.Tensor) or q8.dim() != 4:
        raise ValueError("q8 must be a [B, H, S, D] tensor")
    B, H, S, D = q8.shape
    _expect(q8, "q8", (B, H, S, D), torch.uint8)
    _expect(k8, "k8", (B, H, S, D), torch.uint8, q8)
    _expect(vt8, "vt8", (B, H, D, S), torch.uint8, q8)
    _expect(amax3, "amax3", (3,), torch.float32, q8)
    scale = float(scale if scale is not None else D ** -0.5)
    if out is not None:
        _expect(out, "out", (B, H, S, D), torch.bfloat16, q8)
    if lse is not None:
        _expect(lse, "lse", (B, H, S), torch.float32, q8)
    o = torch.empty((B, H, S, D), dtype=torch.bfloat16, device=q8.device) if out is None else out
    l_t = torch.empty((B, H, S), dtype=torch.float32, device=q8.device) if lse is None else lse
    _check(lib.cpattn_fwd_fp8(_dev(q8, "q8"), _dev(k8, "k8"), _dev(vt8, "vt8"), _dev(amax3, "amax3"),
                              _dev(o, "o"), _dev(l_t, "lse"), B, H, S, D, cp_size, int(causal), scale,
                              _stream(stream)), "cpattn_fwd_fp8")
    return o, l_t


def layer_workspace_bytes(B, S, E, H) -> int:
    return int(lib.cpattn_layer_workspace_bytes(B, S, E, H))


def _bf16(t, name, shape):
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bf16")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return _dev(t, name)


def layer_fwd(x, w_qkv, b_qkv, w_o, b_o, num_heads: int, cp_size: int, causal: bool = True,
              scale=None, workspace=None, stream=None):
    """Attention layer forward (projections, head split, ring attention, head
    merge, output projection).  Returns (y, saved) where saved = (q, k, v, o,
    lse) feeds layer_bwd."""
    B, S, E = x.shape
    H = num_heads
    D = E // H
    scale = float(scale if scale is not None else D ** -0.5)
    if workspace is None:
        workspace = torch.empty(layer_workspace_bytes(B, S, E, H), dtype=torch.uint8, device=x.device)
    y = torch.empty_like(x)
    q, k, v, o = (torch.empty((B, H, S, D), dtype=x.dtype, device=x.device) for _ in range(4))
    lse = torch.empty((B, H, S), dtype=torch.float32, device=x.device)
    st = lib.cpattn_layer_fwd(_bf16(x, "x", (B, S, E)), _bf16(w_qkv, "w_qkv", (3 * E, E)),
                              _bf16(b_qkv, "b_qkv", (3 * E,)), _bf16(w_o, "w_o", (E, E)),
                              _bf16(b_o, "b_o", (E,)), _dev(y, "y"), _dev(q, "q"), _dev(k, "k"),
                              _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"), B, S, E, H, cp_size,
                              int(causal), scale, ctypes.c_void_p(workspace.data_ptr()),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "cpattn_layer_fwd")
    return y, (q, k, v, o, lse)


def layer_bwd(x, w_qkv, w_o, saved, dy, num_heads: int, cp_size: int, causal: bool = True,
              scale=None, workspace=None, stream=None):
    """Attention layer backward: returns (dx, dw_qkv, db_qkv, dw_o, db_o)."""
    B, S, E = x.shape
    H = num_heads
    D = E // H
    scale = float(scale if scale is not None else D ** -0.5)
    q, k, v, o, lse = saved
    _expect(lse, "lse", (B, H, S), torch.float32, x)
    if workspace is None:
        workspace = torch.empty(layer_workspace_bytes(B, S, E, H), dtype=torch.uint8, device=x.device)
    dx = torch.empty_like(x)
    dw_qkv = torch.empty_like(w_qkv)
    db_qkv = torch.empty((3 * E,), dtype=x.dtype, device=x.device)
    dw_o = torch.empty_like(w_o)
    db_o = torch.empty((E,), dtype=x.dtype, device=x.device)
    st = lib.cpattn_layer_bwd(_bf16(x, "x", (B, S, E)), _bf16(w_qkv, "w_qkv", (3 * E, E)),
                              _bf16(w_o, "w_o", (E, E)), _bf16(q, "q", (B, H, S, D)),
                              _bf16(k, "k", (B, H, S, D)), _bf16(v, "v", (B, H, S, D)),
                              _bf16(o, "o", (B, H, S, D)), _dev(lse, "lse"), _bf16(dy, "dy", (B, S, E)),
                              _dev(dx, "dx"), _dev(dw_qkv, "dw_qkv"), _dev(db_qkv, "db_qkv"),
                              _dev(dw_o, "dw_o"), _dev(db_o, "db_o"), B, S, E, H, cp_size, int(causal),
                              scale, ctypes.c_void_p(workspace.data_ptr()),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "cpattn_layer_bwd")
    return dx, dw_qkv, db_qkv, dw_o, db_o


def sync_status(stream=None) -> int:
    return int(lib.cpattn_sync_status(_stream(stream)))


def check_device_status(stream=None):
    _check(sync_status(stream), "device status")


def launch_count() -> int:
    return int(lib.cpattn_launch_count())


def set_path(path: int) -> int:
    return int(lib.cpattn_set_path(int(path)))


def last_path() -> int:
    return int(lib.cpattn_last_path())


def debug_stall(n: int) -> int:
    return int(lib.cpattn_debug_stall(int(n)))


KERNEL_KINDS = {0: "tc_fwd", 1: "simt_fwd", 2: "merge", 3: "finalize", 4: "bwd_delta",
                5: "simt_dkdv", 6: "simt_dq", 7: "tc_dkdv", 8: "tc_dq", 9: "layer_heads",
                10: "layer_colsum", 11: "accumulate", 12: "gemm", 13: "tc_fwd_fp8",
                14: "quant_e4m3"}


def profile(on: bool) -> int:
    return int(lib.cpattn_profile(int(on)))


def profile_read(kind: int):
    """(total_ms, launches) of one kernel kind since profile(True)."""
    ms = ctypes.c_double(0)
    n = ctypes.c_longlong(0)
    _check(lib.cpattn_profile_read(int(kind), ctypes.byref(ms), ctypes.byref(n)), "cpattn_profile_read")
    return ms.value, n.value
