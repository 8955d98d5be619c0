"""Thin ctypes binding of the C ABI in include/ispa.h.

Argument marshalling only: checks dtypes, devices and shapes, allocates
outputs and workspaces through torch's caching allocator, and passes raw
device pointers plus the current CUDA stream to the library. Every step of
the computation runs in the library's CUDA kernels; there is no fallback.
The function names are those of the C entry points.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libispa.so")

ISPA_OK = 0
ISPA_ERR_ARG = -1
ISPA_ERR_UNSUPPORTED = -2
ISPA_ERR_WORKSPACE = -3
ISPA_ERR_CUDA = -4
ISPA_ERR_NO_DEVICE = -5
ISPA_STATUS_TIMEOUT = 1
ISPA_STATUS_FP16_RANGE = 2
ISPA_STATUS_NOT_SPD = 4
ISPA_STATUS_NONFINITE = 8

EXPORTED = (
    "ispa_status_string", "ispa_version", "ispa_kernel_launches",
    "ispa_dual_attention_workspace_size", "ispa_dual_attention", "ispa_local_attention",
    "ispa_gram_accumulate", "ispa_absorb_workspace_size", "ispa_absorb_solve",
    "ispa_absorb_solve_noalloc", "ispa_absorb_solve_batched", "ispa_layer_error_batched",
    "ispa_layer_error_workspace_size", "ispa_layer_error", "ispa_rank_layers",
    "ispa_weight_gram_batched", "ispa_layer_error_wwt_batched",
    "ispa_full_attention_workspace_size", "ispa_full_attention", "ispa_absorbed_weight",
    "ispa_project", "ispa_quantize_weight_int8", "ispa_project_w8a8_workspace_size",
    "ispa_project_w8a8", "ispa_attention_units", "ispa_attention_set_splits",
    "ispa_set_wait_limit_ns", "ispa_dual_attention_layers_workspace_size",
    "ispa_dual_attention_layers",
)


class IspaKV(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("len", ctypes.c_int64)]


class IspaKVLayers(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("len", ctypes.c_int64),
                ("layer_stride", ctypes.c_int64)]


class IspaError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {ispa_status_string(code)} ({code})" if what else
                         f"{ispa_status_string(code)} ({code})")


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m kv_cache_absorption_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "ispa_status_string": (ctypes.c_char_p, [I]),
        "ispa_version": (I, []),
        "ispa_kernel_launches": (ctypes.c_uint64, []),
        "ispa_dual_attention_workspace_size": (SZ, [I64, I64, I64, I64, I, I]),
        "ispa_attention_units": (I64, [I64, I64, I64, I64, I, P, P]),
        "ispa_attention_set_splits": (I, [I, I]),
        "ispa_set_wait_limit_ns": (I, [ctypes.c_uint64]),
        "ispa_dual_attention": (I, [P, I64, I, I, IspaKV, IspaKV, IspaKV, F, P, P, P, P, P, P,
                                    P, SZ, P, P]),
        "ispa_local_attention": (I, [P, I64, I, I, IspaKV, IspaKV, F, P, P, P, P, SZ, P, P]),
        "ispa_dual_attention_layers_workspace_size": (SZ, [I, I64, I64, I64, I64, I, I]),
        "ispa_dual_attention_layers": (I, [I, P, I64, I64, I, I, IspaKVLayers, IspaKVLayers,
                                           IspaKVLayers, F, P, P, P, I64, P, P, P, I64, P, SZ,
                                           P, P]),
        "ispa_full_attention_workspace_size": (SZ, [I64, I64, I64, I64, I, I]),
        "ispa_full_attention": (I, [P, I64, I, I, IspaKV, IspaKV, IspaKV, F, P, P, P, SZ, P, P]),
        "ispa_absorbed_weight": (I, [P, P, I, P, P]),
        "ispa_project": (I, [P, I64, I, P, P, I, P, P]),
        "ispa_quantize_weight_int8": (I, [P, P, I, P, P, P]),
        "ispa_project_w8a8_workspace_size": (SZ, [I64, I]),
        "ispa_project_w8a8": (I, [P, I64, I, P, P, P, I, P, SZ, P, P]),
        "ispa_gram_accumulate": (I, [P, P, I64, I, P, I, I, P, P]),
        "ispa_absorb_workspace_size": (SZ, [I]),
        "ispa_absorb_solve": (I, [P, P, I, F, P, P, P, P, SZ, P, P]),
        "ispa_absorb_solve_noalloc": (I, [P, P, I, F, P, P, P, P, P]),
        "ispa_absorb_solve_batched": (I, [I, P, I64, P, I64, I, F, P, I64, P, I64, P, P, SZ, P, P]),
        "ispa_layer_error_batched": (I, [I, P, I64, P, I64, P, I64, P, I64, P, I, P, P, SZ, P]),
        "ispa_layer_error_workspace_size": (SZ, [I]),
        "ispa_layer_error": (I, [P, P, P, P, P, I, P, P, SZ, P]),
        "ispa_rank_layers": (I, [P, I, I, P, P, P]),
        "ispa_weight_gram_batched": (I, [I, P, I64, I, P, I64, P, P]),
        "ispa_layer_error_wwt_batched": (I, [I, P, I64, P, I64, P, I64, P, I64, P, I, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def ispa_status_string(code: int) -> str:
    return _load().ispa_status_string(int(code)).decode()


def ispa_version() -> int:
    return _load().ispa_version()


def ispa_kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(_load().ispa_kernel_launches())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, what: str):
    if rc != ISPA_OK:
        raise IspaError(rc, what)


def _dev_tensor(t: torch.Tensor, dtype, name: str, ndim: Optional[int] = None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")
    return t


def _kv(k: Optional[torch.Tensor], v: Optional[torch.Tensor], heads: int, hd: int, name: str):
    if k is None or k.shape[0] == 0:
        return IspaKV(None, None, 0)
    _dev_tensor(k, torch.bfloat16, name + " keys", 3)
    _dev_tensor(v, torch.bfloat16, name + " values", 3)
    if tuple(k.shape[1:]) != (heads, hd) or k.shape != v.shape:
        raise ValueError(f"{name}: keys/values must be [len, {heads}, {hd}]")
    return IspaKV(k.data_ptr(), v.data_ptr(), k.shape[0])


def new_status(device=None) -> torch.Tensor:
    """A zeroed device status word for the calls that report device-side
    conditions."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def read_status(status: torch.Tensor) -> int:
    """Synchronises and returns the device status bits."""
    return int(status.item())


def ispa_dual_attention_workspace_size(nq: int, sink_len: int, local_len: int, hist_len: int,
                                       heads: int, head_dim: int) -> int:
    return _load().ispa_dual_attention_workspace_size(nq, sink_len, local_len, hist_len, heads,
                                                      head_dim)


def ispa_dual_attention(q, k_sink, v_sink, k_loc, v_loc, k_hist=None, v_hist=None, scale=None,
                        a_loc=None, d_out=None, want_a_full=True, want_lse=True,
                        workspace=None, status=None, stream=None) -> dict:
    """Dual-stream attention of one chunk. q, k_*, v_*: [n, heads, head_dim]
    bf16 CUDA tensors. Returns a dict with a_loc and d ([nq, d] fp32), and,
    on request, a_full ([nq, d] bf16), lse_loc/lse_hist/lse_full ([heads, nq]
    fp32) and the status word."""
    _dev_tensor(q, torch.bfloat16, "q", 3)
    nq, heads, hd = q.shape
    d = heads * hd
    sink = _kv(k_sink, v_sink, heads, hd, "sink")
    loc = _kv(k_loc, v_loc, heads, hd, "local")
    hist = _kv(k_hist, v_hist, heads, hd, "history")
    dev = q.device
    if scale is None:
        scale = hd ** -0.5
    a_loc = torch.empty(nq, d, dtype=torch.float32, device=dev) if a_loc is None else a_loc
    d_out = torch.empty(nq, d, dtype=torch.float32, device=dev) if d_out is None else d_out
    a_full = torch.empty(nq, d, dtype=torch.bfloat16, device=dev) if want_a_full else None
    lse = [torch.empty(heads, nq, dtype=torch.float32, device=dev) if want_lse else None
           for _ in range(3)]
    need = ispa_dual_attention_workspace_size(nq, sink.len, loc.len, hist.len, heads, hd)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    rc = _load().ispa_dual_attention(
        _ptr(q), nq, heads, hd, sink, loc, hist, float(scale), _ptr(a_loc), _ptr(d_out),
        _ptr(a_full), _ptr(lse[0]), _ptr(lse[1]), _ptr(lse[2]), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream))
    _check(rc, "ispa_dual_attention")
    return {"a_loc": a_loc, "d": d_out, "a_full": a_full, "lse_loc": lse[0], "lse_hist": lse[1],
            "lse_full": lse[2], "status": status}


def ispa_dual_attention_layers_workspace_size(n_layers, nq, sink_len, local_len, hist_len, heads,
                                              head_dim) -> int:
    return int(_load().ispa_dual_attention_layers_workspace_size(
        n_layers, nq, sink_len, local_len, hist_len, heads, head_dim))


def _kv_layers(k: Optional[torch.Tensor], v: Optional[torch.Tensor], L: int, heads: int, hd: int,
               name: str):
    """[L, len, heads, head_dim] keys and values (each layer contiguous, the
    layers at a common stride) as an ispa_kv_layers."""
    if k is None or k.shape[1] == 0:
        return IspaKVLayers(None, None, 0, 0)
    for t, what in ((k, "keys"), (v, "values")):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} {what}: expected a CUDA bf16 tensor")
        if t.dim() != 4 or tuple(t.shape) != (L, k.shape[1], heads, hd) or not t[0].is_contiguous():
            raise ValueError(f"{name} {what}: expected [{L}, len, {heads}, {hd}] with contiguous layers")
    if k.stride(0) != v.stride(0):
        raise ValueError(f"{name}: keys and values must share their layer stride")
    return IspaKVLayers(k.data_ptr(), v.data_ptr(), k.shape[1], k.stride(0) if L > 1 else 0)


def ispa_dual_attention_layers(q, k_sink, v_sink, k_loc, v_loc, k_hist=None, v_hist=None,
                               scale=None, a_loc=None, d_out=None, a_full=None, lse=None,
                               workspace=None, status=None, stream=None) -> dict:
    """Dual-stream attention of the same chunk of L layers in one launch.
    q: [L, nq, heads, head_dim]; k_*, v_*: [L, len, heads, head_dim] bf16
    (each layer contiguous, any common layer stride). Outputs a_loc, d
    ([L, nq, d] fp32), a_full ([L, nq, d] bf16) and, with ``lse`` a list of
    three [L, heads, nq] fp32 tensors (or True to allocate them), the LSEs."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4 or not q[0].is_contiguous():
        raise ValueError("q: expected [L, nq, heads, head_dim] with contiguous layers")
    L, nq, heads, hd = q.shape
    d = heads * hd
    sink = _kv_layers(k_sink, v_sink, L, heads, hd, "sink")
    loc = _kv_layers(k_loc, v_loc, L, heads, hd, "local")
    hist = _kv_layers(k_hist, v_hist, L, heads, hd, "history")
    dev = q.device
    if scale is None:
        scale = hd ** -0.5
    f32 = dict(dtype=torch.float32, device=dev)
    a_loc = torch.empty(L, nq, d, **f32) if a_loc is None else a_loc
    d_out = torch.empty(L, nq, d, **f32) if d_out is None else d_out
    a_full = torch.empty(L, nq, d, dtype=torch.bfloat16, device=dev) if a_full is None else a_full
    for t in (a_loc, d_out, a_full):
        if t.shape != (L, nq, d) or not t[0].is_contiguous() or t.stride(0) != a_loc.stride(0):
            raise ValueError("outputs: expected [L, nq, d] with contiguous layers and one stride")
    if lse is True:
        lse = [torch.empty(L, heads, nq, **f32) for _ in range(3)]
    lse = lse or [None, None, None]
    lse_stride = next((t.stride(0) for t in lse if t is not None), 0)
    for t in lse:
        if t is not None and (t.shape != (L, heads, nq) or not t[0].is_contiguous()
                              or t.stride(0) != lse_stride):
            raise ValueError("lse: expected [L, heads, nq] with contiguous layers and one stride")
    need = ispa_dual_attention_layers_workspace_size(L, nq, sink.len, loc.len, hist.len, heads, hd)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    rc = _load().ispa_dual_attention_layers(
        L, _ptr(q), q.stride(0) if L > 1 else 0, nq, heads, hd, sink, loc, hist, float(scale),
        _ptr(a_loc), _ptr(d_out), _ptr(a_full), a_loc.stride(0) if L > 1 else 0, _ptr(lse[0]),
        _ptr(lse[1]), _ptr(lse[2]), lse_stride if L > 1 else 0, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream))
    _check(rc, "ispa_dual_attention_layers")
    return {"a_loc": a_loc, "d": d_out, "a_full": a_full, "lse_loc": lse[0], "lse_hist": lse[1],
            "lse_full": lse[2], "status": status}


def ispa_local_attention(q, k_sink, v_sink, k_loc, v_loc, scale=None, out_dtype=torch.bfloat16,
                         want_lse=False, workspace=None, status=None, stream=None) -> dict:
    """Local (sink + current chunk) attention of an L-Layer. Returns a dict
    with out ([nq, d] in out_dtype: bf16 or fp32), lse and the status word."""
    _dev_tensor(q, torch.bfloat16, "q", 3)
    nq, heads, hd = q.shape
    sink = _kv(k_sink, v_sink, heads, hd, "sink")
    loc = _kv(k_loc, v_loc, heads, hd, "local")
    dev = q.device
    if scale is None:
        scale = hd ** -0.5
    out = torch.empty(nq, heads * hd, dtype=out_dtype, device=dev)
    lse = torch.empty(heads, nq, dtype=torch.float32, device=dev) if want_lse else None
    need = ispa_dual_attention_workspace_size(nq, sink.len, loc.len, 0, heads, hd)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    f32 = out if out_dtype == torch.float32 else None
    b16 = out if out_dtype == torch.bfloat16 else None
    if f32 is None and b16 is None:
        raise TypeError("out_dtype must be torch.float32 or torch.bfloat16")
    rc = _load().ispa_local_attention(
        _ptr(q), nq, heads, hd, sink, loc, float(scale), _ptr(f32), _ptr(b16), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream))
    _check(rc, "ispa_local_attention")
    return {"out": out, "lse": lse, "status": status}


def ispa_attention_units(nq: int, sink_len: int, local_len: int, hist_len: int,
                         heads: int) -> tuple:
    """(units, local key ranges, history key ranges) of an attention call of
    this shape. Host only."""
    ls, hs = ctypes.c_int(0), ctypes.c_int(0)
    n = _load().ispa_attention_units(nq, sink_len, local_len, hist_len, heads, ctypes.byref(ls),
                                     ctypes.byref(hs))
    return int(n), ls.value, hs.value


def ispa_set_wait_limit_ns(ns: int = 0) -> None:
    """Limit of the kernels' pipeline waits for later launches (0 = default
    2 s); a wait past it ends the kernel with ISPA_STATUS_TIMEOUT."""
    _check(_load().ispa_set_wait_limit_ns(int(ns)), "ispa_set_wait_limit_ns")


def ispa_attention_set_splits(local_splits: int = 0, hist_splits: int = 0) -> None:
    """Force the key-range split counts of later attention calls (0 = automatic;
    hist_splits = -1: joint units, one per head and query pair, where a call
    has a history and returns A_loc)."""
    _check(_load().ispa_attention_set_splits(int(local_splits), int(hist_splits)),
           "ispa_attention_set_splits")


def ispa_full_attention_workspace_size(nq, sink_len, local_len, hist_len, heads, head_dim) -> int:
    return _load().ispa_full_attention_workspace_size(nq, sink_len, local_len, hist_len, heads,
                                                      head_dim)


def ispa_full_attention(q, k_sink, v_sink, k_loc, v_loc, k_hist=None, v_hist=None, scale=None,
                        want_lse=False, out=None, workspace=None, status=None, stream=None) -> dict:
    """Full attention of an F-Layer over sink, current chunk and history.
    Returns a dict with out ([nq, d] bf16), lse and the status word."""
    _dev_tensor(q, torch.bfloat16, "q", 3)
    nq, heads, hd = q.shape
    sink = _kv(k_sink, v_sink, heads, hd, "sink")
    loc = _kv(k_loc, v_loc, heads, hd, "local")
    hist = _kv(k_hist, v_hist, heads, hd, "history")
    dev = q.device
    if scale is None:
        scale = hd ** -0.5
    out = torch.empty(nq, heads * hd, dtype=torch.bfloat16, device=dev) if out is None else out
    lse = torch.empty(heads, nq, dtype=torch.float32, device=dev) if want_lse else None
    need = ispa_full_attention_workspace_size(nq, sink.len, loc.len, hist.len, heads, hd)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    rc = _load().ispa_full_attention(
        _ptr(q), nq, heads, hd, sink, loc, hist, float(scale), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream))
    _check(rc, "ispa_full_attention")
    return {"out": out, "lse": lse, "status": status}


def ispa_absorbed_weight(W, dW=None, out=None, stream=None):
    """bf16(W + dW) (or bf16(W)) for the streaming projection: [d, d] bf16."""
    _dev_tensor(W, torch.float32, "W", 2)
    if dW is not None:
        _dev_tensor(dW, torch.float32, "dW", 2)
    dim = W.shape[0]
    out = torch.empty(dim, dim, dtype=torch.bfloat16, device=W.device) if out is None else out
    rc = _load().ispa_absorbed_weight(_ptr(W), _ptr(dW), dim, _ptr(out), _stream(stream))
    _check(rc, "ispa_absorbed_weight")
    return out


def ispa_project(a, w, out=None, out_dtype=torch.bfloat16, status=None, stream=None):
    """out [rows, d] = a [rows, d] (bf16) x w [d, d] (bf16), fp32 accumulation."""
    _dev_tensor(a, torch.bfloat16, "a", 2)
    _dev_tensor(w, torch.bfloat16, "w", 2)
    rows, dim = a.shape
    if out is None:
        out = torch.empty(rows, dim, dtype=out_dtype, device=a.device)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be bf16 or fp32")
    status = new_status(a.device) if status is None else status
    rc = _load().ispa_project(_ptr(a), rows, dim, _ptr(w), _ptr(out),
                              1 if out.dtype == torch.float32 else 0, _ptr(status), _stream(stream))
    _check(rc, "ispa_project")
    return out


def ispa_quantize_weight_int8(W, dW=None, wq_t=None, w_scale=None, stream=None):
    """8-bit codes of W' = W (+ dW) per output column, transposed ([d, d] int8,
    row n = column n of W'), and the column scales ([d] fp32)."""
    _dev_tensor(W, torch.float32, "W", 2)
    if dW is not None:
        _dev_tensor(dW, torch.float32, "dW", 2)
    dim = W.shape[0]
    wq_t = torch.empty(dim, dim, dtype=torch.int8, device=W.device) if wq_t is None else wq_t
    w_scale = torch.empty(dim, dtype=torch.float32, device=W.device) if w_scale is None else w_scale
    rc = _load().ispa_quantize_weight_int8(_ptr(W), _ptr(dW), dim, _ptr(wq_t), _ptr(w_scale),
                                           _stream(stream))
    _check(rc, "ispa_quantize_weight_int8")
    return wq_t, w_scale


def ispa_project_w8a8_workspace_size(rows: int, dim: int) -> int:
    return _load().ispa_project_w8a8_workspace_size(rows, dim)


def ispa_project_w8a8(a, wq_t, w_scale, out=None, out_dtype=torch.bfloat16, workspace=None,
                      status=None, stream=None):
    """out [rows, d] = W8A8 product of a [rows, d] (bf16, quantised per row
    on the fly) and the weight codes from ispa_quantize_weight_int8."""
    _dev_tensor(a, torch.bfloat16, "a", 2)
    _dev_tensor(wq_t, torch.int8, "wq_t", 2)
    _dev_tensor(w_scale, torch.float32, "w_scale", 1)
    rows, dim = a.shape
    if out is None:
        out = torch.empty(rows, dim, dtype=out_dtype, device=a.device)
    if workspace is None:
        workspace = torch.empty(max(ispa_project_w8a8_workspace_size(rows, dim), 256),
                                dtype=torch.uint8, device=a.device)
    status = new_status(a.device) if status is None else status
    rc = _load().ispa_project_w8a8(_ptr(a), rows, dim, _ptr(wq_t), _ptr(w_scale), _ptr(out),
                                   1 if out.dtype == torch.float32 else 0, _ptr(workspace),
                                   workspace.numel(), _ptr(status), _stream(stream))
    _check(rc, "ispa_project_w8a8")
    return out


def ispa_gram_accumulate(a_loc, d, M=None, accumulate=False, want_s=True, status=None,
                         stream=None):
    """M[0:d,0:d] (G) (+)= A_loc^T A_loc, M[0:d,d:2d] (R) (+)= A_loc^T D,
    M[d:2d,d:2d] (S) (+)= D^T D; M is [2d, 2d] fp32. ``status``: a device
    status word (``new_status``) that receives ISPA_STATUS_* bits; one is made
    when not given. Returns M."""
    _dev_tensor(a_loc, torch.float32, "a_loc", 2)
    _dev_tensor(d, torch.float32, "d", 2)
    rows, dim = a_loc.shape
    if d.shape != a_loc.shape:
        raise ValueError("a_loc and d must have the same shape")
    if M is None:
        M = torch.empty(2 * dim, 2 * dim, dtype=torch.float32, device=a_loc.device)
        accumulate = False
    _dev_tensor(M, torch.float32, "M", 2)
    status = new_status(a_loc.device) if status is None else status
    rc = _load().ispa_gram_accumulate(_ptr(a_loc), _ptr(d), rows, dim, _ptr(M), int(bool(accumulate)),
                                      int(bool(want_s)), _ptr(status), _stream(stream))
    _check(rc, "ispa_gram_accumulate")
    return M


def ispa_absorb_workspace_size(dim: int) -> int:
    return _load().ispa_absorb_workspace_size(dim)


def ispa_absorb_solve(M, W, lam: float = 0.0, workspace=None, status=None, stream=None) -> dict:
    """Delta W solving (G + lambda I) Delta W = R W (lam <= 0: 1e-2 tr(G)/d).
    Returns dW, B = R W, the lambda used (device float) and the status word."""
    _dev_tensor(M, torch.float32, "M", 2)
    _dev_tensor(W, torch.float32, "W", 2)
    dim = W.shape[0]
    if tuple(M.shape) != (2 * dim, 2 * dim) or W.shape[1] != dim:
        raise ValueError("M must be [2d, 2d] and W [d, d]")
    dev = W.device
    dW = torch.empty(dim, dim, dtype=torch.float32, device=dev)
    B = torch.empty(dim, dim, dtype=torch.float32, device=dev)
    lam_out = torch.empty(1, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(ispa_absorb_workspace_size(dim), dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    rc = _load().ispa_absorb_solve(_ptr(M), _ptr(W), dim, float(lam), _ptr(dW), _ptr(B),
                                   _ptr(lam_out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _ptr(status),
                                   _stream(stream))
    _check(rc, "ispa_absorb_solve")
    return {"dW": dW, "B": B, "lam": lam_out, "status": status}


def ispa_absorb_solve_noalloc(M, W, lam: float = 0.0, status=None, stream=None) -> dict:
    """ispa_absorb_solve without a workspace, for callers that cannot allocate
    device memory when they solve: the scratch is an array inside the library
    (dim <= 512; concurrent calls on one GPU race). The output buffers are
    allocated here only because this binding returns new tensors."""
    _dev_tensor(M, torch.float32, "M", 2)
    _dev_tensor(W, torch.float32, "W", 2)
    dim = W.shape[0]
    if tuple(M.shape) != (2 * dim, 2 * dim) or W.shape[1] != dim:
        raise ValueError("M must be [2d, 2d] and W [d, d]")
    dev = W.device
    dW = torch.empty(dim, dim, dtype=torch.float32, device=dev)
    B = torch.empty(dim, dim, dtype=torch.float32, device=dev)
    lam_out = torch.empty(1, dtype=torch.float32, device=dev)
    status = new_status(dev) if status is None else status
    rc = _load().ispa_absorb_solve_noalloc(_ptr(M), _ptr(W), dim, float(lam), _ptr(dW), _ptr(B),
                                           _ptr(lam_out), _ptr(status), _stream(stream))
    _check(rc, "ispa_absorb_solve_noalloc")
    return {"dW": dW, "B": B, "lam": lam_out, "status": status}


def ispa_absorb_solve_batched(M, W, lam: float = 0.0, dW=None, B=None, lam_out=None,
                              workspace=None, status=None, stream=None) -> dict:
    """Delta W of L layers in one call. M: [L, 2d, 2d], W: [L, d, d] fp32
    (contiguous, so layer strides are 4 d^2 and d^2 elements). Returns dW and
    B ([L, d, d]), the lambdas ([L]) and the status word."""
    _dev_tensor(M, torch.float32, "M", 3)
    _dev_tensor(W, torch.float32, "W", 3)
    L, dim = W.shape[0], W.shape[1]
    if tuple(M.shape) != (L, 2 * dim, 2 * dim) or W.shape[2] != dim:
        raise ValueError("M must be [L, 2d, 2d] and W [L, d, d]")
    dev = W.device
    dW = torch.empty(L, dim, dim, dtype=torch.float32, device=dev) if dW is None else dW
    B = torch.empty(L, dim, dim, dtype=torch.float32, device=dev) if B is None else B
    lam_out = torch.empty(L, dtype=torch.float32, device=dev) if lam_out is None else lam_out
    if workspace is None:
        workspace = torch.empty(L * ispa_absorb_workspace_size(dim), dtype=torch.uint8, device=dev)
    status = new_status(dev) if status is None else status
    dd = dim * dim
    rc = _load().ispa_absorb_solve_batched(
        L, _ptr(M), 4 * dd, _ptr(W), dd, dim, float(lam), _ptr(dW), dW.stride(0), _ptr(B),
        B.stride(0), _ptr(lam_out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream))
    _check(rc, "ispa_absorb_solve_batched")
    return {"dW": dW, "B": B, "lam": lam_out, "status": status}


def ispa_layer_error_batched(M, W, dW, B, lam, err=None, workspace=None, stream=None):
    """Reconstruction errors of L layers: device double [L, 2]."""
    for t, n in ((M, "M"), (W, "W"), (dW, "dW"), (B, "B")):
        _dev_tensor(t, torch.float32, n, 3)
    _dev_tensor(lam, torch.float32, "lam", 1)
    L, dim = W.shape[0], W.shape[1]
    dev = W.device
    err = torch.empty(L, 2, dtype=torch.float64, device=dev) if err is None else err
    if workspace is None:
        workspace = torch.empty(L * ispa_layer_error_workspace_size(dim), dtype=torch.uint8,
                                device=dev)
    dd = dim * dim
    rc = _load().ispa_layer_error_batched(
        L, _ptr(M), 4 * dd, _ptr(W), dd, _ptr(dW), dW.stride(0), _ptr(B), B.stride(0), _ptr(lam),
        dim, _ptr(err), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(rc, "ispa_layer_error_batched")
    return err


def ispa_weight_gram_batched(W, P=None, status=None, stream=None):
    """P[l] = W[l] W[l]^T for W [L, d, d] fp32 (contiguous)."""
    _dev_tensor(W, torch.float32, "W", 3)
    L, dim = W.shape[0], W.shape[1]
    P = torch.empty_like(W) if P is None else P
    _dev_tensor(P, torch.float32, "P", 3)
    status = new_status(W.device) if status is None else status
    rc = _load().ispa_weight_gram_batched(L, _ptr(W), W.stride(0), dim, _ptr(P), P.stride(0),
                                          _ptr(status), _stream(stream))
    _check(rc, "ispa_weight_gram_batched")
    return P


def ispa_layer_error_wwt_batched(M, P, dW, B, lam, err=None, workspace=None, stream=None):
    """Reconstruction errors of L layers from P = W W^T: device double [L, 2]."""
    for t, n in ((M, "M"), (P, "P"), (dW, "dW"), (B, "B")):
        _dev_tensor(t, torch.float32, n, 3)
    _dev_tensor(lam, torch.float32, "lam", 1)
    L, dim = P.shape[0], P.shape[1]
    dev = P.device
    err = torch.empty(L, 2, dtype=torch.float64, device=dev) if err is None else err
    workspace = (torch.empty(L * ispa_layer_error_workspace_size(dim), dtype=torch.uint8,
                             device=dev) if workspace is None else workspace)
    rc = _load().ispa_layer_error_wwt_batched(
        L, _ptr(M), M.stride(0), _ptr(P), P.stride(0), _ptr(dW), dW.stride(0), _ptr(B),
        B.stride(0), _ptr(lam), dim, _ptr(err), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "ispa_layer_error_wwt_batched")
    return err


def ispa_layer_error_workspace_size(dim: int) -> int:
    return _load().ispa_layer_error_workspace_size(dim)


def ispa_layer_error(M, W, dW, B, lam, err=None, workspace=None, stream=None):
    """Reconstruction error of one layer: device double[2] =
    {||E||^2, ||E||^2 / ||A_full W||^2} (written into ``err`` if given)."""
    for t, n in ((M, "M"), (W, "W"), (dW, "dW"), (B, "B"), (lam, "lam")):
        _dev_tensor(t, torch.float32, n)
    dim = W.shape[0]
    dev = W.device
    if err is None:
        err = torch.empty(2, dtype=torch.float64, device=dev)
    if workspace is None:
        workspace = torch.empty(ispa_layer_error_workspace_size(dim), dtype=torch.uint8, device=dev)
    rc = _load().ispa_layer_error(_ptr(M), _ptr(W), _ptr(dW), _ptr(B), _ptr(lam), dim, _ptr(err),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream))
    _check(rc, "ispa_layer_error")
    return err


def ispa_rank_layers(err, K: int, stream=None):
    """Stable ascending ranking of layers by relative error (err: device
    double [n_layers, 2]). Returns (perm int32 [n], selected uint8 [n])."""
    _dev_tensor(err, torch.float64, "err")
    n = err.numel() // 2
    perm = torch.empty(n, dtype=torch.int32, device=err.device)
    sel = torch.empty(n, dtype=torch.uint8, device=err.device)
    rc = _load().ispa_rank_layers(_ptr(err), n, int(K), _ptr(perm), _ptr(sel), _stream(stream))
    _check(rc, "ispa_rank_layers")
    return perm, sel
