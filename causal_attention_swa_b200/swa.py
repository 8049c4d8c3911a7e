"""Thin ctypes binding of libswa.so (C ABI in include/swa.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  torch provides device memory (outputs and
workspaces are torch tensors) and the current CUDA stream.  If the library
has not been built, or no CUDA device is present, calls raise instead of
falling back to anything else.

Function names follow the C ABI: ``attn_fwd`` -> ``swa_attn_fwd`` and so on.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libswa.so")

SWA_OK, SWA_ERR_INVALID_ARGUMENT, SWA_ERR_UNSUPPORTED, SWA_ERR_CUDA, SWA_ERR_DEVICE_TIMEOUT = range(5)
SWA_F32, SWA_BF16 = 0, 1

# Every symbol include/swa.h declares.
EXPORTS = (
    "swa_attn_fwd_workspace_size", "swa_attn_fwd", "swa_attn_bwd_workspace_size",
    "swa_attn_bwd", "swa_nw_workspace_size", "swa_nw_regrid", "swa_get_device_error",
    "swa_status_string", "swa_last_error_message", "swa_last_launch_count",
    "swa_profile_kernel", "swa_attn_fwd_noalloc", "swa_selftest_wait_timeout",
    "swa_attn_grad_workspace_size", "swa_attn_grad", "swa_nw_regrid_nd",
    "swa_nw_regrid_bwd_workspace_size", "swa_nw_regrid_bwd", "swa_qkv_proj",
    "swa_attn_merge", "swa_attn_bwd_acc", "swa_f32_to_bf16",
)
(SWA_KERNEL_NONE, SWA_KERNEL_ATTN_FWD, SWA_KERNEL_ATTN_BWD, SWA_KERNEL_NW, SWA_KERNEL_NW_BWD,
 SWA_KERNEL_QKV) = range(6)


class SwaError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status} ({_status_name(status)}): {message}")
        self.status = status


_lib = None


def _status_name(st: int) -> str:
    names = ["SWA_OK", "SWA_ERR_INVALID_ARGUMENT", "SWA_ERR_UNSUPPORTED", "SWA_ERR_CUDA",
             "SWA_ERR_DEVICE_TIMEOUT"]
    return names[st] if 0 <= st < len(names) else f"unknown({st})"


def load_library():
    """Load libswa.so with ctypes (no CUDA work).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m causal_attention_swa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I, SZ, F = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t,
                        ctypes.c_float)
    lib.swa_attn_fwd_workspace_size.argtypes = [I64, I64, I64, I64, I]
    lib.swa_attn_fwd_workspace_size.restype = SZ
    lib.swa_attn_fwd.argtypes = [P, P, P, P, P, I64, I64, I64, I64, I, I, P, SZ, P]
    lib.swa_attn_fwd.restype = I
    lib.swa_attn_bwd_workspace_size.argtypes = [I64, I64, I64, I64, I]
    lib.swa_attn_bwd_workspace_size.restype = SZ
    lib.swa_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I64, I64, I64, I64, I, I, P, SZ, P]
    lib.swa_attn_bwd.restype = I
    lib.swa_attn_grad_workspace_size.argtypes = [I64, I64, I64, I64, I]
    lib.swa_attn_grad_workspace_size.restype = SZ
    lib.swa_attn_grad.argtypes = [P, P, P, P, P, P, P, P, I64, I64, I64, I64, I, I, P, SZ, P]
    lib.swa_attn_grad.restype = I
    lib.swa_nw_workspace_size.argtypes = [I64, I64]
    lib.swa_nw_workspace_size.restype = SZ
    lib.swa_nw_regrid.argtypes = [P, I64, P, P, I64, F, P, P, SZ, P]
    lib.swa_nw_regrid.restype = I
    lib.swa_nw_regrid_nd.argtypes = [P, I64, P, P, I64, I, F, P, P, SZ, P]
    lib.swa_nw_regrid_nd.restype = I
    lib.swa_nw_regrid_bwd_workspace_size.argtypes = [I64, I64, I]
    lib.swa_nw_regrid_bwd_workspace_size.restype = SZ
    lib.swa_nw_regrid_bwd.argtypes = [P, I64, P, P, I64, I, F, P, P, P, P, P, SZ, P]
    lib.swa_nw_regrid_bwd.restype = I
    lib.swa_qkv_proj.argtypes = [P, P, P, P, P, I64, I64, I64, I64, I64, I, P]
    lib.swa_qkv_proj.restype = I
    lib.swa_attn_merge.argtypes = [P, P, P, P, P, I64, I64, I, I, P]
    lib.swa_attn_merge.restype = I
    lib.swa_attn_bwd_acc.argtypes = [P, P, P, P, P, P, P, P, P, I64, I64, I64, I64, I, I, P, SZ, P]
    lib.swa_attn_bwd_acc.restype = I
    lib.swa_f32_to_bf16.argtypes = [P, P, I64, P]
    lib.swa_f32_to_bf16.restype = I
    lib.swa_get_device_error.argtypes = [P]
    lib.swa_get_device_error.restype = I
    lib.swa_selftest_wait_timeout.argtypes = [P]
    lib.swa_selftest_wait_timeout.restype = I
    lib.swa_status_string.argtypes = [I]
    lib.swa_status_string.restype = ctypes.c_char_p
    lib.swa_last_error_message.argtypes = []
    lib.swa_last_error_message.restype = ctypes.c_char_p
    lib.swa_last_launch_count.argtypes = []
    lib.swa_last_launch_count.restype = I
    lib.swa_profile_kernel.argtypes = [I, P, P]
    lib.swa_profile_kernel.restype = None
    _lib = lib
    return lib


def _check(st: int, where: str) -> None:
    if st != SWA_OK:
        msg = load_library().swa_last_error_message().decode(errors="replace")
        raise SwaError(st, where, msg)


def _stream_ptr(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SWA_BF16
    if t.dtype == torch.float32:
        return SWA_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bfloat16 or float32")


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _require_like(ref, named, what):
    """The C ABI takes sizes from `ref` only, so every other tensor must have
    the shape, dtype and device that it implies (checked before any launch)."""
    for name, t in named.items():
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        shape, dtype = what(name)
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != ref.device:
            raise ValueError(f"{name}: expected shape {tuple(shape)}, dtype {dtype} on "
                             f"{ref.device}; got {tuple(t.shape)}, {t.dtype} on {t.device}")


def _require_cuda(*ts):
    for t in ts:
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def last_launch_count() -> int:
    """Kernels the last successful call on this thread enqueued."""
    return int(load_library().swa_last_launch_count())


def profile_kernel(which: int, start=None, stop=None) -> None:
    """swa_profile_kernel: later calls on this thread record the torch.cuda.Event
    pair around kernel `which` (SWA_KERNEL_*); which = SWA_KERNEL_NONE stops."""
    lib = load_library()
    if which == SWA_KERNEL_NONE or start is None or stop is None:
        lib.swa_profile_kernel(SWA_KERNEL_NONE, None, None)
        return
    lib.swa_profile_kernel(which, ctypes.c_void_p(start.cuda_event),
                           ctypes.c_void_p(stop.cuda_event))


def attn_fwd_workspace_size(B, H, N, D, dtype_code) -> int:
    return int(load_library().swa_attn_fwd_workspace_size(B, H, N, D, dtype_code))


def attn_bwd_workspace_size(B, H, N, D, dtype_code) -> int:
    return int(load_library().swa_attn_bwd_workspace_size(B, H, N, D, dtype_code))


def attn_grad_workspace_size(B, H, N, D, dtype_code) -> int:
    return int(load_library().swa_attn_grad_workspace_size(B, H, N, D, dtype_code))


def nw_workspace_size(M, S) -> int:
    return int(load_library().swa_nw_workspace_size(M, S))


def _workspace(nbytes: int, device, ws):
    if nbytes == 0:
        return None
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def attn_fwd(q, k, v, causal: bool = True, out=None, lse=None, workspace=None):
    """swa_attn_fwd: q, k, v [B,H,N,64] bf16 or fp32 CUDA tensors ->
    (out [B,H,N,64] same dtype, lse [B,H,N] fp32)."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a [B, H, N, D] tensor")
    B, H, N, D = q.shape
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _require_like(q, {"k": k, "v": v, "out": out, "lse": lse},
                  lambda n: ((B, H, N), torch.float32) if n == "lse" else (q.shape, q.dtype))
    lib = load_library()
    _require_cuda(q, k, v, out, lse)
    nbytes = attn_fwd_workspace_size(B, H, N, D, dt)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib.swa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, D,
                          int(bool(causal)), dt, _ptr(ws), nbytes, _stream_ptr(q.device))
    _check(st, "swa_attn_fwd")
    return out, lse


def attn_bwd(q, k, v, out, dout, lse, causal: bool = True, dq=None, dk=None, dv=None,
             workspace=None):
    """swa_attn_bwd -> (dq, dk, dv), each [B,H,N,64] of q's dtype."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a [B, H, N, D] tensor")
    B, H, N, D = q.shape
    dt = _dtype_code(q)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    _require_like(q, {"k": k, "v": v, "out": out, "dout": dout, "lse": lse, "dq": dq, "dk": dk,
                      "dv": dv},
                  lambda n: ((B, H, N), torch.float32) if n == "lse" else (q.shape, q.dtype))
    lib = load_library()
    _require_cuda(q, k, v, out, dout, lse, dq, dk, dv)
    nbytes = attn_bwd_workspace_size(B, H, N, D, dt)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib.swa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                          _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, D, int(bool(causal)), dt,
                          _ptr(ws), nbytes, _stream_ptr(q.device))
    _check(st, "swa_attn_bwd")
    return dq, dk, dv


def attn_grad(q, k, v, causal: bool = True, out=None, lse=None, dq=None, dk=None, dv=None,
              workspace=None):
    """swa_attn_grad: forward and the gradient of 1/2 sum out^2 in one call ->
    (out, lse, dq, dk, dv)."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a [B, H, N, D] tensor")
    B, H, N, D = q.shape
    dt = _dtype_code(q)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    _require_like(q, {"k": k, "v": v, "out": out, "lse": lse, "dq": dq, "dk": dk, "dv": dv},
                  lambda n: ((B, H, N), torch.float32) if n == "lse" else (q.shape, q.dtype))
    lib = load_library()
    _require_cuda(q, k, v, out, lse, dq, dk, dv)
    nbytes = attn_grad_workspace_size(B, H, N, D, dt)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib.swa_attn_grad(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dq), _ptr(dk),
                           _ptr(dv), B, H, N, D, int(bool(causal)), dt, _ptr(ws), nbytes,
                           _stream_ptr(q.device))
    _check(st, "swa_attn_grad")
    return out, lse, dq, dk, dv


def nw_regrid(targets, sources, vals, h: float = 0.5, out=None, workspace=None):
    """swa_nw_regrid: targets [M,2], sources [S,2], vals [S] fp32 -> out [M] fp32."""
    if not isinstance(targets, torch.Tensor) or targets.dim() != 2 or \
            not isinstance(sources, torch.Tensor) or sources.dim() != 2:
        raise ValueError("targets and sources must be [M, 2] and [S, 2] tensors")
    M, S = targets.shape[0], sources.shape[0]
    out = torch.empty((M,), dtype=torch.float32, device=targets.device) if out is None else out
    shapes = {"targets": (M, 2), "sources": (S, 2), "vals": (S,), "out": (M,)}
    _require_like(targets, {"targets": targets, "sources": sources, "vals": vals, "out": out},
                  lambda n: (shapes[n], torch.float32))
    lib = load_library()
    _require_cuda(targets, sources, vals, out)
    nbytes = nw_workspace_size(M, S)
    ws = _workspace(nbytes, targets.device, workspace)
    st = lib.swa_nw_regrid(_ptr(targets), M, _ptr(sources), _ptr(vals), S, float(h), _ptr(out),
                           _ptr(ws), nbytes, _stream_ptr(targets.device))
    _check(st, "swa_nw_regrid")
    return out


def _nw_points(targets, sources):
    if not isinstance(targets, torch.Tensor) or targets.dim() != 2 or \
            not isinstance(sources, torch.Tensor) or sources.dim() != 2:
        raise ValueError("targets and sources must be [M, d] and [S, d] tensors")
    return targets.shape[0], sources.shape[0], targets.shape[1]


def nw_regrid_nd(targets, sources, vals, h: float = 0.5, out=None, workspace=None):
    """swa_nw_regrid_nd: targets [M,d], sources [S,d] (d = 1, 2, 3), vals [S]
    fp32 -> out [M] fp32."""
    M, S, d = _nw_points(targets, sources)
    out = torch.empty((M,), dtype=torch.float32, device=targets.device) if out is None else out
    shapes = {"targets": (M, d), "sources": (S, d), "vals": (S,), "out": (M,)}
    _require_like(targets, {"targets": targets, "sources": sources, "vals": vals, "out": out},
                  lambda n: (shapes[n], torch.float32))
    lib = load_library()
    _require_cuda(targets, sources, vals, out)
    nbytes = nw_workspace_size(M, S)
    ws = _workspace(nbytes, targets.device, workspace)
    st = lib.swa_nw_regrid_nd(_ptr(targets), M, _ptr(sources), _ptr(vals), S, d, float(h),
                              _ptr(out), _ptr(ws), nbytes, _stream_ptr(targets.device))
    _check(st, "swa_nw_regrid_nd")
    return out


def nw_regrid_bwd(targets, sources, vals, gout, h: float = 0.5, workspace=None):
    """swa_nw_regrid_bwd -> (dtargets [M,d], dsources [S,d], dvals [S])."""
    M, S, d = _nw_points(targets, sources)
    dt = torch.empty_like(targets)
    ds = torch.empty_like(sources)
    dv = torch.empty((S,), dtype=torch.float32, device=targets.device)
    shapes = {"targets": (M, d), "sources": (S, d), "vals": (S,), "gout": (M,)}
    _require_like(targets, {"targets": targets, "sources": sources, "vals": vals, "gout": gout},
                  lambda n: (shapes[n], torch.float32))
    lib = load_library()
    _require_cuda(targets, sources, vals, gout, dt, ds, dv)
    nbytes = int(lib.swa_nw_regrid_bwd_workspace_size(M, S, d))
    ws = _workspace(nbytes, targets.device, workspace)
    st = lib.swa_nw_regrid_bwd(_ptr(targets), M, _ptr(sources), _ptr(vals), S, d, float(h),
                               _ptr(gout), _ptr(dt), _ptr(ds), _ptr(dv), _ptr(ws), nbytes,
                               _stream_ptr(targets.device))
    _check(st, "swa_nw_regrid_bwd")
    return dt, ds, dv


def qkv_proj(x, w, H: int, q=None, k=None, v=None):
    """swa_qkv_proj: x [B, N, C] bf16, w [3*H*64, C] bf16 -> q, k, v
    [B, H, N, 64] bf16."""
    if not isinstance(x, torch.Tensor) or x.dim() != 3:
        raise ValueError("x must be a [B, N, C] tensor")
    B, N, C = x.shape
    shape = (B, H, N, 64)
    q = torch.empty(shape, dtype=x.dtype, device=x.device) if q is None else q
    k = torch.empty(shape, dtype=x.dtype, device=x.device) if k is None else k
    v = torch.empty(shape, dtype=x.dtype, device=x.device) if v is None else v
    shapes = {"x": (B, N, C), "w": (3 * H * 64, C), "q": shape, "k": shape, "v": shape}
    _require_like(x, {"x": x, "w": w, "q": q, "k": k, "v": v}, lambda n: (shapes[n], x.dtype))
    lib = load_library()
    _require_cuda(x, w, q, k, v)
    st = lib.swa_qkv_proj(_ptr(x), _ptr(w), _ptr(q), _ptr(k), _ptr(v), B, N, C, H, 64,
                          _dtype_code(x), _stream_ptr(x.device))
    _check(st, "swa_qkv_proj")
    return q, k, v


def attn_merge(out_part, lse_part, out_acc, lse_acc, first: bool, out_final=None):
    """swa_attn_merge: merge a partial result (out_part [B,H,N,64] bf16 or
    fp32, lse_part [B,H,N] fp32) over one key set into the float32
    accumulator (out_acc [B,H,N,64], lse_acc [B,H,N]) over a disjoint set;
    with out_final, also write the merged rows in out_part's dtype."""
    if not isinstance(out_part, torch.Tensor) or out_part.dim() != 4:
        raise ValueError("out_part must be a [B, H, N, D] tensor")
    B, H, N, D = out_part.shape
    named = {"lse_part": lse_part, "out_acc": out_acc, "lse_acc": lse_acc}
    shapes = {"lse_part": ((B, H, N), torch.float32), "out_acc": ((B, H, N, D), torch.float32),
              "lse_acc": ((B, H, N), torch.float32), "out_final": (out_part.shape, out_part.dtype)}
    if out_final is not None:
        named["out_final"] = out_final
    _require_like(out_part, named, lambda n: shapes[n])
    lib = load_library()
    _require_cuda(out_part, *named.values())
    st = lib.swa_attn_merge(_ptr(out_part), _ptr(lse_part), _ptr(out_acc), _ptr(lse_acc),
                            _ptr(out_final), B * H * N, D, int(bool(first)),
                            _dtype_code(out_part), _stream_ptr(out_part.device))
    _check(st, "swa_attn_merge")
    return out_acc, lse_acc


def attn_bwd_acc(q, k, v, out, dout, lse, dq_acc, dk_acc, dv_acc, causal: bool = True,
                 workspace=None):
    """swa_attn_bwd_acc: like attn_bwd (bf16 q, k, v, out, dout [B,H,N,64], lse
    [B,H,N]) but adds dq, dk, dv to the float32 sums dq_acc, dk_acc, dv_acc."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a [B, H, N, D] tensor")
    B, H, N, D = q.shape
    dt = _dtype_code(q)
    shapes = {"lse": ((B, H, N), torch.float32)}
    for n in ("dq_acc", "dk_acc", "dv_acc"):
        shapes[n] = (q.shape, torch.float32)
    _require_like(q, {"k": k, "v": v, "out": out, "dout": dout, "lse": lse, "dq_acc": dq_acc,
                      "dk_acc": dk_acc, "dv_acc": dv_acc},
                  lambda n: shapes.get(n, (q.shape, q.dtype)))
    lib = load_library()
    _require_cuda(q, k, v, out, dout, lse, dq_acc, dk_acc, dv_acc)
    nbytes = attn_bwd_workspace_size(B, H, N, D, dt)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib.swa_attn_bwd_acc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                              _ptr(dq_acc), _ptr(dk_acc), _ptr(dv_acc), B, H, N, D,
                              int(bool(causal)), dt, _ptr(ws), nbytes, _stream_ptr(q.device))
    _check(st, "swa_attn_bwd_acc")
    return dq_acc, dk_acc, dv_acc


def f32_to_bf16(src, dst=None):
    """swa_f32_to_bf16: a float32 CUDA tensor rounded into a bf16 one."""
    if dst is None:
        dst = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    if src.dtype != torch.float32 or dst.dtype != torch.bfloat16 or src.shape != dst.shape:
        raise ValueError("src must be float32 and dst bfloat16 of the same shape")
    _require_cuda(src, dst)
    st = load_library().swa_f32_to_bf16(_ptr(src), _ptr(dst), src.numel(),
                                        _stream_ptr(src.device))
    _check(st, "swa_f32_to_bf16")
    return dst


def selftest_wait_timeout(device=None) -> None:
    """swa_selftest_wait_timeout on the current stream (a kernel whose bounded
    waits run out; read the result with get_device_error)."""
    dev = torch.device("cuda") if device is None else device
    st = int(load_library().swa_selftest_wait_timeout(_stream_ptr(dev)))
    if st != SWA_OK:
        raise SwaError(st, "swa_selftest_wait_timeout",
                       load_library().swa_last_error_message().decode())


def get_device_error(device=None) -> int:
    """swa_get_device_error on the current stream: returns the status."""
    dev = torch.device("cuda") if device is None else device
    return int(load_library().swa_get_device_error(_stream_ptr(dev)))
