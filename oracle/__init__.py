"""Float64 CPU oracle for the fused softmax-weighted average.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package; the product
path (``causal_attention_swa_b200``) never does, and it shares no code with it.

The arithmetic lives in ``swa_oracle.c`` (plain C, IEEE float64, OpenMP over
rows), a restatement of the SQL views of "Show HN: Automatic deduction of
FlashAttention kernel from ~25 lines of SQL" (page 2, demo script
``01_attention.py``: views ATTENTION_WINDOW / ATTENTION_GROUP_BY, queries
GRADIENT and NADARAYA_WATSON).  This module only marshals numpy arrays.

Every function takes and returns float64 arrays in the ``[B, H, N, D]``
row-major layout (``[B, H, N]`` for lse).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Return codes of swa_oracle.c
OK, EINVAL, UNDERFLOW, ENOMEM = 0, 1, 2, 3


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile swa_oracle.c with gcc (IEEE float64: no fast-math, no FMA
    contraction) into liboracle.so next to it."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
           "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        Dbl = ctypes.c_double
        lib.oracle_attn_fwd.argtypes = [P, P, P, P, P, I64, I64, I64, I64, I, Dbl, I]
        lib.oracle_attn_fwd_rows.argtypes = [P, P, P, I64, I64, I, Dbl, P, P, I64, P, P, I]
        lib.oracle_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, I64, I64, I64, I64, I, Dbl, I]
        lib.oracle_attn_bwd_rows.argtypes = [P, P, P, P, P, I64, I64, I, Dbl, P, P, I64, P,
                                             P, P, I64, P, P, I]
        lib.oracle_nw.argtypes = [P, I64, P, P, I64, Dbl, P, I]
        lib.oracle_nw_nd.argtypes = [P, I64, P, P, I64, I, Dbl, P, P, I]
        lib.oracle_nw_bwd.argtypes = [P, I64, P, P, I64, I, Dbl, P, P, P, P, I]
        lib.oracle_max_threads.argtypes = []
        for f in (lib.oracle_attn_fwd, lib.oracle_attn_fwd_rows, lib.oracle_attn_bwd,
                  lib.oracle_attn_bwd_rows, lib.oracle_nw, lib.oracle_nw_nd,
                  lib.oracle_nw_bwd, lib.oracle_max_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, allow_underflow: bool) -> None:
    if rc == OK or (rc == UNDERFLOW and allow_underflow):
        return
    if rc == UNDERFLOW:
        raise OracleError("an existing pair's weight underflowed to 0: the inf/NaN "
                          "pattern would depend on 0*inf (outside the contract)")
    raise OracleError(f"oracle returned status {rc}")


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def default_scale(D: int) -> float:
    """1/sqrt(D): exactly 1/8 at D = 64 (the demo's constant D = 64)."""
    return 1.0 / float(np.sqrt(D))


def attn_fwd(q, k, v, causal: bool = True, scale: float | None = None,
             threads: int = 0, allow_underflow: bool = False):
    """Forward: returns (out [B,H,N,D], lse [B,H,N]) in float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = q.shape
    assert k.shape == q.shape and v.shape == q.shape
    scale = default_scale(D) if scale is None else float(scale)
    out = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    rc = _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                 B, H, N, D, int(bool(causal)), scale, int(threads))
    _check(rc, allow_underflow)
    return out, lse


def attn_fwd_rows(q, k, v, heads, rows, causal: bool = True, scale: float | None = None,
                  threads: int = 0, allow_underflow: bool = False):
    """Forward at sampled rows: sample t = row rows[t] of flattened head
    heads[t] (b*H + h).  Returns (out [n, D], lse [n])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = q.shape
    heads, rows = _i64(heads), _i64(rows)
    n = heads.size
    scale = default_scale(D) if scale is None else float(scale)
    out = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = _load().oracle_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), N, D, int(bool(causal)),
                                      scale, _ptr(heads), _ptr(rows), n, _ptr(out),
                                      _ptr(lse), int(threads))
    _check(rc, allow_underflow)
    return out, lse


def attn_bwd(q, k, v, dout, causal: bool = True, scale: float | None = None,
             threads: int = 0, allow_underflow: bool = False, out=None):
    """Backward for upstream gradient dout (dout = out for loss = 1/2 sum out^2).
    Delta_i = dout_i . out_i is evaluated on ``out`` when given (the stored
    forward output a backward pass receives), else on the oracle's own
    float64 output.  Returns (dq, dk, dv), each [B,H,N,D] float64."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, D = q.shape
    given = None if out is None else _f64(out)
    scale = default_scale(D) if scale is None else float(scale)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                                 ctypes.c_void_p(None) if given is None else _ptr(given),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, D, int(bool(causal)),
                                 scale, int(threads))
    _check(rc, allow_underflow)
    return dq, dk, dv


def attn_bwd_rows(q, k, v, dout, qheads, qrows, kheads, krows, causal: bool = True,
                  scale: float | None = None, threads: int = 0,
                  allow_underflow: bool = False, out=None):
    """Backward at sampled rows: dq at (qheads, qrows), dk and dv at
    (kheads, krows); ``out`` as in attn_bwd.  Returns (dq [nq, D], dk [nk, D],
    dv [nk, D])."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    given = None if out is None else _f64(out)
    B, H, N, D = q.shape
    qheads, qrows, kheads, krows = _i64(qheads), _i64(qrows), _i64(kheads), _i64(krows)
    scale = default_scale(D) if scale is None else float(scale)
    dq = np.empty((qheads.size, D), dtype=np.float64)
    dk = np.empty((kheads.size, D), dtype=np.float64)
    dv = np.empty((kheads.size, D), dtype=np.float64)
    rc = _load().oracle_attn_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                                      ctypes.c_void_p(None) if given is None else _ptr(given),
                                      N, D,
                                      int(bool(causal)), scale, _ptr(qheads), _ptr(qrows),
                                      qheads.size, _ptr(dq), _ptr(kheads), _ptr(krows),
                                      kheads.size, _ptr(dk), _ptr(dv), int(threads))
    _check(rc, allow_underflow)
    return dq, dk, dv


def nw_regrid(targets, sources, vals, h: float = 0.5, threads: int = 0):
    """Nadaraya-Watson regrid: targets [M,2], sources [S,2], vals [S] -> out [M]."""
    targets, sources, vals = _f64(targets), _f64(sources), _f64(vals)
    M, S = targets.shape[0], sources.shape[0]
    out = np.empty((M,), dtype=np.float64)
    rc = _load().oracle_nw(_ptr(targets), M, _ptr(sources), _ptr(vals), S, float(h),
                           _ptr(out), int(threads))
    _check(rc, False)
    return out


def nw_regrid_nd(targets, sources, vals, h: float = 0.5, threads: int = 0, with_z=False):
    """Regrid with points of 1, 2 or 3 coordinates: targets [M, d], sources
    [S, d], vals [S] -> out [M] (and Z [M] = sum of weights if with_z)."""
    targets, sources, vals = _f64(targets), _f64(sources), _f64(vals)
    M, dims = targets.shape
    S = sources.shape[0]
    assert sources.shape[1] == dims
    out = np.empty((M,), dtype=np.float64)
    z = np.empty((M,), dtype=np.float64)
    rc = _load().oracle_nw_nd(_ptr(targets), M, _ptr(sources), _ptr(vals), S, dims, float(h),
                              _ptr(out), _ptr(z), int(threads))
    _check(rc, False)
    return (out, z) if with_z else out


def nw_regrid_bwd(targets, sources, vals, gout, h: float = 0.5, threads: int = 0):
    """Gradient of a loss with dL/dout = gout [M] with respect to targets
    [M, d], sources [S, d] and vals [S]: returns (dtargets, dsources, dvals)."""
    targets, sources, vals, gout = _f64(targets), _f64(sources), _f64(vals), _f64(gout)
    M, dims = targets.shape
    S = sources.shape[0]
    dt, ds = np.empty_like(targets), np.empty_like(sources)
    dv = np.empty((S,), dtype=np.float64)
    rc = _load().oracle_nw_bwd(_ptr(targets), M, _ptr(sources), _ptr(vals), S, dims, float(h),
                               _ptr(gout), _ptr(dt), _ptr(ds), _ptr(dv), int(threads))
    _check(rc, False)
    return dt, ds, dv


def qkv_proj(x, w, H: int, D: int = 64):
    """Fused QKV projection in front of attention ("Wiki notes", page 5,
    mini_attention: Q = x Wq, K = x Wk, V = x Wv), float64.  x [B, N, C];
    w [3 H D, C] stacks the output features of Wq, Wk, Wv, one row per
    feature (q feature h*D + d is row h*D + d, k's rows follow, then v's).
    Returns q, k, v as [B, H, N, D].  One library matmul, then the head split
    (no blocking or fusion)."""
    x, w = _f64(x), _f64(w)
    B, N, C = x.shape
    assert w.shape == (3 * H * D, C)
    y = x.reshape(B * N, C) @ w.T                     # [B*N, 3 H D]
    y = y.reshape(B, N, 3, H, D).transpose(2, 0, 3, 1, 4)
    return tuple(np.ascontiguousarray(y[i]) for i in range(3))
