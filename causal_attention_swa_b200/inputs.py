"""Seeded synthetic inputs for the attention and regrid workloads.

This module draws random numbers and rounds them to the storage types; it
holds none of the method's arithmetic, so both the float64 oracle (tests)
and the CUDA path consume exactly the values produced here.

Recipes (numpy ``default_rng`` = PCG64, one generator per workload):

* ``pages_main``: the demo's ``main()`` of "Show HN: Automatic deduction of
  FlashAttention kernel from ~25 lines of SQL" (page 2): seed 0, for each
  size n in (64, 256) draw q, k, v ~ N(0,1) of shape (n, 64) in that order
  from one generator.  The n = 256 draw is the single-head float64 workload.
* ``pages_mask``: ``check_masks_are_absent_rows``: n = 16, seed 1, q, k, v
  ~ N(0,1), then v[9, 0] = +inf.
* ``pages_nw``: ``check_nadaraya_watson``: seed 2, 64 targets and 256
  sources uniform in [0,1]^2, y = sin(4 x) + cos(3 y).
* ``nw_grid``: 16384 sources uniform in [0,10]^2 with values
  sin(x) cos(y) + 0.1 N(0,1), 16384 targets uniform in [0,10]^2, seed 2,
  stored as float32.
* ``nw_grid_nd``: the regrid workload with points of 1, 2 or 3 coordinates
  uniform in [0,10]^d, values sin(x) cos(y) cos(z) (the factors that exist)
  + 0.1 N(0,1), seed 2, stored as float32; d = 2 is ``nw_grid``.
* ``qkv_inputs``: the projection's input x ~ N(0,1) [B, N, C] and weight
  w ~ N(0, 1/C) [3 H 64, C] (so q, k, v come out ~ N(0,1)), drawn as float32
  in that order and rounded to bfloat16.
* ``attn_bf16_batch``: the same per sequence: sequence b of a batch draws
  its q, k, v [H, N, D] from ``default_rng([seed, b])``, so any block of
  sequences is drawn without the others (the multi-GPU split of one batch).
* ``nw_targets_block``: block r of a regrid's target set -- block 0 is
  ``nw_grid``'s targets, block r > 0 is drawn from ``default_rng([seed, r])``
  uniform in [0,10]^2.
* ``attn_bf16``: Q, K, V iid normal (std per tensor) drawn as float32 in the
  order q, k, v, rounded to bfloat16 (round to nearest even), layout
  [B, H, N, D]; optionally a number of V entries set to +inf at positions
  from ``rng.choice(total, count, replace=False)`` drawn after v.
"""
from __future__ import annotations

import numpy as np

D = 64


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even) and
    return the 16-bit patterns as uint16.  Infinities stay infinities; NaN
    stays a quiet NaN."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact float64 value of bfloat16 bit patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def pages_main(sizes=(64, 256)):
    """{n: (q, k, v)} float64 (n, 64) arrays in the demo main()'s draw order."""
    rng = np.random.default_rng(0)
    out = {}
    for n in sizes:
        q, k, v = (rng.normal(size=(n, D)) for _ in range(3))
        out[n] = (q, k, v)
    return out


def single_head_f64(n: int = 256, inf_at=None):
    """The n-token draw of ``pages_main`` as [1, 1, n, 64] float64 arrays.
    ``inf_at = (j, d)`` puts +inf at V[j, d] of a copy."""
    q, k, v = pages_main()[n]
    v = v.copy()
    if inf_at is not None:
        v[inf_at[0], inf_at[1]] = np.inf
    return tuple(a.reshape(1, 1, n, D) for a in (q, k, v))


def pages_mask(n: int = 16, j: int = 9):
    """check_masks_are_absent_rows inputs as [1, 1, n, 64] float64."""
    rng = np.random.default_rng(1)
    q, k, v = (rng.normal(size=(n, D)) for _ in range(3))
    v[j, 0] = np.inf
    return tuple(a.reshape(1, 1, n, D) for a in (q, k, v))


def pages_nw():
    """check_nadaraya_watson inputs: targets [64,2], sources [256,2], y [256]."""
    rng = np.random.default_rng(2)
    targets, sources = rng.uniform(size=(64, 2)), rng.uniform(size=(256, 2))
    y = np.sin(4 * sources[:, 0]) + np.cos(3 * sources[:, 1])
    return targets, sources, y


def nw_grid(M: int = 16384, S: int = 16384, seed: int = 2):
    """Regrid workload as float32: targets [M,2], sources [S,2], vals [S]."""
    rng = np.random.default_rng(seed)
    sources = rng.uniform(0.0, 10.0, size=(S, 2))
    noise = rng.normal(size=S)
    targets = rng.uniform(0.0, 10.0, size=(M, 2))
    vals = np.sin(sources[:, 0]) * np.cos(sources[:, 1]) + 0.1 * noise
    return (targets.astype(np.float32), sources.astype(np.float32), vals.astype(np.float32))


def nw_grid_nd(M: int = 16384, S: int = 16384, dims: int = 2, seed: int = 2):
    """Regrid workload with points of `dims` coordinates, float32:
    targets [M, dims], sources [S, dims], vals [S]."""
    if dims == 2:
        return nw_grid(M, S, seed)
    rng = np.random.default_rng(seed)
    sources = rng.uniform(0.0, 10.0, size=(S, dims))
    noise = rng.normal(size=S)
    targets = rng.uniform(0.0, 10.0, size=(M, dims))
    vals = np.sin(sources[:, 0]) + 0.1 * noise
    if dims == 3:
        vals = np.sin(sources[:, 0]) * np.cos(sources[:, 1]) * np.cos(sources[:, 2]) + 0.1 * noise
    return (targets.astype(np.float32), sources.astype(np.float32), vals.astype(np.float32))


def qkv_inputs(B: int, N: int, C: int, H: int, seed: int):
    """(x, w) as uint16 bfloat16 bit patterns: x [B, N, C], w [3*H*64, C]."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(size=(B, N, C), dtype=np.float32)
    w = rng.standard_normal(size=(3 * H * D, C), dtype=np.float32) * np.float32(C ** -0.5)
    return bf16_bits(x), bf16_bits(w)


def attn_bf16(B: int, H: int, N: int, seed: int, qk_std: float = 1.0, v_std: float = 1.0,
              n_inf: int = 0):
    """(q, k, v) as uint16 bfloat16 bit patterns [B, H, N, 64], and the flat
    indices of the V entries set to +inf (empty unless n_inf > 0)."""
    rng = np.random.default_rng(seed)
    shape = (B, H, N, D)
    q = rng.standard_normal(size=shape, dtype=np.float32)
    k = rng.standard_normal(size=shape, dtype=np.float32)
    v = rng.standard_normal(size=shape, dtype=np.float32)
    if qk_std != 1.0:
        q *= np.float32(qk_std)
        k *= np.float32(qk_std)
    if v_std != 1.0:
        v *= np.float32(v_std)
    pos = np.zeros(0, dtype=np.int64)
    if n_inf:
        pos = rng.choice(v.size, n_inf, replace=False).astype(np.int64)
        v.reshape(-1)[pos] = np.inf
    return bf16_bits(q), bf16_bits(k), bf16_bits(v), pos


def attn_bf16_batch(B: int, H: int, N: int, seed: int, first: int = 0, qk_std: float = 1.0,
                    v_std: float = 1.0):
    """Sequences first .. first+B-1 of a batch whose sequence b draws q, k, v
    ~ N(0, std^2) [H, N, 64] (float32, then bf16) from default_rng([seed, b]).
    Returns uint16 bf16 patterns q, k, v [B, H, N, 64]."""
    out = [np.empty((B, H, N, D), dtype=np.uint16) for _ in range(3)]
    for i in range(B):
        rng = np.random.default_rng([seed, first + i])
        for t, std in zip(out, (qk_std, qk_std, v_std)):
            x = rng.standard_normal(size=(H, N, D), dtype=np.float32)
            if std != 1.0:
                x *= np.float32(std)
            t[i] = bf16_bits(x)
    return tuple(out)


def nw_targets_block(M: int, block: int, seed: int = 2):
    """Block `block` of M regrid targets (float32 [M, 2])."""
    if block == 0:
        return nw_grid(M, M, seed)[0]
    rng = np.random.default_rng([seed, block])
    return rng.uniform(0.0, 10.0, size=(M, 2)).astype(np.float32)


# Named workloads: shapes and seeds.
WORKLOADS = {
    "attn_fwd_b4h16n4096": dict(B=4, H=16, N=4096, seed=3),
    # drawn per sequence (attn_bf16_batch): the benchmark's batch, split
    # across GPUs by sequences
    "attn_fwdbwd_b2h16n16384": dict(B=2, H=16, N=16384, seed=4),
    "attn_fwdbwd_b1h8n65536": dict(B=1, H=8, N=65536, seed=5, qk_std=0.5),
    # a sequence for an 8-rank ring (16 zigzag chunks of 8192 tokens)
    "attn_ring_b1h8n131072": dict(B=1, H=8, N=131072, seed=6, qk_std=0.5),
}

# 0.01% of V's 1*8*65536*64 entries, rounded: 3355 entries set to +inf.
LONG_CONTEXT_N_INF = int(round(1e-4 * 1 * 8 * 65536 * 64))
