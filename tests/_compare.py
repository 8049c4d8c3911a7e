"""Element-wise comparison of CUDA results with the float64 oracle.

Tolerances (stated once, used by every parity test):
  * float32 path: max |gpu - oracle| <= 1e-5 over the entries where the
    oracle is finite.
  * bf16 path: for every output row (one token's 64 features, the last
    axis), max_d |gpu - oracle| / max(RMS_d(finite oracle entries), 1e-3)
    <= 2e-2.  The RMS is taken per row because the rows' magnitudes span
    decades (out_0 = v_0 while late rows average thousands of values; dq of
    early rows dwarfs later ones): against one tensor-wide RMS, the bf16
    storage rounding of the largest rows alone (2^-9 of the value) would
    exceed the bound.  The floor keeps a row that is exactly zero (dq of a
    single token) from dividing rounding noise by zero; it is stated for
    unit-scale data, and a test whose inputs are scaled by s passes it in the
    output's units (s for out and dv, s^2 for dq and dk when V and dout carry
    the scale).
  * bf16 path, lse: max |gpu - oracle| <= 5e-3 absolute (lse = m + ln z is
    formed in float32 from exactly representable bf16 products, so the
    RMS-relative bound, ~0.2 at |lse| ~ 10, would be needlessly loose).
  * the regrid's gradient (float32): max |gpu - oracle| <= 1e-5 x max(1, max
    |oracle|) per output -- the float32 bound, relative once the values
    exceed 1 (a source's gradient sums over every target near it).
  * every path: the isnan / isposinf / isneginf masks are identical.
"""
from __future__ import annotations

import numpy as np
import torch

F32_ATOL = 1e-5
BF16_REL = 2e-2
RMS_FLOOR = 1e-3
LSE_ATOL = 5e-3


def to_f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def class_masks_equal(got: np.ndarray, want: np.ndarray, name: str) -> None:
    for fn, label in ((np.isnan, "NaN"), (np.isposinf, "+inf"), (np.isneginf, "-inf")):
        g, w = fn(got), fn(want)
        if not np.array_equal(g, w):
            bad = np.argwhere(g != w)
            raise AssertionError(f"{name}: {label} pattern differs at {len(bad)} entries, "
                                 f"first {bad[:5].tolist()}")


def check_f32(got, want, name: str, atol: float = F32_ATOL) -> float:
    g, w = to_f64(got), to_f64(want)
    assert g.shape == w.shape, (name, g.shape, w.shape)
    class_masks_equal(g, w, name)
    fin = np.isfinite(w)
    err = float(np.abs(g[fin] - w[fin]).max()) if fin.any() else 0.0
    assert err <= atol, f"{name}: max abs error {err:.3e} > {atol:.1e}"
    return err


def check_bf16(got, want, name: str, rel: float = BF16_REL, floor: float = RMS_FLOOR) -> float:
    g, w = to_f64(got), to_f64(want)
    assert g.shape == w.shape, (name, g.shape, w.shape)
    class_masks_equal(g, w, name)
    fin = np.isfinite(w)
    if not fin.any():
        return 0.0
    g2 = g.reshape(-1, g.shape[-1])
    w2 = w.reshape(-1, w.shape[-1])
    f2 = fin.reshape(w2.shape)
    wz = np.where(f2, w2, 0.0)
    cnt = np.maximum(f2.sum(axis=1), 1)
    rms = np.sqrt((wz ** 2).sum(axis=1) / cnt)
    diff = np.where(f2, np.abs(g2 - wz), 0.0).max(axis=1)
    ratio = diff / np.maximum(rms, floor)
    err = float(ratio.max())
    worst = int(ratio.argmax())
    assert err <= rel, (f"{name}: max abs error / row RMS = {err:.3e} > {rel:.1e} "
                        f"(row {worst}, rms {rms[worst]:.3e})")
    return err


def check_lse(got, want, name: str, atol: float = LSE_ATOL) -> float:
    return check_f32(got, want, name, atol=atol)


def check_f32_scaled(got, want, name: str, rel: float = F32_ATOL) -> float:
    """float32 bound relative to the output's magnitude once it exceeds 1."""
    w = to_f64(want)
    scale = max(1.0, float(np.abs(w[np.isfinite(w)]).max()) if np.isfinite(w).any() else 1.0)
    return check_f32(got, want, name, atol=rel * scale)
