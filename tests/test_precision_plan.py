"""CPU check of the backward's precision plan, by float32/bf16 emulation of
the tensor-core kernels' arithmetic (fp32 S and dP from bf16 operands, P in
fp32, dS rounded as the kernels round it, fp32 accumulation, bf16 outputs)
against the float64 oracle, with the per-row metric of the GPU tests:

  * dq with dS as bf16 hi + lo stays well inside the 2e-2 bound, while a
    single bf16 rounding of dS comes close to it (the cancellation that
    sum_j dS_ij = 0 brings to sum_j dS_ij k_j);
  * dk with dS^T at bf16 (as the dK/dV kernel takes it) stays inside it.

Emulation only (numpy + the oracle); no GPU."""
import numpy as np
import pytest

import oracle
from causal_attention_swa_b200 import inputs

pytestmark = pytest.mark.parametrize("N", [256, 1024])


def _bf(x):
    return inputs.bf16_to_f64(inputs.bf16_bits(np.asarray(x, np.float32)))


def _f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


def _row_err(g, w):
    rms = np.maximum(np.sqrt((w ** 2).mean(axis=1)), 1e-3)
    return float((np.abs(g - w).max(axis=1) / rms).max())


def test_dq_needs_hi_lo_and_dk_takes_bf16(N):
    rng = np.random.default_rng(N)
    B, H = 1, 2
    bits = [inputs.bf16_bits(rng.standard_normal((B, H, N, 64), dtype=np.float32))
            for _ in range(3)]
    q, k, v = (inputs.bf16_to_f64(b) for b in bits)
    w_out, w_lse = oracle.attn_fwd(q, k, v)
    out = _bf(w_out)  # the stored (bf16) output the backward is given; dout = out
    w_dq, w_dk, _ = oracle.attn_bwd(q, k, v, out, out=out)
    err = {"dq_bf16": 0.0, "dq_hilo": 0.0, "dk_bf16": 0.0}
    for h in range(H):
        Q, K, V, O = q[0, h], k[0, h], v[0, h], out[0, h]
        S = _f32(Q @ K.T)
        P = np.tril(np.exp(S / 8 - w_lse[0, h][:, None]))
        dP = _f32(O @ V.T)
        delta = _f32((O * O).sum(axis=1))
        dS = np.tril(_f32(_f32(P) * (dP - delta[:, None])))
        hi = _bf(dS)
        hilo = hi + _bf(dS - hi)
        err["dq_bf16"] = max(err["dq_bf16"], _row_err(_bf(_f32(hi @ K) / 8), w_dq[0, h]))
        err["dq_hilo"] = max(err["dq_hilo"], _row_err(_bf(_f32(hilo @ K) / 8), w_dq[0, h]))
        err["dk_bf16"] = max(err["dk_bf16"], _row_err(_bf(_f32(hi.T @ Q) / 8), w_dk[0, h]))
    assert err["dq_hilo"] < 1.5e-2, err
    assert err["dk_bf16"] < 2e-2, err
    assert err["dq_hilo"] < err["dq_bf16"], err
