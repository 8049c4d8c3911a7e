"""GPU parity of the QKV projection in front of attention ("Wiki notes",
page 5, mini_attention: Q = x Wq, K = x Wk, V = x Wv) through the C ABI,
against the float64 oracle (x w^T and the head split), element by element:
ragged token counts, an odd head count (a tile that straddles q and k), a
case with several tiles per block of the persistent grid and ragged edges
in both directions, and the projection of the 2 x 16384-token, 16-head
workload (C = 1024).
Tolerance: the bf16 per-row bound of tests/_compare.py."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_swa_b200 import inputs, swa
from _compare import check_bf16

pytestmark = pytest.mark.gpu


def dev16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def check(B, N, C, H, seed):
    xb, wb = inputs.qkv_inputs(B, N, C, H, seed)
    q, k, v = swa.qkv_proj(dev16(xb), dev16(wb), H)
    torch.cuda.synchronize()
    assert swa.last_launch_count() == 1
    assert swa.get_device_error() == swa.SWA_OK
    want = oracle.qkv_proj(inputs.bf16_to_f64(xb), inputs.bf16_to_f64(wb), H)
    for name, g, w in zip("qkv", (q, k, v), want):
        check_bf16(g, w, f"{name} ({B}x{N}x{C}, H={H})")


@pytest.mark.parametrize("B,N,C,H", [(1, 1, 64, 1), (1, 300, 128, 2), (2, 129, 192, 3),
                                     (3, 77, 512, 5)])
def test_qkv_projection_small(B, N, C, H):
    check(B, N, C, H, seed=B * 1000 + N + C + H)


def test_qkv_projection_b2_n16384_c1024_h16():
    check(2, 16384, 1024, 16, seed=6)


def test_qkv_projection_many_tiles_per_block_with_ragged_edges():
    # 20000 tokens (157 token tiles, the last 32 rows) x 960 features (4
    # feature tiles, the last 192 wide): 628 tiles, so every block of the
    # persistent grid takes several and both TMEM accumulators take turns
    check(1, 20000, 128, 5, seed=7)


def test_qkv_projection_rejects_unsupported_shapes():
    x = torch.zeros(1, 8, 96, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(3 * 64, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(swa.SwaError):
        swa.qkv_proj(x, w, 1)  # C = 96 is not a multiple of 64
