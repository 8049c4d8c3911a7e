"""CPU-only checks of the C ABI: libswa.so loads, exports every symbol that
include/swa.h declares, and rejects bad arguments on the host before any
CUDA work (no compute call needs a GPU here)."""
import ctypes
import os
import re

import pytest

from causal_attention_swa_b200 import swa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "swa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"\b(swa_[a-z0-9_]+)\s*\(", text))


@pytest.fixture(scope="module")
def lib():
    from causal_attention_swa_b200 import build
    build.build()
    return swa.load_library()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_symbols()
    assert declared, "no declarations found in include/swa.h"
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(swa.EXPORTS)


def test_status_strings(lib):
    assert lib.swa_status_string(0) == b"SWA_OK"
    assert lib.swa_status_string(4) == b"SWA_ERR_DEVICE_TIMEOUT"


def test_workspace_sizes(lib):
    # bf16 forward: four int32 of per-head information and the per-tile masks
    # of V rows with a non-finite entry (16 bytes per 128-row tile), each
    # rounded to 256 bytes, then the f16 copy of V
    B, H, N, D = 2, 16, 16384, 64
    rows = 2 * 16 * (16384 // 128) * 16
    assert lib.swa_attn_fwd_workspace_size(B, H, N, D, swa.SWA_BF16) == 512 + rows + B * H * N * D * 2
    assert lib.swa_attn_fwd_workspace_size(1, 1, 3, 64, swa.SWA_BF16) == 256 + 256 + 512
    assert lib.swa_attn_fwd_workspace_size(1, 1, 256, 64, swa.SWA_F32) == 0
    # backward: information, the masks (bf16), delta and lse*log2(e) padded to
    # 128-row blocks, and for bf16 four f16 operand copies
    want = 512 + rows + 2 * B * H * N * 4 + 4 * B * H * N * D * 2
    assert lib.swa_attn_bwd_workspace_size(B, H, N, D, swa.SWA_BF16) == want
    assert lib.swa_attn_grad_workspace_size(B, H, N, D, swa.SWA_BF16) == want
    assert lib.swa_attn_bwd_workspace_size(1, 1, 256, 64, swa.SWA_F32) == 256 + 2 * 1024
    assert lib.swa_attn_bwd_workspace_size(1, 1, 300, 64, swa.SWA_F32) == 256 + 2 * 1536
    assert lib.swa_nw_workspace_size(16384, 16384) > 0


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced


@pytest.mark.parametrize("args,code", [
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 32, 1, swa.SWA_BF16), swa.SWA_ERR_UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 16, 64, 1, swa.SWA_BF16), swa.SWA_ERR_INVALID_ARGUMENT),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 64, 1, swa.SWA_BF16), swa.SWA_ERR_INVALID_ARGUMENT),
    ((None, FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, 1, swa.SWA_BF16), swa.SWA_ERR_INVALID_ARGUMENT),
    ((FAKE + 8, FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, 1, swa.SWA_BF16),
     swa.SWA_ERR_INVALID_ARGUMENT),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, 1, 7), swa.SWA_ERR_INVALID_ARGUMENT),
    ((FAKE, FAKE, FAKE, FAKE, FAKE, 300, 300, 16, 64, 1, swa.SWA_BF16), swa.SWA_ERR_UNSUPPORTED),
])
def test_fwd_argument_errors_return_before_launch(lib, args, code):
    st = lib.swa_attn_fwd(*args, FAKE, 1 << 20, None)
    assert st == code, lib.swa_last_error_message()
    assert lib.swa_last_error_message() != b""


def test_fwd_small_workspace_is_rejected(lib):
    st = lib.swa_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 16, 64, 1, swa.SWA_BF16,
                          FAKE, 4, None)
    assert st == swa.SWA_ERR_INVALID_ARGUMENT
    assert b"workspace" in lib.swa_last_error_message()


def test_bwd_argument_errors(lib):
    good = [FAKE] * 9
    st = lib.swa_attn_bwd(*good, 1, 1, 16, 64, 1, swa.SWA_BF16, FAKE, 16, None)
    assert st == swa.SWA_ERR_INVALID_ARGUMENT  # workspace too small
    bad = list(good)
    bad[6] = None  # dq
    st = lib.swa_attn_bwd(*bad, 1, 1, 16, 64, 1, swa.SWA_BF16, FAKE, 1 << 30, None)
    assert st == swa.SWA_ERR_INVALID_ARGUMENT


def test_grad_argument_errors(lib):
    good = [FAKE] * 8
    st = lib.swa_attn_grad(*good, 1, 1, 16, 64, 1, swa.SWA_BF16, FAKE, 16, None)
    assert st == swa.SWA_ERR_INVALID_ARGUMENT  # workspace too small
    assert b"workspace" in lib.swa_last_error_message()
    bad = list(good)
    bad[7] = None  # dv
    st = lib.swa_attn_grad(*bad, 1, 1, 16, 64, 1, swa.SWA_BF16, FAKE, 1 << 30, None)
    assert st == swa.SWA_ERR_INVALID_ARGUMENT
    st = lib.swa_attn_grad(*good, 1, 1, 16, 128, 1, swa.SWA_BF16, FAKE, 1 << 30, None)
    assert st == swa.SWA_ERR_UNSUPPORTED


def test_nw_argument_errors(lib):
    F = ctypes.c_float
    assert lib.swa_nw_regrid(FAKE, 0, FAKE, FAKE, 4, F(0.5), FAKE, FAKE, 1 << 20, None) == \
        swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_nw_regrid(FAKE, 4, FAKE, FAKE, 4, F(0.0), FAKE, FAKE, 1 << 20, None) == \
        swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_nw_regrid(FAKE, 4, FAKE, FAKE, 4, F(float("nan")), FAKE, FAKE, 1 << 20,
                             None) == swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_nw_regrid(FAKE, 4, FAKE + 4, FAKE, 4, F(0.5), FAKE, FAKE, 1 << 20, None) == \
        swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_nw_regrid(FAKE, 4, FAKE, FAKE, 4, F(0.5), FAKE, FAKE, 8, None) == \
        swa.SWA_ERR_INVALID_ARGUMENT


def test_nw_nd_and_gradient_argument_errors(lib):
    F = ctypes.c_float
    for dims, code in ((0, swa.SWA_ERR_UNSUPPORTED), (4, swa.SWA_ERR_UNSUPPORTED)):
        assert lib.swa_nw_regrid_nd(FAKE, 4, FAKE, FAKE, 4, dims, F(0.5), FAKE, FAKE, 1 << 20,
                                    None) == code
        assert lib.swa_nw_regrid_bwd(FAKE, 4, FAKE, FAKE, 4, dims, F(0.5), FAKE, FAKE, FAKE,
                                     FAKE, FAKE, 1 << 30, None) == code
    assert lib.swa_nw_regrid_bwd(FAKE, 4, FAKE, FAKE, 4, 3, F(0.5), None, FAKE, FAKE, FAKE,
                                 FAKE, 1 << 30, None) == swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_nw_regrid_bwd(FAKE, 4, FAKE, FAKE, 4, 3, F(0.5), FAKE, FAKE, FAKE, FAKE,
                                 FAKE, 8, None) == swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_nw_regrid_bwd_workspace_size(16384, 16384, 2) > 0
    # the largest S the API accepts plans at most 65535 source chunks (grid.y):
    # one target's partials then take at most 65535 x 8 bytes
    assert 0 < lib.swa_nw_workspace_size(1, 1 << 31) <= (65535 * 8 + 255) // 256 * 256


def test_merge_argument_errors(lib):
    ok = (FAKE, FAKE, FAKE, FAKE, None, 128, 64, 1, swa.SWA_BF16, None)

    def call(**kw):
        names = ("op", "lp", "oa", "la", "of", "rows", "D", "first", "dt", "s")
        args = dict(zip(names, ok))
        args.update(kw)
        return lib.swa_attn_merge(*(args[n] for n in names))
    assert call(D=32) == swa.SWA_ERR_UNSUPPORTED
    assert call(rows=0) == swa.SWA_ERR_INVALID_ARGUMENT
    assert call(rows=(1 << 31) + 1) == swa.SWA_ERR_INVALID_ARGUMENT
    assert call(op=None) == swa.SWA_ERR_INVALID_ARGUMENT
    assert call(la=FAKE + 4) == swa.SWA_ERR_INVALID_ARGUMENT
    assert call(of=FAKE + 8) == swa.SWA_ERR_INVALID_ARGUMENT
    assert call(dt=7) == swa.SWA_ERR_INVALID_ARGUMENT


def test_accumulating_backward_and_cast_argument_errors(lib):
    ws = 1 << 30
    args = [FAKE] * 9 + [1, 2, 256, 64, 1, swa.SWA_BF16, FAKE, ws, None]
    for i in (6, 7, 8):  # a missing float32 sum
        bad = list(args)
        bad[i] = None
        assert lib.swa_attn_bwd_acc(*bad) == swa.SWA_ERR_INVALID_ARGUMENT
    f32 = list(args)
    f32[14] = swa.SWA_F32
    assert lib.swa_attn_bwd_acc(*f32) == swa.SWA_ERR_UNSUPPORTED
    small = list(args)
    small[16] = 64
    assert lib.swa_attn_bwd_acc(*small) == swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_f32_to_bf16(FAKE, FAKE, 12, None) == swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_f32_to_bf16(FAKE, FAKE, 0, None) == swa.SWA_ERR_INVALID_ARGUMENT
    assert lib.swa_f32_to_bf16(None, FAKE, 64, None) == swa.SWA_ERR_INVALID_ARGUMENT


def test_product_path_does_not_import_the_oracle():
    """The CUDA binding never reaches the oracle (no CPU fallback)."""
    pkg = os.path.join(ROOT, "causal_attention_swa_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "swa_oracle" not in text and "liboracle" not in text, f


@pytest.mark.parametrize("bad", ["k_shape", "v_dtype", "out_shape", "lse_dtype"])
def test_binding_rejects_mismatched_tensors_before_any_launch(bad):
    """The C ABI takes B, H, N, D from q alone; the binding must refuse any
    other tensor whose shape or dtype disagrees (it would be read out of
    bounds), before touching the GPU."""
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    k, v = q.clone(), q.clone()
    out, lse = q.clone(), torch.zeros(1, 2, 8, dtype=torch.float32)
    if bad == "k_shape":
        k = torch.zeros(1, 2, 7, 64, dtype=torch.bfloat16)
    elif bad == "v_dtype":
        v = v.float()
    elif bad == "out_shape":
        out = torch.zeros(1, 2, 8, 32, dtype=torch.bfloat16)
    else:
        lse = lse.double()
    with pytest.raises(ValueError, match="expected shape"):
        swa.attn_fwd(q, k, v, out=out, lse=lse)
    with pytest.raises(ValueError, match="expected shape"):
        swa.attn_bwd(q, k, v, out, out, lse)
    if bad != "lse_dtype":
        with pytest.raises(ValueError, match="expected shape"):
            swa.attn_grad(q, k, v, out=out)


def test_binding_rejects_mismatched_regrid_tensors():
    import torch
    t = torch.zeros(5, 2)
    src = torch.zeros(7, 2)
    with pytest.raises(ValueError, match="expected shape"):
        swa.nw_regrid(t, src, torch.zeros(6))
