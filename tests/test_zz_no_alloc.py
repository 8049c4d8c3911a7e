"""swa_attn_fwd_noalloc: the attention forward for callers that cannot
allocate device memory (their host application owns every device buffer,
or their latency budget rules out cudaMalloc and its synchronisation).  Its
per-head scratch lives in a static device array shared by every call, so
this test makes two calls in a row -- the first with a head whose V holds
+inf (its flag gets set), the second with all heads finite (the flag must
have been cleared) -- and checks each against the float64 oracle with the
parity tests' tolerances, through the C ABI.  Without room for an f16 copy
of V its P V products take bf16 operands, so it is not bitwise equal to
swa_attn_fwd: each is within the per-row bound of the exact result, so the
two lie within twice that bound of each other.  It is collected last so a
failure here cannot hide the other tests' results."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from causal_attention_swa_b200 import inputs, swa
from _compare import BF16_REL, check_bf16, check_f32, check_lse

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = swa.load_library()
    f = lib.swa_attn_fwd_noalloc
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f.argtypes = [P, P, P, P, P, I64, I64, I64, I64, I, I, P]
    f.restype = I
    return lib, f


def _call_noalloc(q, k, v, causal=True):
    lib, f = _noalloc_fn()
    B, H, N, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dt = swa.SWA_BF16 if q.dtype == torch.bfloat16 else swa.SWA_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = f(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
           ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
           ctypes.c_void_p(lse.data_ptr()), B, H, N, D, int(causal), dt, stream)
    assert st == swa.SWA_OK, lib.swa_last_error_message()
    return out, lse


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def test_noalloc_forward_matches_the_oracle_twice_in_a_row():
    torch.cuda.init()
    rng = np.random.default_rng(77)
    shape = (2, 3, 300, 64)
    first = [inputs.bf16_bits(rng.standard_normal(shape, dtype=np.float32)) for _ in range(3)]
    first[2][1, 2, 150, 9] = 0x7F80           # +inf in V of head (1, 2)
    second = [inputs.bf16_bits(rng.standard_normal(shape, dtype=np.float32)) for _ in range(3)]
    for bits in (first, second):
        q, k, v = (_bf16_dev(b) for b in bits)
        got_out, got_lse = _call_noalloc(q, k, v)
        want_out, want_lse = swa.attn_fwd(q, k, v, causal=True)
        torch.cuda.synchronize()
        assert swa.get_device_error() == swa.SWA_OK
        # the float64 oracle (classes of the +inf head included)
        w_out, w_lse = oracle.attn_fwd(*(inputs.bf16_to_f64(b) for b in bits))
        check_bf16(got_out, w_out, "out (noalloc vs oracle)")
        check_lse(got_lse, w_lse, "lse (noalloc vs oracle)")
        # the workspace forward: both within BF16_REL of the exact rows
        check_bf16(got_out, want_out, "out (noalloc vs workspace forward)", rel=2 * BF16_REL)
        check_lse(got_lse, want_lse, "lse (noalloc vs workspace forward)")
    o = got_out.float().cpu().numpy()
    assert np.isfinite(o).all()                # second call: no stale flag, no inf


def test_noalloc_forward_allocates_no_device_memory():
    """After a first call (which looks up the static array's address), more
    calls change neither the device's free memory nor torch's allocations."""
    rng = np.random.default_rng(5)
    bits = [inputs.bf16_bits(rng.standard_normal((1, 4, 512, 64), dtype=np.float32))
            for _ in range(3)]
    q, k, v = (_bf16_dev(b) for b in bits)
    out = torch.empty_like(q)
    lse = torch.empty((1, 4, 512), dtype=torch.float32, device=q.device)
    lib, f = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = (ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(lse.data_ptr()), 1, 4, 512, 64, 1, swa.SWA_BF16, stream)
    assert f(*args) == swa.SWA_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(5):
        assert f(*args) == swa.SWA_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == alloc0


def test_noalloc_forward_float32_path():
    q, k, v = (torch.from_numpy(a.astype(np.float32)).cuda()
               for a in inputs.single_head_f64(256, inf_at=(100, 3)))
    for _ in range(2):
        got_out, got_lse = _call_noalloc(q, k, v)
        want_out, want_lse = swa.attn_fwd(q, k, v, causal=True)
        torch.cuda.synchronize()
        check_f32(got_out, want_out, "out f32 (noalloc)")
        check_f32(got_lse, want_lse, "lse f32 (noalloc)")


def test_noalloc_rejects_more_heads_than_its_static_scratch_holds():
    lib, f = _noalloc_fn()
    fake = ctypes.c_void_p(1 << 20)
    st = f(fake, fake, fake, fake, fake, 1, 4097, 16, 64, 1, swa.SWA_BF16, None)
    assert st == swa.SWA_ERR_UNSUPPORTED
    assert b"4096" in lib.swa_last_error_message()
