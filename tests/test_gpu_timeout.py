"""Failure detection on the GPU without a fault: a kernel whose bounded waits
(parked and polling, one block each) run out (nothing arrives at their
barriers) leaves SWA_ERR_DEVICE_TIMEOUT in the
device error word, the word is cleared once read, and the context stays
usable: an attention call afterwards still matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_swa_b200 import inputs, swa
from _compare import check_bf16, check_lse

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_stays_usable():
    torch.cuda.synchronize()
    assert swa.get_device_error() == swa.SWA_OK
    swa.selftest_wait_timeout()
    assert swa.get_device_error() == swa.SWA_ERR_DEVICE_TIMEOUT
    assert swa.get_device_error() == swa.SWA_OK  # read once, then cleared
    rng = np.random.default_rng(21)
    bits = [inputs.bf16_bits(rng.standard_normal((1, 2, 300, 64), dtype=np.float32))
            for _ in range(3)]
    q, k, v = (torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda() for b in bits)
    out, lse = swa.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert swa.get_device_error() == swa.SWA_OK
    w_out, w_lse = oracle.attn_fwd(*(inputs.bf16_to_f64(b) for b in bits))
    check_bf16(out, w_out, "out")
    check_lse(lse, w_lse, "lse")
