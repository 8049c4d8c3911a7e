"""GPU parity of the attention path (through the C ABI) against the float64
oracle, element by element.

Workloads: the demo's own inputs ("Show HN: Automatic deduction of
FlashAttention kernel from ~25 lines of SQL", main(): seed 0, 64 and 256
tokens, D = 64) on the float32 path; the mask test of
check_masks_are_absent_rows on both paths; small bf16 shapes that span
several 128-row tiles with ragged tails; non-finite V and dout on the
tensor-core path; and the three large bf16 workloads (4x16x4096 forward in
full, 2x16x16384 forward+backward, 1x8x65536 forward+backward with and
without 0.01% of V set to +inf), checked on whole heads and at sampled rows
against the oracle and everywhere through properties that hold at any size.

Two backward comparisons:
  * end to end (the GRADIENT query, swa_attn_grad): dq, dk, dv of
    loss = 1/2 sum out^2 from q, k, v alone, against the oracle's gradient
    at its own float64 output;
  * the kernel unit test (swa_attn_bwd): the GPU's stored bf16 output fed
    back as dout = out, against the oracle's backward at that same stored
    output (same dout, same Delta basis on both sides).
Tolerances: tests/_compare.py.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_swa_b200 import inputs, swa
from _compare import RMS_FLOOR, check_bf16, check_f32, check_lse, to_f64

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


# Kernels one bf16 call enqueues: forward = V scan + the f16- and bf16-operand
# tensor-core instances; backward = prep + (dK/dV and dQ kernels) x (f16 and
# bf16 instances); gradient = prep + forward (2) + backward (4).  No call of
# the bf16 path enqueues a CUDA-core attention kernel, whatever V and dout
# hold.
BF16_FWD_LAUNCHES, BF16_BWD_LAUNCHES, BF16_GRAD_LAUNCHES = 3, 5, 7


def run_fwd_bwd(q, k, v, causal=True, backward=True):
    out, lse = swa.attn_fwd(q, k, v, causal=causal)
    if q.dtype == torch.bfloat16:
        assert swa.last_launch_count() == BF16_FWD_LAUNCHES
    grads = swa.attn_bwd(q, k, v, out, out, lse, causal=causal) if backward else None
    if backward and q.dtype == torch.bfloat16:
        assert swa.last_launch_count() == BF16_BWD_LAUNCHES
    torch.cuda.synchronize()
    assert swa.get_device_error() == swa.SWA_OK
    return out, lse, grads


def run_grad(q, k, v, causal=True):
    """swa_attn_grad: (out, lse, dq, dk, dv) of loss = 1/2 sum out^2."""
    res = swa.attn_grad(q, k, v, causal=causal)
    if q.dtype == torch.bfloat16:
        assert swa.last_launch_count() == BF16_GRAD_LAUNCHES
    torch.cuda.synchronize()
    assert swa.get_device_error() == swa.SWA_OK
    return res


def check_end_to_end(q, k, v, res, causal=True, what="", v_scale=1.0):
    """The GRADIENT query end to end: swa_attn_grad's (out, lse, dq, dk, dv)
    against the oracle's forward and its gradient of 1/2 sum out^2 at its own
    float64 output (q, k, v float64 [B, H, N, 64]).  v_scale: the scale of V
    (the RMS floor in the outputs' units)."""
    w_out, w_lse = oracle.attn_fwd(q, k, v, causal=causal)
    check_bf16(res[0], w_out, f"out (gradient call){what}", floor=RMS_FLOOR * v_scale)
    check_lse(res[1], w_lse, f"lse (gradient call){what}")
    w = oracle.attn_bwd(q, k, v, w_out, causal=causal)
    for name, g, ww, f in zip(("dq", "dk", "dv"), res[2:], w, (2, 2, 1)):
        check_bf16(g, ww, f"{name} end to end{what}", floor=RMS_FLOOR * v_scale ** f)


# ------------------------------------------------------------ float32 path

@pytest.mark.parametrize("n", [64, 256])
def test_f32_demo_inputs_forward_and_gradient(n):
    q, k, v = (a[None, None] for a in inputs.pages_main()[n])
    out, lse, (dq, dk, dv) = run_fwd_bwd(dev_f32(q), dev_f32(k), dev_f32(v))
    w_out, w_lse = oracle.attn_fwd(q, k, v)
    check_f32(out, w_out, "out")
    check_f32(lse, w_lse, "lse")
    w_dq, w_dk, w_dv = oracle.attn_bwd(q, k, v, w_out)
    check_f32(dq, w_dq, "dq")
    check_f32(dk, w_dk, "dk")
    check_f32(dv, w_dv, "dv")


def test_f32_single_head_inf_in_v():
    """+inf at V[100, 3] of the 256-token draw: exact inf/NaN pattern of out
    and of every gradient, finite entries within 1e-5."""
    q, k, v = inputs.single_head_f64(256, inf_at=(100, 3))
    out, lse, (dq, dk, dv) = run_fwd_bwd(dev_f32(q), dev_f32(k), dev_f32(v))
    w_out, w_lse = oracle.attn_fwd(q, k, v)
    check_f32(out, w_out, "out")
    o = to_f64(out)[0, 0]
    assert np.isfinite(o[:100]).all() and np.isposinf(o[100:, 3]).all()
    check_f32(lse, w_lse, "lse")
    w = oracle.attn_bwd(q, k, v, w_out)
    for name, g, ww in zip(("dq", "dk", "dv"), (dq, dk, dv), w):
        check_f32(g, ww, name)


def test_f32_inf_survives_a_rescale_that_underflows():
    """+inf at V[0, 3], then (in a later 16-key chunk of the pair-by-pair
    kernel) key 20 scoring 120 above the others: the running max jumps by
    120 / ln 2 ~ 173 in the log2 domain, the rescale factor 2^-173 flushes
    to 0, and the +inf already accumulated must stay +inf (the oracle's
    weight e^-120 of key 0 is > 0), not become 0 * inf = NaN."""
    N, D = 32, 64
    q = np.zeros((1, 1, N, D))
    k = np.zeros((1, 1, N, D))
    v = np.random.default_rng(3).normal(size=(1, 1, N, D))
    q[..., 0] = 1.0
    k[0, 0, 20, 0] = 960.0           # s = q.k / 8 = 120 for key 20
    v[0, 0, 0, 3] = np.inf
    out, lse, _ = run_fwd_bwd(dev_f32(q), dev_f32(k), dev_f32(v), backward=False)
    w_out, w_lse = oracle.attn_fwd(q, k, v)
    assert np.isposinf(to_f64(out)[0, 0, 20:, 3]).all()
    check_f32(out, w_out, "out")
    check_f32(lse, w_lse, "lse", atol=1e-4)  # |lse| ~ 120: float32 spacing 7.6e-6


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pages_mask_test(dtype):
    """check_masks_are_absent_rows: n = 16, seed 1, V[9, 0] = +inf."""
    q, k, v = inputs.pages_mask(16, 9)
    if dtype == "f32":
        tq, tk, tv = dev_f32(q), dev_f32(k), dev_f32(v)
    else:
        tq, tk, tv = (dev_bf16(inputs.bf16_bits(a.astype(np.float32))) for a in (q, k, v))
    out, _, _ = run_fwd_bwd(tq, tk, tv, backward=False)
    o = to_f64(out)[0, 0]
    assert np.isfinite(o[:9]).all()
    assert np.isposinf(o[9:, 0]).all()
    assert np.isfinite(o[:, 1:]).all()


# --------------------------------------------------------------- bf16 path

def bf16_case(B, H, N, seed, std=1.0):
    rng = np.random.default_rng(seed)
    bits = [inputs.bf16_bits(std * rng.standard_normal((B, H, N, 64), dtype=np.float32))
            for _ in range(3)]
    return bits, [inputs.bf16_to_f64(b) for b in bits]


@pytest.mark.parametrize("N", [1, 7, 64, 127, 128, 129, 255, 256, 257, 383, 640])
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_small_shapes_forward_and_gradient(N, causal):
    bits, (q, k, v) = bf16_case(2, 3, N, seed=N)
    out, lse, (dq, dk, dv) = run_fwd_bwd(*(dev_bf16(b) for b in bits), causal=causal)
    w_out, w_lse = oracle.attn_fwd(q, k, v, causal=causal)
    check_bf16(out, w_out, "out")
    check_lse(lse, w_lse, "lse")
    # the gradient of 1/2 sum out^2 at the GPU's stored (bf16) output, which
    # the backward is given: dout = out, and Delta is evaluated on it
    w = oracle.attn_bwd(q, k, v, to_f64(out), causal=causal, out=to_f64(out))
    for name, g, ww in zip(("dq", "dk", "dv"), (dq, dk, dv), w):
        check_bf16(g, ww, name)
    check_end_to_end(q, k, v, run_grad(*(dev_bf16(b) for b in bits), causal=causal),
                     causal=causal)


def test_bf16_mixed_finite_and_nonfinite_heads():
    """Heads with a non-finite V and heads without, in one call: every head
    takes the tensor-core kernels (the launch counts), and every output,
    inf/NaN pattern included, matches the oracle."""
    bits, (q, k, v) = bf16_case(1, 4, 300, seed=42)
    vb = bits[2].copy()
    vb[0, 1, 200, 5] = 0x7F80   # +inf
    vb[0, 3, 17, 60] = 0xFF80   # -inf
    vb[0, 3, 250, 60] = 0x7F80  # +inf after -inf: NaN from row 250 on
    v = inputs.bf16_to_f64(vb)
    out, lse, (dq, dk, dv) = run_fwd_bwd(dev_bf16(bits[0]), dev_bf16(bits[1]), dev_bf16(vb))
    w_out, w_lse = oracle.attn_fwd(q, k, v)
    check_bf16(out, w_out, "out")
    check_lse(lse, w_lse, "lse")
    w = oracle.attn_bwd(q, k, v, to_f64(out), out=to_f64(out))
    for name, g, ww in zip(("dq", "dk", "dv"), (dq, dk, dv), w):
        check_bf16(g, ww, name)
    check_end_to_end(q, k, v, run_grad(dev_bf16(bits[0]), dev_bf16(bits[1]), dev_bf16(vb)))


# Non-finite values on the tensor-core path: classes placed on the diagonal
# (masked pairs of the diagonal tile meet them), at tile edges, in the
# ragged tail, and both infinities or a NaN in one column.
NONFINITE_V = [
    [(0, 0, 0x7F80)],                                  # key 0: every row sees it
    [(5, 3, 0x7F80), (130, 3, 0xFF80)],                # +inf, later -inf: NaN from 130
    [(127, 10, 0xFF80), (128, 11, 0x7FC0)],            # tile edge; a NaN
    [(200, 63, 0x7F80), (200, 62, 0xFF80), (299, 1, 0x7F80)],  # last row
]


@pytest.mark.parametrize("case", range(len(NONFINITE_V)))
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_nonfinite_v_tensor_core(case, causal):
    bits, (q, k, v) = bf16_case(1, 2, 300, seed=100 + case)
    vb = bits[2].copy()
    for row, col, pat in NONFINITE_V[case]:
        vb[0, 1, row, col] = pat
    v = inputs.bf16_to_f64(vb)
    out, lse, (dq, dk, dv) = run_fwd_bwd(dev_bf16(bits[0]), dev_bf16(bits[1]), dev_bf16(vb),
                                         causal=causal)
    w_out, w_lse = oracle.attn_fwd(q, k, v, causal=causal)
    check_bf16(out, w_out, "out")
    check_lse(lse, w_lse, "lse")
    w = oracle.attn_bwd(q, k, v, to_f64(out), causal=causal, out=to_f64(out))
    for name, g, ww in zip(("dq", "dk", "dv"), (dq, dk, dv), w):
        check_bf16(g, ww, name)
    check_end_to_end(q, k, v,
                     run_grad(dev_bf16(bits[0]), dev_bf16(bits[1]), dev_bf16(vb), causal=causal),
                     causal=causal)


@pytest.mark.parametrize("causal", [True, False])
def test_bf16_nonfinite_dout_general(causal):
    """A dout that is not out, holding +inf, -inf and NaN in rows of the
    diagonal block (masked pairs there meet them in dV += P^T dO): the
    backward matches the oracle's, classes included."""
    bits, (q, k, v) = bf16_case(1, 2, 300, seed=7)
    rng = np.random.default_rng(8)
    db = inputs.bf16_bits(rng.standard_normal((1, 2, 300, 64), dtype=np.float32))
    for row, col, pat in [(3, 0, 0x7F80), (100, 7, 0xFF80), (130, 7, 0x7F80), (140, 9, 0x7FC0),
                          (255, 2, 0xFF80), (299, 63, 0x7F80)]:
        db[0, 0, row, col] = pat
    dout = inputs.bf16_to_f64(db)
    tq, tk, tv = (dev_bf16(b) for b in bits)
    out, lse = swa.attn_fwd(tq, tk, tv, causal=causal)
    dq, dk, dv = swa.attn_bwd(tq, tk, tv, out, dev_bf16(db), lse, causal=causal)
    assert swa.last_launch_count() == BF16_BWD_LAUNCHES
    torch.cuda.synchronize()
    assert swa.get_device_error() == swa.SWA_OK
    w = oracle.attn_bwd(q, k, v, dout, causal=causal, out=to_f64(out))
    for name, g, ww in zip(("dq", "dk", "dv"), (dq, dk, dv), w):
        check_bf16(g, ww, name)


def test_bf16_wide_range_v_takes_bf16_operands():
    """V scaled by 2^16 in one head: beyond f16, so that head's products run
    with bf16 operands (the other head stays on f16); both match the oracle
    (forward; backward at the stored output).  The RMS floor is taken in the
    outputs' units (x 2^16 for out and dv, x 2^32 for dq and dk): dq of row 0
    is exactly 0, and float32 evaluates it as the difference of two dot
    products of size ~2^32.  The end-to-end gradient is compared on the f16
    head only: a bf16-operand head's backward receives out at bf16 as dout,
    and the few-key rows' dq then carries that rounding amplified."""
    bits, (q, k, v) = bf16_case(1, 2, 400, seed=9)
    vb = bits[2].copy()
    sc = 2.0 ** 16
    vb[0, 0] = inputs.bf16_bits(inputs.bf16_to_f32(vb[0, 0]) * np.float32(sc))
    v = inputs.bf16_to_f64(vb)
    out, lse, (dq, dk, dv) = run_fwd_bwd(dev_bf16(bits[0]), dev_bf16(bits[1]), dev_bf16(vb))
    w_out, w_lse = oracle.attn_fwd(q, k, v)
    check_bf16(out, w_out, "out", floor=RMS_FLOOR * sc)
    check_lse(lse, w_lse, "lse")
    w = oracle.attn_bwd(q, k, v, to_f64(out), out=to_f64(out))
    for name, g, ww, f in zip(("dq", "dk", "dv"), (dq, dk, dv), w, (2, 2, 1)):
        check_bf16(g, ww, name, floor=RMS_FLOOR * sc ** f)
    res = run_grad(dev_bf16(bits[0]), dev_bf16(bits[1]), dev_bf16(vb))
    w_out, w_lse = oracle.attn_fwd(q, k, v)
    check_bf16(res[0], w_out, "out (gradient call)", floor=RMS_FLOOR * sc)
    check_lse(res[1], w_lse, "lse (gradient call)")
    sl = (slice(0, 1), slice(1, 2))  # the f16 head
    check_end_to_end(q[sl], k[sl], v[sl], tuple(t[sl] for t in res), what=" (f16 head)")


# ------------------------------------------------------ large bf16 workloads

def sample_rows(rng, BH, N, n):
    heads = rng.integers(0, BH, size=n)
    rows = rng.integers(0, N, size=n)
    fixed_rows = np.array([0, 1, 127, 128, 129, N - 1], dtype=np.int64)
    heads = np.concatenate([heads, rng.integers(0, BH, size=fixed_rows.size)])
    rows = np.concatenate([rows, fixed_rows])
    return heads, rows


def check_forward_sampled(out, lse, q, k, v, heads, rows, causal=True):
    N = q.shape[2]
    w_out, w_lse = oracle.attn_fwd_rows(q, k, v, heads, rows, causal=causal)
    g_out = to_f64(out).reshape(-1, N, 64)[heads, rows]
    g_lse = to_f64(lse).reshape(-1, N)[heads, rows]
    check_bf16(g_out, w_out, "out (sampled rows)")
    check_lse(g_lse, w_lse, "lse (sampled rows)")


def check_forward_properties(out, lse, qb, kb, vb):
    """Row 0 sees key 0 alone: out_0 = v_0 exactly; lse_i >= s_ii."""
    o0 = out[:, :, 0].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(o0, vb[:, :, 0])
    q = torch.from_numpy(inputs.bf16_to_f32(qb)).cuda()
    k = torch.from_numpy(inputs.bf16_to_f32(kb)).cuda()
    sii = (q * k).sum(-1) / 8.0
    assert bool((lse >= sii - 1e-3 * sii.abs().clamp(min=1)).all())


def test_bf16_forward_b4_h16_n4096_every_element():
    wl = inputs.WORKLOADS["attn_fwd_b4h16n4096"]
    qb, kb, vb, _ = inputs.attn_bf16(**wl)
    out, lse, _ = run_fwd_bwd(dev_bf16(qb), dev_bf16(kb), dev_bf16(vb), backward=False)
    assert bool(torch.isfinite(out).all()) and bool(torch.isfinite(lse).all())
    check_forward_properties(out, lse, qb, kb, vb)
    q, k, v = (inputs.bf16_to_f64(b) for b in (qb, kb, vb))
    w_out, w_lse = oracle.attn_fwd(q, k, v)
    check_bf16(out, w_out, "out (every element)")
    check_lse(lse, w_lse, "lse (every element)")


def _backward_sampled(qb, kb, vb, out, lse, dq, dk, dv, n_q, n_k, tail, seed):
    B, H, N, _ = qb.shape
    q, k, v = (inputs.bf16_to_f64(b) for b in (qb, kb, vb))
    o = to_f64(out)
    rng = np.random.default_rng(seed)
    qh, qr = sample_rows(rng, B * H, N, n_q)
    kh = rng.integers(0, B * H, size=n_k)
    kr = N - 1 - rng.integers(0, tail, size=n_k)
    w_dq, w_dk, w_dv = oracle.attn_bwd_rows(q, k, v, o, qh, qr, kh, kr, out=o)
    check_bf16(to_f64(dq).reshape(-1, N, 64)[qh, qr], w_dq, "dq (sampled rows)")
    check_bf16(to_f64(dk).reshape(-1, N, 64)[kh, kr], w_dk, "dk (sampled rows)")
    check_bf16(to_f64(dv).reshape(-1, N, 64)[kh, kr], w_dv, "dv (sampled rows)")


def test_bf16_forward_backward_b2_h16_n16384():
    """The benchmark's batch (two sequences drawn per sequence, seed 4)."""
    wl = inputs.WORKLOADS["attn_fwdbwd_b2h16n16384"]
    qb, kb, vb = inputs.attn_bf16_batch(**wl)
    out, lse, (dq, dk, dv) = run_fwd_bwd(dev_bf16(qb), dev_bf16(kb), dev_bf16(vb))
    for t in (out, lse, dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    check_forward_properties(out, lse, qb, kb, vb)
    q, k, v = (inputs.bf16_to_f64(b) for b in (qb, kb, vb))
    heads, rows = sample_rows(np.random.default_rng(1), 32, wl["N"], 48)
    check_forward_sampled(out, lse, q, k, v, heads, rows)
    _backward_sampled(qb, kb, vb, out, lse, dq, dk, dv, n_q=24, n_k=6, tail=256, seed=2)
    # the heaviest keys too: key 0 and key 129 each collect dk, dv from ~16384 queries
    o = to_f64(out)
    N = wl["N"]
    kh, kr = np.array([7, 7], dtype=np.int64), np.array([0, 129], dtype=np.int64)
    _, w_dk, w_dv = oracle.attn_bwd_rows(q, k, v, o, np.zeros(0, np.int64),
                                         np.zeros(0, np.int64), kh, kr, out=o)
    check_bf16(to_f64(dk).reshape(-1, N, 64)[kh, kr], w_dk, "dk (first keys)")
    check_bf16(to_f64(dv).reshape(-1, N, 64)[kh, kr], w_dv, "dv (first keys)")
    # the gradient call at full size; whole heads: every row of out, lse and
    # of the end-to-end dq, dk, dv
    res = run_grad(dev_bf16(qb), dev_bf16(kb), dev_bf16(vb))
    for t in res:
        assert bool(torch.isfinite(t).all())
    for h in (0, 21):
        b_, h_ = divmod(h, wl["H"])
        sl = (slice(b_, b_ + 1), slice(h_, h_ + 1))
        check_end_to_end(q[sl], k[sl], v[sl], tuple(t[sl] for t in res), what=f" (head {h})")


@pytest.mark.parametrize("with_inf", [False, True])
def test_bf16_long_context_b1_h8_n65536(with_inf):
    wl = inputs.WORKLOADS["attn_fwdbwd_b1h8n65536"]
    n_inf = inputs.LONG_CONTEXT_N_INF if with_inf else 0
    qb, kb, vb, pos = inputs.attn_bf16(**wl, n_inf=n_inf)
    assert pos.size == n_inf
    out, lse, (dq, dk, dv) = run_fwd_bwd(dev_bf16(qb), dev_bf16(kb), dev_bf16(vb))
    N = wl["N"]
    # Full-size property: out[h, i, d] = +inf exactly when some V[h, j, d] = +inf
    # with j <= i; every other entry (and lse) is finite.
    o = to_f64(out)[0]
    first = np.full((wl["H"], 64), N, dtype=np.int64)
    if n_inf:
        _, h_, j_, d_ = np.unravel_index(pos, (1, wl["H"], N, 64))
        np.minimum.at(first, (h_, d_), j_)
    want_inf = np.arange(N)[None, :, None] >= first[:, None, :]
    assert np.array_equal(np.isposinf(o), want_inf)
    assert np.isfinite(o[~want_inf]).all()
    assert bool(torch.isfinite(lse).all())
    q, k, v = (inputs.bf16_to_f64(b) for b in (qb, kb, vb))
    heads, rows = sample_rows(np.random.default_rng(3), wl["H"], N, 24)
    check_forward_sampled(out, lse, q, k, v, heads, rows)
    _backward_sampled(qb, kb, vb, out, lse, dq, dk, dv, n_q=12, n_k=3, tail=64, seed=4)
    # the gradient call at full size; one whole head: every row of out, lse
    # and the end-to-end gradient (with the injection: its inf/NaN pattern
    # exactly, the rest in tolerance)
    del out, lse, dq, dk, dv
    res = run_grad(dev_bf16(qb), dev_bf16(kb), dev_bf16(vb))
    h = 6 if with_inf else 3
    sl = (slice(0, 1), slice(h, h + 1))
    check_end_to_end(q[sl], k[sl], v[sl], tuple(t[sl] for t in res), what=f" (head {h})")


# --------------------------------------------------- non-causal (causal = 0)

def test_bf16_noncausal_b1_h4_n2048_every_element():
    """Every pair exists (the ABI's causal = 0): all tiles, none skipped or
    masked except past N; compared element by element with the oracle."""
    bits, (q, k, v) = bf16_case(1, 4, 2048, seed=11)
    out, lse, (dq, dk, dv) = run_fwd_bwd(*(dev_bf16(b) for b in bits), causal=False)
    w_out, w_lse = oracle.attn_fwd(q, k, v, causal=False)
    check_bf16(out, w_out, "out")
    check_lse(lse, w_lse, "lse")
    w = oracle.attn_bwd(q, k, v, to_f64(out), causal=False, out=to_f64(out))
    for name, g, ww in zip(("dq", "dk", "dv"), (dq, dk, dv), w):
        check_bf16(g, ww, name)


def test_bf16_noncausal_b2_h16_n16384_sampled():
    """The non-causal call at the benchmark's size and launch configuration,
    checked at sampled rows (keys anywhere: each sees all 16384 queries)."""
    wl = inputs.WORKLOADS["attn_fwdbwd_b2h16n16384"]
    qb, kb, vb = inputs.attn_bf16_batch(**wl)
    out, lse, (dq, dk, dv) = run_fwd_bwd(dev_bf16(qb), dev_bf16(kb), dev_bf16(vb), causal=False)
    for t in (out, lse, dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    q, k, v = (inputs.bf16_to_f64(b) for b in (qb, kb, vb))
    N = wl["N"]
    rng = np.random.default_rng(12)
    heads, rows = sample_rows(rng, 32, N, 16)
    check_forward_sampled(out, lse, q, k, v, heads, rows, causal=False)
    o = to_f64(out)
    qh, qr = sample_rows(rng, 32, N, 8)
    kh = np.array([5, 5], dtype=np.int64)
    kr = np.array([0, N // 2 + 17], dtype=np.int64)
    w_dq, w_dk, w_dv = oracle.attn_bwd_rows(q, k, v, o, qh, qr, kh, kr, causal=False, out=o)
    check_bf16(to_f64(dq).reshape(-1, N, 64)[qh, qr], w_dq, "dq (sampled rows)")
    check_bf16(to_f64(dk).reshape(-1, N, 64)[kh, kr], w_dk, "dk (sampled rows)")
    check_bf16(to_f64(dv).reshape(-1, N, 64)[kh, kr], w_dv, "dv (sampled rows)")
