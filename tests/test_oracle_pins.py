"""Pins for the float64 oracle, each tied to something other than the oracle
itself: central finite differences, closed forms, invariants, the pages'
printed worked examples and mask test, and library special cases (torch's
float64 CPU attention with autograd, the pages' own numpy regrid check).

Sources: "Show HN: Automatic deduction of FlashAttention kernel from ~25
lines of SQL" (page 2: views ATTENTION_WINDOW / ATTENTION_GROUP_BY, queries
GRADIENT and NADARAYA_WATSON, functions attention(), main(),
check_masks_are_absent_rows, check_nadaraya_watson) and "Wiki notes"
(page 5: mini_attention, the Python softmax and its worked example).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from causal_attention_swa_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng_qkv(seed, B, H, N, D, std=1.0):
    rng = np.random.default_rng(seed)
    return tuple(std * rng.normal(size=(B, H, N, D)) for _ in range(3))


# ---------------------------------------------------------------- backward

def _loss_and_grad_fd(q, k, v, causal, scale, dout_fixed, eps=1e-5):
    """Central differences of L = sum(dout_fixed * out) (or 1/2 sum out^2 when
    dout_fixed is None) with respect to every entry of q, k, v."""
    def loss(q_, k_, v_):
        out, _ = oracle.attn_fwd(q_, k_, v_, causal=causal, scale=scale)
        if dout_fixed is None:
            return 0.5 * float(np.sum(out * out))
        return float(np.sum(dout_fixed * out))

    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        x = args[which]
        g = np.zeros_like(x)
        flat = x.reshape(-1)
        gflat = g.reshape(-1)
        for idx in range(flat.size):
            old = flat[idx]
            flat[idx] = old + eps
            lp = loss(*args)
            flat[idx] = old - eps
            lm = loss(*args)
            flat[idx] = old
            gflat[idx] = (lp - lm) / (2 * eps)
        grads.append(g)
    return grads


@pytest.mark.parametrize("N,D", [(1, 4), (2, 4), (4, 4), (16, 4), (1, 64), (4, 64), (16, 64)])
@pytest.mark.parametrize("causal", [True, False])
def test_backward_matches_central_differences(N, D, causal):
    """dq, dk, dv of 1/2 sum out^2 (query GRADIENT, dout = out) against central
    differences of the forward: relative error <= 1e-6."""
    q, k, v = _rng_qkv(100 + N + D, 1, 1, N, D)
    scale = 1.0 / math.sqrt(D)
    out, _ = oracle.attn_fwd(q, k, v, causal=causal, scale=scale)
    got = oracle.attn_bwd(q, k, v, out, causal=causal, scale=scale)
    want = _loss_and_grad_fd(q, k, v, causal, scale, None)
    for name, g, w in zip("qkv", got, want):
        denom = max(np.abs(w).max(), 1e-300)
        rel = np.abs(g - w).max() / denom
        assert rel <= 1e-6, (name, rel)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_general_dout_matches_central_differences(causal):
    """The backward for an arbitrary upstream gradient (L = sum dout*out)."""
    N, D = 8, 4
    q, k, v = _rng_qkv(7, 1, 2, N, D)
    dout = np.random.default_rng(8).normal(size=q.shape)
    got = oracle.attn_bwd(q, k, v, dout, causal=causal, scale=0.5)
    want = _loss_and_grad_fd(q, k, v, causal, 0.5, dout)
    for name, g, w in zip("qkv", got, want):
        rel = np.abs(g - w).max() / np.abs(w).max()
        assert rel <= 1e-6, (name, rel)


# ---------------------------------------------------------- closed forms

def test_row0_sees_only_key0_exactly():
    """Causal predicate q.t >= k.t includes the diagonal: row 0 sees key 0
    alone, so w = exp(0) = 1, z = 1 and out_0 = v_0 exactly; lse_0 = s_00."""
    q, k, v = _rng_qkv(1, 2, 3, 37, 64)
    out, lse = oracle.attn_fwd(q, k, v, causal=True)
    assert np.array_equal(out[:, :, 0], v[:, :, 0])
    s00 = np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]) / 8.0
    assert np.allclose(lse[:, :, 0], s00, rtol=0, atol=1e-14)


def test_single_token_returns_v():
    q, k, v = _rng_qkv(2, 1, 1, 1, 64)
    for causal in (True, False):
        out, lse = oracle.attn_fwd(q, k, v, causal=causal)
        assert np.array_equal(out, v)
        assert abs(lse[0, 0, 0] - float(q[0, 0, 0] @ k[0, 0, 0]) / 8.0) < 1e-14


def test_equal_keys_give_prefix_mean_and_log_count():
    """All keys equal => every score of row i is the same => uniform weights:
    out_i = mean(v_0..v_i) and lse_i = s_i + ln(i+1) (causal);
    out_i = mean(v) and lse_i = s_i + ln N (non-causal)."""
    N, D = 50, 64
    rng = np.random.default_rng(3)
    q = rng.normal(size=(1, 1, N, D))
    krow = rng.normal(size=D)
    k = np.broadcast_to(krow, (1, 1, N, D)).copy()
    v = rng.normal(size=(1, 1, N, D))
    s = (q[0, 0] @ krow) / 8.0
    out, lse = oracle.attn_fwd(q, k, v, causal=True)
    prefix_mean = np.cumsum(v[0, 0], axis=0) / np.arange(1, N + 1)[:, None]
    assert np.abs(out[0, 0] - prefix_mean).max() < 1e-13
    assert np.abs(lse[0, 0] - (s + np.log(np.arange(1, N + 1)))).max() < 1e-13
    out, lse = oracle.attn_fwd(q, k, v, causal=False)
    assert np.abs(out[0, 0] - v[0, 0].mean(axis=0)).max() < 1e-13
    assert np.abs(lse[0, 0] - (s + np.log(N))).max() < 1e-13


def test_weights_sum_to_one_and_masked_weights_are_zero():
    """With V = identity (N <= D) out_i is the weight row P_i: each row sums
    to 1, is positive on the existing pairs j <= i and zero elsewhere."""
    N, D = 40, 64
    q, k, _ = _rng_qkv(4, 1, 1, N, D)
    v = np.zeros((1, 1, N, D))
    v[0, 0, np.arange(N), np.arange(N)] = 1.0
    out, _ = oracle.attn_fwd(q, k, v, causal=True)
    P = out[0, 0, :, :N]
    assert np.abs(P.sum(axis=1) - 1.0).max() < 1e-14
    assert np.all(P[np.tril_indices(N)] > 0)
    assert np.all(P[np.triu_indices(N, 1)] == 0)
    assert np.all(out[0, 0, :, N:] == 0)


def test_softmax_worked_example_printed_values():
    """Page 5's worked example: logits [3, 1, -2] -> exp(val - max) =
    1.0, 0.1353..., 0.0067... (printed to four decimals)."""
    g = json.load(open(os.path.join(GOLDEN, "softmax_worked_example.json")))
    logits = g["logits"]
    n = len(logits)
    # One query against n keys with D = 3, scale 1: score_j = logits[j].
    q = np.zeros((1, 1, n, 3))
    q[0, 0, 0, 0] = 1.0
    k = np.zeros((1, 1, n, 3))
    k[0, 0, :, 0] = logits
    v = np.eye(n, 3).reshape(1, 1, n, 3)
    out, lse = oracle.attn_fwd(q, k, v, causal=False, scale=1.0)
    p = out[0, 0, 0]
    z = math.exp(lse[0, 0, 0] - g["max_val"])
    w = p * z
    for got, printed in zip(w, g["exp_shifted_printed"]):
        lo = float(printed)
        assert lo <= got < lo + 1e-4, (got, printed)
    # and the closed form exp(-2), exp(-5)
    assert np.allclose(w, np.exp(np.array(g["shifted"])), rtol=1e-14, atol=0)
    assert abs(p.sum() - 1) < 1e-15


def test_mini_attention_structure_brute_force():
    """Page 5's mini_attention: seq 4, d_model 8, d_k = d_v = 4, Q = xWq,
    K = xWk, V = xWv, softmax over keys (axis 1), no scale, no mask.  The
    oracle (non-causal, scale 1) equals a hand-unrolled 4x4 evaluation that
    exponentiates without subtracting the max (the pages print no numbers,
    so this pins structure only)."""
    rng = np.random.default_rng(5)
    x = rng.normal(size=(4, 8))
    wq, wk, wv = (rng.normal(size=(8, 4)) * 0.3 for _ in range(3))
    Q, K, V = x @ wq, x @ wk, x @ wv
    out, _ = oracle.attn_fwd(Q[None, None], K[None, None], V[None, None],
                             causal=False, scale=1.0)
    want = np.zeros((4, 4))
    for i in range(4):
        e = [math.exp(sum(Q[i, c] * K[j, c] for c in range(4))) for j in range(4)]
        tot = e[0] + e[1] + e[2] + e[3]
        for d in range(4):
            want[i, d] = sum(e[j] / tot * V[j, d] for j in range(4))
    assert np.abs(out[0, 0] - want).max() < 1e-13


# ------------------------------------------------------------ invariants

def test_shifting_every_key_by_one_vector_moves_only_lse():
    """Adding u to every key adds scale*q_i.u to every score of row i: the
    row max cancels it out of w/z, so out, dq, dv and dk are unchanged, and
    lse moves by scale*q_i.u.  With |shift| > 710 this fails without the max
    subtraction (exp overflows)."""
    N, D = 24, 64
    q, k, v = _rng_qkv(6, 1, 2, N, D)
    u = np.full(D, 400.0)
    k2 = k + u
    out, lse = oracle.attn_fwd(q, k, v)
    out2, lse2 = oracle.attn_fwd(q, k2, v)
    shift = (q @ u) / 8.0
    assert np.abs(shift).max() > 710  # exp would overflow float64
    assert np.abs(out - out2).max() < 1e-11
    assert np.abs((lse2 - lse) - shift).max() < 1e-9
    g = oracle.attn_bwd(q, k, v, out)
    g2 = oracle.attn_bwd(q, k2, v, out2)
    for a, b in zip(g, g2):
        assert np.abs(a - b).max() < 1e-9 * max(1.0, np.abs(a).max())


def test_gradient_through_row_max_sums_to_zero():
    """The loss is invariant to a common shift of every key, so
    sum_j dK_j = scale * sum_i (sum_j dS_ij) q_i = 0 (the view's comment: the
    max subtraction's gradient sums to zero)."""
    for causal in (True, False):
        q, k, v = _rng_qkv(9, 2, 2, 33, 64)
        out, _ = oracle.attn_fwd(q, k, v, causal=causal)
        _, dk, _ = oracle.attn_bwd(q, k, v, out, causal=causal)
        tot = dk.sum(axis=2)
        assert np.abs(tot).max() < 1e-12 * np.abs(dk).max() * 33


# --------------------------------------------------- absent-row semantics

def test_pages_mask_test_pattern():
    """check_masks_are_absent_rows: +inf at V[9, 0], n = 16, seed 1."""
    g = json.load(open(os.path.join(GOLDEN, "mask_absent_rows.json")))
    q, k, v = inputs.pages_mask(g["n"], g["inf_row"])
    assert np.isposinf(v[0, 0, g["inf_row"], g["inf_col"]])
    out, _ = oracle.attn_fwd(q, k, v, causal=True)
    o = out[0, 0]
    j = g["inf_row"]
    assert np.isfinite(o[:j]).all()
    assert np.isposinf(o[j:, 0]).all()
    assert np.isfinite(o[:, 1:]).all()


def test_single_head_inf_pattern_and_backward_classes():
    """+inf at V[100, 3] of the 256-token draw: only queries i >= 100 see it,
    in column 3 only.  In the backward (dout = out) dV[j, 3] is +inf for
    every j <= 255 because every row i >= 100 carries +inf in dO[:, 3]."""
    q, k, v = inputs.single_head_f64(256, inf_at=(100, 3))
    out, lse = oracle.attn_fwd(q, k, v)
    o = out[0, 0]
    assert np.isfinite(o[:100]).all()
    assert np.isposinf(o[100:, 3]).all()
    assert np.isfinite(np.delete(o, 3, axis=1)).all()
    assert np.isfinite(lse).all()
    dq, dk, dv = oracle.attn_bwd(q, k, v, out)
    assert np.isposinf(dv[0, 0, :, 3]).all()
    # rows i < 100 see only finite values and have finite Delta: finite dq
    assert np.isfinite(dq[0, 0, :100]).all()
    # rows i >= 100 have Delta = +inf: dS = P (dP - inf) = -inf or NaN
    assert not np.isfinite(dq[0, 0, 100:]).any()


def test_noncausal_inf_reaches_every_row():
    q, k, v = inputs.pages_mask(16, 9)
    out, _ = oracle.attn_fwd(q, k, v, causal=False)
    assert np.isposinf(out[0, 0, :, 0]).all()
    assert np.isfinite(out[0, 0, :, 1:]).all()


def test_inf_and_neg_inf_in_one_column_give_nan_after_both():
    q, k, v = _rng_qkv(11, 1, 1, 20, 64)
    v[0, 0, 5, 7] = np.inf
    v[0, 0, 12, 7] = -np.inf
    out, _ = oracle.attn_fwd(q, k, v)
    c = out[0, 0, :, 7]
    assert np.isfinite(c[:5]).all()
    assert np.isposinf(c[5:12]).all()
    assert np.isnan(c[12:]).all()


# ------------------------------------------------------ library special case

@pytest.mark.parametrize("n", [64, 256])
def test_matches_torch_float64_sdpa_and_autograd(n):
    """The demo's own inputs (main(): seed 0, sizes 64 and 256) against torch's
    float64 CPU scaled_dot_product_attention with is_causal and autograd of
    1/2 sum out^2, standing in for the demo's JAX attention() and jax.grad."""
    q, k, v = inputs.pages_main()[n]
    tq, tk, tv = (torch.tensor(a[None, None], dtype=torch.float64, requires_grad=True)
                  for a in (q, k, v))
    tout = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    (0.5 * (tout * tout).sum()).backward()
    out, _ = oracle.attn_fwd(q[None, None], k[None, None], v[None, None])
    assert np.abs(out - tout.detach().numpy()).max() < 1e-12
    dq, dk, dv = oracle.attn_bwd(q[None, None], k[None, None], v[None, None], out)
    for g, t in zip((dq, dk, dv), (tq, tk, tv)):
        assert np.abs(g - t.grad.numpy()).max() < 1e-11


def test_sampled_rows_match_full_evaluation():
    """The sampled entry points return the same numbers as the full ones."""
    q, k, v = _rng_qkv(12, 2, 3, 40, 64)
    for causal in (True, False):
        out, lse = oracle.attn_fwd(q, k, v, causal=causal)
        dq, dk, dv = oracle.attn_bwd(q, k, v, out, causal=causal)
        heads = np.array([0, 5, 3, 2])
        rows = np.array([0, 39, 17, 1])
        o_s, l_s = oracle.attn_fwd_rows(q, k, v, heads, rows, causal=causal)
        flat_out, flat_lse = out.reshape(6, 40, 64), lse.reshape(6, 40)
        assert np.array_equal(o_s, flat_out[heads, rows])
        assert np.array_equal(l_s, flat_lse[heads, rows])
        dq_s, dk_s, dv_s = oracle.attn_bwd_rows(q, k, v, out, heads, rows, heads, rows,
                                                causal=causal)
        assert np.abs(dq_s - dq.reshape(6, 40, 64)[heads, rows]).max() < 1e-14
        assert np.abs(dk_s - dk.reshape(6, 40, 64)[heads, rows]).max() < 1e-14
        assert np.abs(dv_s - dv.reshape(6, 40, 64)[heads, rows]).max() < 1e-14


# ------------------------------------------------------------ regrid

def test_nw_pages_numpy_check():
    """check_nadaraya_watson: 64 targets, 256 sources in [0,1]^2, the demo's
    numpy reference (w @ y) / w.sum(1) with w = exp(-dist2 / 0.25)."""
    t, s, y = inputs.pages_nw()
    dist2 = ((t[:, None, :] - s[None, :, :]) ** 2).sum(-1)
    w = np.exp(-dist2 / 0.25)
    want = (w @ y) / w.sum(axis=1)
    got = oracle.nw_regrid(t, s, y, h=0.5)
    assert np.abs(got - want).max() < 1e-13


def test_nw_closed_forms():
    """Bandwidth h = 0.5 means the divisor 0.25 = h^2: a source at distance
    0.5 weighs exp(-1) against 1 for a coincident one (exp(-1/2) would mean
    the textbook 2h^2 reading)."""
    s = np.array([[1.0, 1.0], [1.5, 1.0]])
    vals = np.array([2.0, -3.0])
    t = np.array([[1.0, 1.0], [1.25, 1.0], [1.0, 1.5]])
    got = oracle.nw_regrid(t, s, vals, h=0.5)
    e = math.exp(-1.0)
    assert abs(got[0] - (2.0 + e * -3.0) / (1 + e)) < 1e-15
    assert abs(got[1] - (-0.5)) < 1e-15          # midpoint: equal weights
    e2 = math.exp(-(0.25 + 0.25) / 0.25)          # distance^2 = 0.5 to s[1]
    assert abs(got[2] - (e * 2.0 + e2 * -3.0) / (e + e2)) < 1e-15
    # one source: out = v; constant values: out = the constant
    rng = np.random.default_rng(0)
    tt = rng.uniform(0, 2, size=(30, 2))
    assert np.all(oracle.nw_regrid(tt, s[:1], vals[:1]) == 2.0)
    ss = rng.uniform(0, 2, size=(50, 2))
    c = oracle.nw_regrid(tt, ss, np.full(50, 0.7))
    assert np.abs(c - 0.7).max() < 1e-15
    # co-located sources: the mean of their values
    m = oracle.nw_regrid(tt, np.full((5, 2), 0.3), np.arange(5.0))
    assert np.abs(m - 2.0).max() < 1e-14


def test_nw_all_weights_underflow_is_nan():
    """A target so far from every source that each weight underflows: 0/0."""
    got = oracle.nw_regrid(np.array([[100.0, 100.0]]), np.array([[0.0, 0.0]]),
                           np.array([1.0]))
    assert np.isnan(got[0])


def test_delta_on_a_given_output_moves_gradients_by_the_closed_form():
    """Delta_i = dout_i . out_i evaluated on a given (stored) output: a change
    E of that output shifts Delta by delta_i = dout_i . E_i, which moves
    dq_i by -scale delta_i (P K)_i and dk_j by -scale sum_i P_ij delta_i q_i,
    and leaves dv unchanged.  P comes from the forward with V = identity."""
    N, D = 48, 64
    q, k, v = _rng_qkv(13, 1, 1, N, D)
    for causal in (True, False):
        out, _ = oracle.attn_fwd(q, k, v, causal=causal)
        eye = np.zeros((1, 1, N, D))
        eye[0, 0, np.arange(N), np.arange(N)] = 1.0
        P = oracle.attn_fwd(q, k, eye, causal=causal)[0][0, 0, :, :N]
        E = np.random.default_rng(14).normal(size=out.shape) * 1e-2
        dq0, dk0, dv0 = oracle.attn_bwd(q, k, v, out, causal=causal)
        dq1, dk1, dv1 = oracle.attn_bwd(q, k, v, out, causal=causal, out=out + E)
        dq2, dk2, dv2 = oracle.attn_bwd(q, k, v, out, causal=causal, out=out)
        assert np.array_equal(dq0, dq2) and np.array_equal(dk0, dk2) and np.array_equal(dv0, dv2)
        delta = (out[0, 0] * E[0, 0]).sum(axis=1)
        assert np.array_equal(dv0, dv1)
        want_dq = -(delta[:, None] * (P @ k[0, 0])) / 8.0
        want_dk = -(P.T @ (delta[:, None] * q[0, 0])) / 8.0
        assert np.abs((dq1 - dq0)[0, 0] - want_dq).max() < 1e-12
        assert np.abs((dk1 - dk0)[0, 0] - want_dk).max() < 1e-12


# ------------------------------------------------- regrid in 1-3 dimensions

def _nw_points(seed, M, S, dims, lo=0.0, hi=1.5):
    rng = np.random.default_rng(seed)
    return (rng.uniform(lo, hi, size=(M, dims)), rng.uniform(lo, hi, size=(S, dims)),
            rng.normal(size=S), rng.normal(size=M))


def test_nw_nd_two_dims_is_the_pages_regrid():
    """In two dimensions the generalised regrid is the NADARAYA_WATSON view
    itself (the demo's numpy check's inputs)."""
    t, s, y = inputs.pages_nw()
    assert np.abs(oracle.nw_regrid_nd(t, s, y, h=0.5) - oracle.nw_regrid(t, s, y, h=0.5)).max() \
        < 1e-15


def test_nw_nd_zero_coordinates_reduce_the_dimension():
    """A coordinate that is 0 for every point adds 0 to every squared
    distance: 3-D with z = 0 gives the 2-D result, 2-D with y = 0 the 1-D."""
    t, s, y, _ = _nw_points(21, 9, 13, 2)
    pad = lambda a: np.concatenate([a, np.zeros((a.shape[0], 1))], axis=1)  # noqa: E731
    assert np.abs(oracle.nw_regrid_nd(pad(t), pad(s), y) - oracle.nw_regrid_nd(t, s, y)).max() \
        < 1e-15
    assert np.abs(oracle.nw_regrid_nd(pad(t[:, :1]), pad(s[:, :1]), y)
                  - oracle.nw_regrid_nd(t[:, :1], s[:, :1], y)).max() < 1e-15


def test_nw_nd_closed_forms():
    """3-D: a source at squared distance h^2 weighs exp(-1) against a
    coincident one; one source gives out = v everywhere."""
    s = np.array([[0.0, 0.0, 0.0], [0.3, 0.4, 0.0]])    # |s1 - s0| = 0.5 = h
    vals = np.array([1.0, 4.0])
    got = oracle.nw_regrid_nd(np.zeros((1, 3)), s, vals, h=0.5)
    e = math.exp(-1.0)
    assert abs(got[0] - (1.0 + 4.0 * e) / (1.0 + e)) < 1e-15
    t = np.random.default_rng(3).uniform(-1, 1, size=(7, 3))
    assert np.all(oracle.nw_regrid_nd(t, s[:1], vals[:1]) == 1.0)


@pytest.mark.parametrize("dims", [1, 2, 3])
def test_nw_backward_matches_central_differences(dims):
    """L = sum_p g_p out_p: dL/dtargets, dL/dsources and dL/dvals against
    central differences of the forward (relative error <= 1e-6)."""
    t, s, y, g = _nw_points(30 + dims, 5, 7, dims)
    h = 0.7
    dt, ds, dv = oracle.nw_regrid_bwd(t, s, y, g, h=h)

    def loss(t_, s_, y_):
        return float(np.dot(g, oracle.nw_regrid_nd(t_, s_, y_, h=h)))

    eps = 1e-6
    for arr, grad, which in ((t, dt, 0), (s, ds, 1), (y, dv, 2)):
        fd = np.zeros_like(arr)
        flat, fflat = arr.reshape(-1), fd.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            args = [t, s, y]
            flat[i] = old + eps
            lp = loss(*args)
            flat[i] = old - eps
            lm = loss(*args)
            flat[i] = old
            fflat[i] = (lp - lm) / (2 * eps)
        err = np.abs(grad - fd).max() / max(np.abs(fd).max(), 1e-12)
        assert err <= 1e-6, (which, err)


def test_nw_backward_invariants_and_closed_forms():
    """Shifting every point by one vector leaves out unchanged, so the
    position gradients sum to zero; sum_q dv_q = sum_p g_p (each row of P
    sums to 1); one source: out = v for every target, so the position
    gradients vanish and dv = sum_p g_p; constant values likewise."""
    t, s, y, g = _nw_points(40, 11, 17, 3)
    dt, ds, dv = oracle.nw_regrid_bwd(t, s, y, g, h=0.6)
    tot = dt.sum(axis=0) + ds.sum(axis=0)
    assert np.abs(tot).max() < 1e-12 * (np.abs(dt).max() + np.abs(ds).max())
    assert abs(dv.sum() - g.sum()) < 1e-12 * np.abs(g).sum()
    dt1, ds1, dv1 = oracle.nw_regrid_bwd(t, s[:1], y[:1], g, h=0.6)
    # out = (w v) / w is v up to one rounding, so v - out is 0 or one ulp of v
    assert np.abs(dt1).max() < 1e-14 and np.abs(ds1).max() < 1e-14
    assert abs(dv1[0] - g.sum()) < 1e-13
    dtc, dsc, _ = oracle.nw_regrid_bwd(t, s, np.full(17, 0.25), g, h=0.6)
    assert np.abs(dtc).max() < 1e-15 and np.abs(dsc).max() < 1e-15


# ------------------------------------------------------- QKV projection

def test_qkv_projection_brute_force():
    """q[b,h,n,d] = sum_c x[b,n,c] w[h D + d, c], k and v from the next row
    blocks: against a plain triple loop on a tiny case."""
    rng = np.random.default_rng(50)
    B, N, C, H, D = 2, 3, 5, 2, 3
    x = rng.normal(size=(B, N, C))
    w = rng.normal(size=(3 * H * D, C))
    q, k, v = oracle.qkv_proj(x, w, H, D)
    for which, t in enumerate((q, k, v)):
        for b in range(B):
            for h in range(H):
                for n in range(N):
                    for d in range(D):
                        want = sum(x[b, n, c] * w[which * H * D + h * D + d, c] for c in range(C))
                        assert abs(t[b, h, n, d] - want) < 1e-13


def test_qkv_projection_is_mini_attentions_x_times_w():
    """Page 5's mini_attention (seq 4, d_model 8, d_k = d_v = 4): with the
    rows of w taken from the columns of Wq, Wk, Wv (one head), the projection
    gives x Wq, x Wk, x Wv; selecting rows of the identity picks features."""
    rng = np.random.default_rng(5)
    x = rng.normal(size=(4, 8))
    wq, wk, wv = (rng.normal(size=(8, 4)) for _ in range(3))
    q, k, v = oracle.qkv_proj(x[None], np.concatenate([wq.T, wk.T, wv.T]), 1, 4)
    for got, wm in ((q, wq), (k, wk), (v, wv)):
        assert np.abs(got[0, 0] - x @ wm).max() < 1e-14
    eye = np.eye(8)[[0, 1, 2, 3, 4, 5, 6, 7, 0, 1, 2, 3]]   # q, k: features 0-3, 4-7; v: 0-3
    q, k, v = oracle.qkv_proj(x[None], eye, 1, 4)
    assert np.array_equal(q[0, 0], x[:, :4]) and np.array_equal(k[0, 0], x[:, 4:])
    assert np.array_equal(v[0, 0], x[:, :4])
