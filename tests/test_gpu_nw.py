"""GPU parity of the Nadaraya-Watson regrid (through the C ABI) against the
float64 oracle: the demo's own check_nadaraya_watson inputs ("Show HN:
Automatic deduction of FlashAttention kernel from ~25 lines of SQL",
64 targets x 256 sources in [0,1]^2), the 16384 x 16384 grid in [0,10]^2
(every target), ragged sizes, and the degenerate cases (one source,
constant values, all weights underflowing -> NaN).  Tolerance: float32
path, max abs error <= 1e-5 (tests/_compare.py)."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_swa_b200 import inputs, swa
from _compare import check_f32, check_f32_scaled

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def run(t, s, v, h=0.5):
    out = swa.nw_regrid(dev(t), dev(s), dev(v), h=h)
    torch.cuda.synchronize()
    return out


def test_nw_demo_inputs():
    t, s, y = inputs.pages_nw()
    t32, s32, y32 = (a.astype(np.float32) for a in (t, s, y))
    got = run(t32, s32, y32)
    check_f32(got, oracle.nw_regrid(t32, s32, y32, h=0.5), "nw demo")


def test_nw_grid_16384():
    t, s, v = inputs.nw_grid()
    got = run(t, s, v)
    want = oracle.nw_regrid(t, s, v, h=0.5)
    check_f32(got, want, "nw 16384x16384")


@pytest.mark.parametrize("M,S", [(1, 1), (1, 5000), (1023, 17), (1025, 2049), (3000, 4097),
                                 (70000, 300)])
def test_nw_ragged_sizes(M, S):
    rng = np.random.default_rng(M * 7 + S)
    t = rng.uniform(0, 3, size=(M, 2)).astype(np.float32)
    s = rng.uniform(0, 3, size=(S, 2)).astype(np.float32)
    v = rng.normal(size=S).astype(np.float32)
    check_f32(run(t, s, v), oracle.nw_regrid(t, s, v, h=0.5), f"nw {M}x{S}")


def test_nw_degenerate_cases():
    rng = np.random.default_rng(0)
    t = rng.uniform(0, 2, size=(100, 2)).astype(np.float32)
    one = np.array([[1.0, 1.0]], np.float32)
    got = run(t, one, np.array([2.5], np.float32)).cpu().numpy()
    assert np.abs(got - 2.5).max() <= 2.5 * 2.0 ** -22  # (w v) / w: two roundings
    s = rng.uniform(0, 2, size=(300, 2)).astype(np.float32)
    got = run(t, s, np.full(300, 0.7, np.float32)).cpu().numpy()
    assert np.abs(got - 0.7).max() < 1e-6
    far = run(np.array([[100.0, 100.0]], np.float32), one, np.array([1.0], np.float32))
    assert bool(torch.isnan(far).all())
    # another bandwidth: h = 0.25 -> divisor 0.0625
    s2 = rng.uniform(0, 2, size=(500, 2)).astype(np.float32)
    v2 = rng.normal(size=500).astype(np.float32)
    check_f32(run(t, s2, v2, h=0.25), oracle.nw_regrid(t, s2, v2, h=0.25), "nw h=0.25")


# ------------------------------------------ points of 1, 2 or 3 coordinates

def run_nd(t, s, v, h=0.5):
    out = swa.nw_regrid_nd(dev(t), dev(s), dev(v), h=h)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dims", [1, 2, 3])
@pytest.mark.parametrize("M,S", [(1, 1), (1023, 17), (3000, 4097)])
def test_nw_nd_ragged_sizes(dims, M, S):
    rng = np.random.default_rng(M * 11 + S + dims)
    t = rng.uniform(0, 3, size=(M, dims)).astype(np.float32)
    s = rng.uniform(0, 3, size=(S, dims)).astype(np.float32)
    v = rng.normal(size=S).astype(np.float32)
    check_f32(run_nd(t, s, v), oracle.nw_regrid_nd(t, s, v, h=0.5), f"nw {dims}-d {M}x{S}")


@pytest.mark.parametrize("dims", [1, 3])
def test_nw_nd_grid_16384(dims):
    t, s, v = inputs.nw_grid_nd(16384, 16384, dims)
    check_f32(run_nd(t, s, v), oracle.nw_regrid_nd(t, s, v, h=0.5), f"nw {dims}-d 16384x16384")


def test_nw_nd_two_dims_is_swa_nw_regrid():
    t, s, v = inputs.nw_grid(3000, 5000)
    a = run_nd(t, s, v)
    b = run(t, s, v)
    assert torch.equal(a, b)


# ---------------------------------------------------------- regrid gradient

def run_bwd(t, s, v, g, h=0.5):
    res = swa.nw_regrid_bwd(dev(t), dev(s), dev(v), dev(g), h=h)
    torch.cuda.synchronize()
    assert swa.get_device_error() == swa.SWA_OK
    return res


def check_bwd(t, s, v, g, h, what):
    dt, ds, dv = run_bwd(t, s, v, g, h)
    w_dt, w_ds, w_dv = oracle.nw_regrid_bwd(t, s, v, g, h=h)
    check_f32_scaled(dt, w_dt, f"dtargets {what}")
    check_f32_scaled(ds, w_ds, f"dsources {what}")
    check_f32_scaled(dv, w_dv, f"dvals {what}")


@pytest.mark.parametrize("dims", [1, 2, 3])
@pytest.mark.parametrize("M,S", [(1, 1), (5, 3000), (2500, 2), (1023, 2049), (3000, 4097)])
def test_nw_gradient_ragged_sizes(dims, M, S):
    rng = np.random.default_rng(M * 13 + S + dims)
    t = rng.uniform(0, 3, size=(M, dims)).astype(np.float32)
    s = rng.uniform(0, 3, size=(S, dims)).astype(np.float32)
    v = rng.normal(size=S).astype(np.float32)
    g = rng.normal(size=M).astype(np.float32)
    check_bwd(t, s, v, g, 0.5, f"{dims}-d {M}x{S}")


@pytest.mark.parametrize("dims", [1, 2, 3])
def test_nw_gradient_single_source(dims):
    """One source: out_p = (w v) / w = v, so dsources is 0 in exact
    arithmetic.  float32 leaves out_p within two roundings of v, and each
    term (2/h^2) g_p (v - out_p) (t_p - s) keeps that rounding: with random
    roundings the sum stays within 4 standard deviations of
    (2/h^2) 2^-23 |v| sqrt(sum_p g_p^2 (t_p - s)^2).  dtargets and dvals
    (= sum_p g_p) are compared as usual."""
    M, h = 2500, 0.5
    rng = np.random.default_rng(77 + dims)
    t = rng.uniform(0, 3, size=(M, dims)).astype(np.float32)
    s = rng.uniform(0, 3, size=(1, dims)).astype(np.float32)
    v = rng.normal(size=1).astype(np.float32)
    g = rng.normal(size=M).astype(np.float32)
    dt, ds, dv = run_bwd(t, s, v, g, h)
    w_dt, _, w_dv = oracle.nw_regrid_bwd(t, s, v, g, h=h)
    check_f32_scaled(dt, w_dt, f"dtargets {dims}-d one source")
    check_f32_scaled(dv, w_dv, f"dvals {dims}-d one source")
    sigma = (2.0 / h ** 2) * 2.0 ** -23 * abs(float(v[0])) * \
        float(np.sqrt((g[:, None].astype(np.float64) ** 2 * (t - s) ** 2).sum(axis=0)).max())
    assert float(np.abs(ds.cpu().numpy()).max()) <= 4 * sigma, (ds, sigma)


@pytest.mark.parametrize("dims", [2, 3])
def test_nw_gradient_grid_16384(dims):
    """The regrid workload (16384 targets and sources in [0,10]^d) with
    loss = 1/2 sum out^2: gout = out (the oracle's)."""
    t, s, v = inputs.nw_grid_nd(16384, 16384, dims)
    g = oracle.nw_regrid_nd(t, s, v, h=0.5).astype(np.float32)
    check_bwd(t, s, v, g, 0.5, f"{dims}-d 16384x16384")


def test_nw_gradient_demo_inputs_and_another_bandwidth():
    t, s, y = inputs.pages_nw()
    t32, s32, y32 = (a.astype(np.float32) for a in (t, s, y))
    g = np.ones(64, np.float32)
    check_bwd(t32, s32, y32, g, 0.5, "demo inputs")
    check_bwd(t32, s32, y32, g, 0.25, "demo inputs h=0.25")
