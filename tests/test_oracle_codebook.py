"""Pins for the oracle's binary16 rounding and Lloyd-Max codebook (CPU only).

Each check ties the oracle to something other than itself: numpy's float16 cast, closed
forms, the uniform special case, the printed MSE figures, an independent scipy
evaluation of the centroid condition, and a direct minimisation of the distortion.
"""
import math

import numpy as np
import pytest
from scipy import integrate, optimize, special

import oracle
from conftest import golden


def test_round_half_matches_numpy_cast():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e6, 2.0 ** -24, 2.0 ** -25,
         3 * 2.0 ** -26, 2.0 ** -14, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2049.0, 2051.0],
    ])
    got = oracle.round_half(v)
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).astype(np.float64)
    assert np.array_equal(got, want)


def beta_1bit(d):
    return math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)


@pytest.mark.parametrize("d", [8, 64, 128, 200, 1024])
def test_one_bit_closed_form(d):
    # E|u| for one coordinate of a uniform unit vector, and D = 1 - d c^2.
    c, t, mse, _ = oracle.codebook(d, 1)
    cf = beta_1bit(d)
    assert abs(c[1] - cf) < 1e-12 and c[0] == -c[1]
    assert abs(mse - (1 - d * cf * cf)) < 1e-12
    # printed: 1-bit centroids +-sqrt(2/(pi d)) (large-d form), within 0.5% at these d
    if d >= 64:
        assert abs(c[1] / math.sqrt(2 / (math.pi * d)) - 1) < 5e-3


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_uniform_law_is_the_uniform_quantizer(bits):
    # d = 3: one coordinate of a uniform point on the 2-sphere is uniform on [-1, 1]
    # (Archimedes); the Lloyd-Max quantizer is then the uniform one with D = 4^-B.
    c, t, mse, _ = oracle.codebook(3, bits)
    nl = 1 << bits
    want = -1 + (2 * np.arange(nl) + 1) / nl
    assert np.max(np.abs(c - want)) < 1e-13
    assert abs(mse - 4.0 ** -bits) < 1e-13


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_printed_mse_large_d(bits):
    # The page's figures are the d -> infinity values, printed truncated.
    printed = golden("lloyd_max_mse.txt")[f"mse_{bits}"]
    unit = {1: 0.01, 2: 0.001, 3: 0.01, 4: 0.001}[bits]  # one unit of the last printed digit
    _, _, mse_g, _ = oracle.codebook(128, bits, law="gauss")
    _, _, mse_b, _ = oracle.codebook(100000, bits, law="beta")
    for mse in (mse_g, mse_b):
        assert printed <= mse < printed + unit


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_beta_tends_to_gaussian(bits):
    cg, _, mg, _ = oracle.codebook(100000, bits, law="gauss")
    cb, _, mb, _ = oracle.codebook(100000, bits, law="beta")
    assert np.max(np.abs(cb - cg) / np.abs(cg)) < 1e-4
    assert abs(mb - mg) < 1e-4


@pytest.mark.parametrize("d", [64, 128, 200])
def test_distortion_bounds(d):
    # 4^-B <= D(B) <= (sqrt(3) pi / 2) 4^-B, and D 4^B grows with B toward the constant.
    rmax = golden("distortion_bound.txt")["ratio_max"]
    assert abs(rmax - math.sqrt(3) * math.pi / 2) < 1e-12
    prev = 0.0
    for bits in (1, 2, 3, 4):
        _, _, mse, _ = oracle.codebook(d, bits)
        ratio = mse * 4.0 ** bits
        assert 1.0 <= ratio <= rmax
        assert ratio > prev
        prev = ratio


@pytest.mark.parametrize("d,bits", [(128, 1), (128, 2), (128, 3), (128, 4), (200, 2), (200, 4)])
def test_symmetry(d, bits):
    c, t, _, _ = oracle.codebook(d, bits)
    nl = 1 << bits
    assert np.array_equal(c[::-1], -c)
    assert t[nl // 2 - 1] == 0.0
    assert np.all(np.diff(c) > 0)
    assert np.array_equal(t, 0.5 * (c[:-1] + c[1:]))


def _beta_pdf(d):
    a = (d - 3) / 2.0
    lb = special.betaln(0.5, (d - 1) / 2.0)
    return lambda u: math.exp(a * math.log1p(-u * u) - lb) if abs(u) < 1 else 0.0


@pytest.mark.parametrize("d,bits", [(128, 2), (128, 3), (200, 2)])
def test_centroid_condition_scipy(d, bits):
    # Independent integration (scipy quad, and the regularised incomplete beta for cell
    # masses): every centroid is the conditional mean of its cell.
    c, t, mse, _ = oracle.codebook(d, bits)
    f = _beta_pdf(d)
    edges = np.concatenate([[-1.0], t, [1.0]])
    a = (d - 1) / 2.0
    for k in range(len(c)):
        lo, hi = edges[k], edges[k + 1]
        mass = special.betainc(a, a, (hi + 1) / 2) - special.betainc(a, a, (lo + 1) / 2)
        first = integrate.quad(lambda u: u * f(u), lo, hi, epsabs=1e-16, epsrel=1e-13, limit=200)[0]
        assert abs(first / mass - c[k]) < 1e-11
    dist = sum(integrate.quad(lambda u, ck=ck: (u - ck) ** 2 * f(u), edges[k], edges[k + 1],
                              epsabs=1e-16, epsrel=1e-12, limit=200)[0] for k, ck in enumerate(c))
    assert abs(d * dist - mse) < 1e-11


def test_direct_minimisation_agrees():
    # A different algorithm: minimise D over the positive centroids (cells by midpoints).
    d, bits = 128, 2
    c, _, mse, _ = oracle.codebook(d, bits)
    f = _beta_pdf(d)

    def dist(pos):
        p = np.sort(np.abs(pos))
        cc = np.concatenate([-p[::-1], p])
        e = np.concatenate([[-1.0], 0.5 * (cc[:-1] + cc[1:]), [1.0]])
        return d * sum(integrate.quad(lambda u, ck=ck: (u - ck) ** 2 * f(u), e[k], e[k + 1],
                                      epsabs=1e-15, epsrel=1e-12)[0] for k, ck in enumerate(cc))

    res = optimize.minimize(dist, [0.03, 0.15], method="Nelder-Mead",
                            options={"xatol": 1e-9, "fatol": 1e-15, "maxiter": 4000})
    assert abs(res.fun - mse) < 1e-10
    assert np.max(np.abs(np.sort(np.abs(res.x)) - c[2:])) < 1e-5
