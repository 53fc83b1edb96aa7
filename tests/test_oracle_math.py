"""Pins of the oracle's random numbers, rotation and Lloyd-Max codebook.

Each check compares the oracle with something other than itself: a published
test vector, a closed form, a textbook special case, an independent library
routine (scipy's regularized incomplete beta), or a known limit.  Page
citations ("TQ") refer to "TurboQuant explained" (a2a-mcp.org).
"""

import math

import numpy as np
import pytest
from scipy import special, stats

from oracle import tq_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# --- SplitMix64 / Box-Muller ------------------------------------------------

def test_splitmix64_published_vector():
    # The reference SplitMix64 (Steele, Lea & Flood 2014; Vigna's splitmix64.c)
    # seeded with 1234567 emits these first five outputs.
    expect = [6457827717110365317, 3203168211198807973, 9817491932198370423,
              4593380528125082431, 16408922859458223821]
    assert [int(v) for v in O.splitmix64(1234567, 5)] == expect


def test_splitmix64_counter_form_matches_stream_cut():
    a = O.splitmix64(99, 40)
    b = O.splitmix64(99, 15, start=25)
    assert np.array_equal(a[25:], b)


def test_uniforms_range_and_mean():
    u = O.uniforms(7, 200_000)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 4 * math.sqrt(1 / 12 / len(u))


def test_box_muller_is_standard_normal():
    z = O.gaussians(0x5EED0001, 200_000)
    ks = stats.kstest(z, "norm")
    assert ks.pvalue > 1e-3
    assert abs(z.mean()) < 4 / math.sqrt(len(z))
    assert abs(z.var() - 1.0) < 4 * math.sqrt(2 / len(z))


# --- rotation: TQ §Stage 1 ----------------------------------------------------

@pytest.mark.parametrize("d", [2, 8, 128, 200])
def test_rotation_orthogonal_and_qr(d):
    Pi, R, G = O.rotation(d, 0x5EED0001)
    assert np.max(np.abs(Pi.T @ Pi - np.eye(d))) <= 1e-12
    assert np.max(np.abs(Pi @ R - G)) <= 1e-12 * max(1.0, np.max(np.abs(G)))
    assert np.all(np.diag(R) > 0)
    assert np.allclose(np.triu(R), R)


@pytest.mark.parametrize("d", [2, 3, 5, 8])
def test_rotation_equals_gram_schmidt(d):
    # With diag(R) > 0 the Q factor is unique: classical Gram-Schmidt on the
    # columns of G (a textbook routine) must give the same matrix.
    Pi, _, G = O.rotation(d, 12345 + d)
    Q = np.zeros_like(G)
    for k in range(d):
        v = G[:, k].copy()
        for i in range(k):
            v -= (Q[:, i] @ G[:, k]) * Q[:, i]
        Q[:, k] = v / np.linalg.norm(v)
    assert np.max(np.abs(Q - Pi)) < 1e-12


# --- Lloyd-Max for the Beta coordinate law: TQ §Stage 1 ---------------------

@pytest.mark.parametrize("d", [2, 3, 16, 128])
def test_one_bit_closed_form(d):
    # b = 1: the two cells are the half lines, so c = +-E|T| with
    # E|T| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)).  For d = 2 this is 2/pi.
    cb = O.lloyd_max(d, 1)
    e_abs = math.exp(math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d + 1) / 2))
    assert np.allclose(cb.centroids, [-e_abs, e_abs], rtol=0, atol=1e-13)
    if d == 2:
        assert abs(cb.centroids[1] - 2 / math.pi) < 1e-13


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5])
def test_uniform_law_at_d3(b):
    # For d = 3 the coordinate law is uniform on [-1, 1] (Archimedes); its
    # Lloyd-Max quantizer is the uniform one with distortion step^2 / 12.
    cb = O.lloyd_max(3, b)
    K = 1 << b
    step = 2.0 / K
    assert np.allclose(cb.centroids, -1 + step * (np.arange(K) + 0.5), rtol=0, atol=1e-13)
    assert abs(cb.distortion - step ** 2 / 12) < 1e-14


def _cond_mean_closed_form(lo, hi, d):
    # numerator: int t (1-t^2)^((d-3)/2) dt = -(1-t^2)^((d-1)/2) / (d-1)
    # denominator: regularized incomplete beta of (1+t)/2 (scipy, independent)
    a = (d - 1) / 2.0
    C = O.density_const(d)
    num = C * (-(1 - hi ** 2) ** ((d - 1) / 2) + (1 - lo ** 2) ** ((d - 1) / 2)) / (d - 1)
    den = special.betainc(a, a, (1 + hi) / 2) - special.betainc(a, a, (1 + lo) / 2)
    return num / den


@pytest.mark.parametrize("d,b", [(16, 2), (16, 4), (128, 2), (128, 3), (128, 4), (200, 2), (200, 4), (128, 6)])
def test_centroids_are_conditional_means(d, b):
    cb = O.lloyd_max(d, b)
    e = np.concatenate(([-1.0], cb.boundaries, [1.0]))
    ref = _cond_mean_closed_form(e[:-1], e[1:], d)
    assert np.max(np.abs(cb.centroids - ref)) <= 1e-12


@pytest.mark.parametrize("d,b", [(128, 3), (200, 4), (7, 5)])
def test_boundaries_are_midpoints_and_symmetric(d, b):
    cb = O.lloyd_max(d, b)
    c = cb.centroids
    assert np.array_equal(cb.boundaries, 0.5 * (c[1:] + c[:-1]))
    assert np.array_equal(c, -c[::-1])
    assert np.all(np.diff(c) > 0)


def test_distortion_strictly_decreasing_in_b():
    D = [O.lloyd_max(128, b).distortion for b in range(1, 9)]
    assert all(D[i + 1] < D[i] for i in range(7))


def test_distortion_within_information_bounds():
    # Any b-bit code of unit vectors has MSE >= 4^-b (Shannon lower bound on
    # the sphere); the Lloyd-Max scalar code stays below (sqrt(3) pi / 2) 4^-b
    # (Panter-Dite).  Total MSE per unit vector is d * D.
    for b in range(1, 9):
        tot = 128 * O.lloyd_max(128, b).distortion
        assert 4.0 ** -b <= tot <= math.sqrt(3) * math.pi / 2 * 4.0 ** -b


def test_large_d_approaches_gaussian_lloyd_max():
    # sqrt(d) T -> N(0, 1) as d grows, so sqrt(d) c and d D approach Max's
    # (1960) Gaussian table.  Loose: the Beta law differs at O(1/d).
    max_c = {1: [0.7979], 2: [0.4528, 1.510], 3: [0.2451, 0.7560, 1.344, 2.152]}
    max_D = {1: 0.3634, 2: 0.1175, 3: 0.03454, 4: 0.009497}
    for b, cpos in max_c.items():
        cb = O.lloyd_max(4096, b)
        got = cb.centroids[len(cb.centroids) // 2:] * math.sqrt(4096)
        assert np.allclose(got, cpos, rtol=2e-3, atol=0)
    for b, ref in max_D.items():
        assert abs(4096 * O.lloyd_max(4096, b).distortion / ref - 1) < 3e-3
        assert abs(128 * O.lloyd_max(128, b).distortion / ref - 1) < 3e-2


def test_density_integrates_to_one():
    for d in (2, 3, 10, 128, 200):
        P, M1, M2 = O.cell_moments(np.array([-1.0]), np.array([1.0]), d)
        assert abs(P[0] - 1) < 1e-12
        assert abs(M1[0]) < 1e-14
        assert abs(M2[0] - 1.0 / d) < 1e-12      # E[T^2] = 1/d on the sphere


def test_fp16_rounding_is_ieee_nearest_even():
    one_ulp = 2.0 ** -10
    assert float(O.fp16(1 + one_ulp / 2)) == 1.0                  # tie -> even
    assert float(O.fp16(1 + 3 * one_ulp / 2)) == 1 + 2 * one_ulp  # tie -> even
    assert float(O.fp16(1 + one_ulp / 2 + 1e-12)) == 1 + one_ulp
    assert np.isinf(O.fp16(65520.0)) and float(O.fp16(65519.0)) == 65504.0
