"""Pins of the polar-form oracle (oracle/polar_oracle.py) against what the
mathematics fixes: the transform's inverse and norm, the complex argument,
special vectors, the Beta law of the angles (scipy), the conditional means
of the codebook cells (scipy quadrature), the uniform quantizer, Monte Carlo
laws and distortions, and brute force over every codeword of a small case.
"""

import math

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import polar_oracle as P

SEED_PI = 0x5EED0001


def _sphere(seed, n, d):
    x = np.random.default_rng(seed).standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def _beta_angle_pdf(level, phi):
    """Density of a level-l angle from scipy's Beta law of sin^2 phi."""
    k = 1 << (level - 1)
    s, c = np.sin(phi), np.cos(phi)
    return stats.beta(k / 2, k / 2).pdf(s * s) * 2.0 * s * c


# ---------------------------------------------------------------- transform


@pytest.mark.parametrize("d", [2, 4, 8, 128])
def test_round_trip_and_radius(d):
    X = np.random.default_rng(d).standard_normal((50, d)) * np.exp(np.random.default_rng(d + 1).uniform(-3, 3, (50, 1)))
    angles, radius = P.polar_forward(X)
    assert [a.shape[1] for a in angles] == [d >> level for level in range(1, P.n_levels(d) + 1)]
    assert np.allclose(radius, np.linalg.norm(X, axis=1), rtol=1e-14, atol=0)
    assert np.allclose(P.polar_inverse(angles, radius), X, rtol=0, atol=1e-13 * np.abs(X).max())


def test_two_dimensional_angle_is_the_complex_argument():
    X = np.random.default_rng(3).standard_normal((200, 2))
    angles, radius = P.polar_forward(X)
    z = X[:, 0] + 1j * X[:, 1]
    assert np.allclose(angles[0][:, 0], np.angle(z), rtol=0, atol=1e-15)
    assert np.allclose(radius, np.abs(z), rtol=1e-15, atol=0)


def test_special_vectors():
    e0, e7 = np.eye(8)[0], np.eye(8)[7]
    ones = np.ones(8) / math.sqrt(8)
    neg = np.array([-1.0, 0, 0, -1.0, 0, 0, 0, 0]) / math.sqrt(2)
    angles, _ = P.polar_forward(np.stack([e0, e7, ones, neg]))
    h = math.pi / 2
    assert np.array_equal(angles[0][0], [0, 0, 0, 0]) and np.array_equal(angles[1][0], [0, 0])
    assert np.array_equal(angles[0][1], [0, 0, 0, h])
    assert np.array_equal(angles[1][1], [0, h]) and np.array_equal(angles[2][1], [h])
    for lv in range(3):
        assert np.allclose(angles[lv][2], math.pi / 4, rtol=0, atol=1e-15)
    # (-1, 0) has angle pi, (0, -1) angle -pi/2; both pairs have radius 1/sqrt(2)
    assert np.allclose(angles[0][3], [math.pi, -h, 0, 0], rtol=0, atol=1e-15)
    assert np.allclose(angles[1][3], [math.pi / 4, 0], rtol=0, atol=1e-15)


def test_non_power_of_two_is_refused():
    for n in (0, 1, 3, 6, 200):
        with pytest.raises(ValueError):
            P.n_levels(n)


# ---------------------------------------------------------------- angle laws


@pytest.mark.parametrize("level", [2, 3, 4, 5, 7])
def test_angle_law_is_the_beta_law(level):
    k = 1 << (level - 1)
    phi = np.linspace(0.05, math.pi / 2 - 0.05, 9)
    cdf = np.array([P._cell_moments(level, np.array([0.0]), np.array([x]))[0][0] for x in phi])
    assert np.allclose(cdf, stats.beta(k / 2, k / 2).cdf(np.sin(phi) ** 2), rtol=0, atol=1e-12)
    # relative agreement at every point, down to densities of 1e-63 (level 7)
    assert np.allclose(P.angle_density(level, phi), _beta_angle_pdf(level, phi), rtol=1e-10, atol=0)
    total = P._cell_moments(level, np.array([0.0]), np.array([math.pi / 2]))[0][0]
    assert abs(total - 1.0) < 1e-13


def test_level_one_law_is_uniform():
    phi = np.array([-3.0, -1.0, 0.0, 2.5])
    assert np.allclose(P.angle_density(1, phi), 1 / (2 * math.pi))
    assert P.angle_density(1, np.array([3.5]))[0] == 0.0


def test_angles_of_uniform_unit_vectors_follow_the_laws():
    angles, _ = P.polar_forward(_sphere(11, 20000, 64))
    p1 = stats.kstest(angles[0].ravel()[:20000], stats.uniform(-math.pi, 2 * math.pi).cdf).pvalue
    assert p1 > 1e-4
    for level in range(2, 7):
        k = 1 << (level - 1)
        a = angles[level - 1].ravel()[:20000]
        p = stats.kstest(a, lambda x: stats.beta(k / 2, k / 2).cdf(np.sin(x) ** 2)).pvalue
        assert p > 1e-4, (level, p)


# ---------------------------------------------------------------- codebooks


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_level_one_codebook_is_the_uniform_quantizer(bits):
    cb = P.angle_lloyd_max(1, bits)
    K = 1 << bits
    step = 2 * math.pi / K
    assert np.allclose(cb.centroids, -math.pi + step * (np.arange(K) + 0.5), rtol=0, atol=1e-12)
    assert abs(cb.distortion - step * step / 12) < 1e-12


@pytest.mark.parametrize("level", [2, 3, 5, 6])
@pytest.mark.parametrize("bits", [1, 2, 4])
def test_codebook_cells_are_conditional_means(level, bits):
    cb = P.angle_lloyd_max(level, bits)
    c, t = cb.centroids, cb.boundaries
    assert np.all(np.diff(c) > 0)
    assert np.allclose(t, 0.5 * (c[1:] + c[:-1]), rtol=0, atol=1e-15)
    assert np.allclose(c + c[::-1], math.pi / 2, rtol=0, atol=1e-14)
    e = np.concatenate(([0.0], t, [math.pi / 2]))
    for i in range(len(c)):
        p = integrate.quad(lambda x: _beta_angle_pdf(level, x), e[i], e[i + 1], epsabs=1e-14, epsrel=1e-13)[0]
        m = integrate.quad(lambda x: x * _beta_angle_pdf(level, x), e[i], e[i + 1], epsabs=1e-14, epsrel=1e-13)[0]
        assert abs(c[i] - m / p) < 1e-9, (level, bits, i)


def test_distortion_falls_with_bits_and_matches_monte_carlo():
    angles, _ = P.polar_forward(_sphere(12, 4096, 32))
    for level in range(1, 6):
        prev = math.inf
        for bits in (1, 2, 3, 4):
            cb = P.angle_lloyd_max(level, bits)
            assert cb.distortion < prev
            prev = cb.distortion
            a = angles[level - 1].ravel()
            err = (a - cb.centroids[P.quantize_angles([a], [cb])[0]]) ** 2
            sigma = err.std() / math.sqrt(err.size)
            assert abs(err.mean() - cb.distortion) < 4 * sigma + 1e-12, (level, bits)


# ---------------------------------------------------------------- codec


def test_encode_is_nearest_centroid_and_every_codeword_decodes_to_a_unit_vector():
    codec = P.make_polar_codec(4, 2, SEED_PI)
    X = np.random.default_rng(13).standard_normal((500, 4))
    enc = P.polar_encode(codec, X)
    for a, i, book in zip(enc.angles, enc.idx, codec.books):
        brute = np.argmin(np.abs(a[..., None] - book.centroids), axis=-1)
        assert np.array_equal(i, brute)
    # all 4^3 codewords of d = 4, b = 2 (2 level-1 angles, 1 level-2 angle)
    grid = np.array(np.meshgrid(range(4), range(4), range(4), indexing="ij")).reshape(3, -1).T
    U = P.polar_decode_unit(codec, [grid[:, :2], grid[:, 2:]])
    assert np.allclose(np.linalg.norm(U, axis=1), 1.0, rtol=0, atol=1e-15)
    assert len({tuple(np.round(u, 12)) for u in U}) == 64


def test_reconstruction_error_falls_with_bits_and_logits_follow():
    X = np.random.default_rng(14).standard_normal((400, 16)) * 3.0
    Q = np.random.default_rng(15).standard_normal((8, 16))
    exact = Q @ X.T
    prev_mse, prev_err = math.inf, math.inf
    for bits in (1, 2, 3, 4):
        codec = P.make_polar_codec(16, bits, SEED_PI)
        enc = P.polar_encode(codec, X)
        Xh = P.polar_decode(codec, enc)
        mse = np.mean(np.sum((Xh - X) ** 2, axis=1) / np.sum(X * X, axis=1))
        L = P.polar_logits(codec, Q, enc)
        assert np.allclose(L, Q @ Xh.T, rtol=0, atol=1e-12 * np.abs(L).max())
        err = np.abs(L - exact).max() / np.abs(exact).max()
        assert mse < prev_mse and err < prev_err
        prev_mse, prev_err = mse, err
    assert prev_mse < 0.02


def test_zero_vector_decodes_to_zero():
    codec = P.make_polar_codec(8, 2, SEED_PI)
    enc = P.polar_encode(codec, np.zeros((2, 8)))
    assert np.array_equal(P.polar_decode(codec, enc), np.zeros((2, 8)))


def test_qjl_on_the_polar_residual_is_unbiased_with_closed_form_variance():
    # Stage 2 over the polar stage 1: with Pi fixed and 1000 seeds for S the
    # mean error is within 3 sigma / sqrt(1000) of 0, and the variance matches
    # ||k||^2 ||r||^2 (pi/2)/m (||q||^2 - (2/pi) <q, r/||r||>^2).
    d, b, m = 64, 2, 64
    rng = np.random.default_rng(16)
    k = rng.standard_normal(d) * 1.5
    q = rng.standard_normal(d)
    base = P.make_polar_codec(d, b, SEED_PI)
    est = []
    for seed in range(1000):
        codec = P.PolarCodec(d, b, base.Pi, base.books, m, np.random.default_rng(5000 + seed).standard_normal((m, d)))
        enc = P.polar_encode(codec, k[None, :])
        u = k / np.linalg.norm(k)
        r = u - P.polar_decode_unit(codec, enc.idx)[0] @ codec.Pi
        # un-rounded side values, so that only the sketch is random
        enc.norm16 = np.array([np.linalg.norm(k)])
        enc.rnorm16 = np.array([np.linalg.norm(r)])
        est.append(P.polar_logits(codec, q[None, :], enc)[0, 0])
    err = np.array(est) - q @ k
    sigma = err.std(ddof=1)
    assert abs(err.mean()) < 3 * sigma / math.sqrt(len(err))
    rhat = r / np.linalg.norm(r)
    var_cf = (k @ k) * (r @ r) * (math.pi / 2) / m * (q @ q - (2 / math.pi) * (q @ rhat) ** 2)
    chi2 = (len(err) - 1) * sigma ** 2 / var_cf
    lo, hi = stats.chi2.ppf([0.0005, 0.9995], len(err) - 1)
    assert lo < chi2 < hi


def test_stage_one_logit_is_biased_where_the_sketch_is_not():
    # The stage-1 estimate <q, x_hat> alone is off by <q, ||x|| Pi^T r> for
    # this key; averaging the sketch term over seeds removes that offset.
    d, b, m = 32, 1, 32
    rng = np.random.default_rng(17)
    k, q = rng.standard_normal(d), rng.standard_normal(d)
    base = P.make_polar_codec(d, b, SEED_PI)
    stage1 = P.polar_logits(base, q[None, :], P.polar_encode(base, k[None, :]))[0, 0]
    vals = []
    for seed in range(600):
        codec = P.PolarCodec(d, b, base.Pi, base.books, m, np.random.default_rng(7000 + seed).standard_normal((m, d)))
        vals.append(P.polar_logits(codec, q[None, :], P.polar_encode(codec, k[None, :]))[0, 0])
    vals = np.array(vals)
    se = vals.std(ddof=1) / math.sqrt(len(vals))
    exact = q @ k
    assert abs(stage1 - exact) > 6 * se          # stage 1 alone misses by many standard errors
    assert abs(vals.mean() - exact) < 4 * se + 2e-3 * abs(exact)   # fp16 side values only
