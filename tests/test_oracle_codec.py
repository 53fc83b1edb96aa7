"""Pins of the oracle's quantize / QJL / logit / value steps and of the
packed record layout.

"TQ" is the page "TurboQuant explained" (a2a-mcp.org).  Statistical checks
use fixed seeds and bounds of several standard errors.
"""

import math
import os

import numpy as np
import pytest
from scipy import stats

from oracle import tq_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _page_figure(name):
    """A figure printed on the page, from tests/golden/page_figures.txt."""
    path = os.path.join(os.path.dirname(__file__), "golden", "page_figures.txt")
    for line in open(path, encoding="utf-8"):
        parts = line.split()
        if parts and not line.startswith("#") and parts[0] == name:
            return float(parts[1])
    raise KeyError(name)


def _unit_rows(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


@pytest.mark.parametrize("d", [16, 128])
def test_rotated_coordinates_follow_beta_law(d):
    # TQ §Stage 1: after the rotation each coordinate of a unit vector is
    # Beta((d-1)/2, (d-1)/2) on [-1, 1].  Kolmogorov-Smirnov against scipy.
    rng = np.random.default_rng(1)
    Pi, _, _ = O.rotation(d, 0x5EED0001)
    y = (_unit_rows(rng, 20000, d) @ Pi.T)[:, 3]
    a = (d - 1) / 2
    assert stats.kstest(y, stats.beta(a, a, loc=-1, scale=2).cdf).pvalue > 1e-3


def test_indices_are_nearest_centroids_brute_force():
    # Lloyd-Max cells in one dimension are the Voronoi cells of the centroids.
    rng = np.random.default_rng(2)
    codec = O.make_codec(16, 3, 16, 11, 12)
    enc = O.encode(codec, rng.standard_normal((64, 16)))
    c = codec.cb.centroids
    for n in range(64):
        for j in range(16):
            assert enc.idx[n, j] == int(np.argmin(np.abs(enc.y[n, j] - c)))


def test_empirical_mse_matches_codebook_distortion():
    # E||u - Pi^T c[idx]||^2 over random unit vectors equals d * D_b.
    d, b = 128, 3
    rng = np.random.default_rng(3)
    codec = O.make_codec(d, b, 0, 0x5EED0001, 0)
    U = _unit_rows(rng, 20000, d)
    enc = O.encode(codec, U)
    err = np.sum((U - codec.cb.centroids[enc.idx] @ codec.Pi) ** 2, axis=1)
    se = err.std() / math.sqrt(len(err))
    assert abs(err.mean() - d * codec.cb.distortion) < 5 * se


@pytest.mark.parametrize("d,b", [(64, 1), (64, 3), (128, 1), (128, 2), (128, 3), (200, 2), (200, 3), (256, 3)])
def test_reconstruction_levels_eight_bit_fixed_point(d, b):
    # b <= 3: every level is an integer times 2^-f with |integer| <= 127, f is
    # the largest such exponent, each level moved by at most 2^-(f+1), the
    # set stays antisymmetric and ascending, and the distortion of the
    # rounded levels (exact moments of the Beta law per cell) exceeds the
    # Lloyd-Max optimum by less than 0.3 %.
    cb = O.lloyd_max(d, b)
    lev, f = O.reconstruction_levels(cb.centroids)
    k = lev * 2.0 ** f
    assert np.all(k == np.round(k)) and np.max(np.abs(k)) <= 127
    assert np.max(np.abs(cb.centroids)) * 2.0 ** (f + 1) > 127
    assert np.max(np.abs(lev - cb.centroids)) <= 2.0 ** -(f + 1)
    assert np.array_equal(lev, -lev[::-1]) and np.all(np.diff(lev) > 0)
    e = np.concatenate(([-1.0], cb.boundaries, [1.0]))
    P, M1, M2 = O.cell_moments(e[:-1], e[1:], d)
    D_rec = float(np.sum(M2 - 2.0 * lev * M1 + lev * lev * P))
    assert cb.distortion <= D_rec < cb.distortion * 1.003


def test_reconstruction_levels_fp16_beyond_eight_levels():
    cb = O.lloyd_max(128, 4)
    lev, f = O.reconstruction_levels(cb.centroids)
    assert f is None and np.array_equal(lev, O.fp16(cb.centroids).astype(np.float64))


def test_three_bit_cosine_similarity_community_figure():
    # TQ §Stage 2 quotes a reconstruction cosine of 0.983+ at 3 bits; the
    # MSE-stage reconstruction alone gives sqrt(1 - d D_3) ~ 0.983.
    d = 128
    rng = np.random.default_rng(4)
    codec = O.make_codec(d, 3, 0, 0x5EED0001, 0)
    U = _unit_rows(rng, 5000, d)
    enc = O.encode(codec, U)
    V = O.dequantize(codec, enc.idx, np.ones(len(U), np.float16))
    cos = np.sum(U * V, axis=1) / np.linalg.norm(V, axis=1)
    figure = _page_figure("cosine_similarity_3bit_min")      # 0.983, a lower bound
    assert figure - 0.003 <= cos.mean() <= figure + 0.003
    assert abs(cos.mean() - math.sqrt(1 - d * codec.cb.distortion)) < 2e-3


def test_qjl_estimator_unbiased_over_seeds_with_closed_form_variance():
    # TQ §Stage 2: the sign sketch corrects the inner-product bias.  With Pi
    # fixed and 1000 seeds for S, the mean error is within 3 sigma / sqrt(1000)
    # of 0, and the variance matches the closed form
    # ||k||^2 ||r||^2 (pi/2)/m (||q||^2 - (2/pi) <q, r/||r||>^2).
    d, b, m = 128, 3, 128
    rng = np.random.default_rng(5)
    k = rng.standard_normal(d) * 2.0
    q = rng.standard_normal(d)
    base = O.make_codec(d, b, m, 0x5EED0001, 0)
    est = []
    for seed in range(1000):
        S = O.qjl_matrix(m, d, 1000 + seed)
        codec = O.Codec(d, b, m, base.Pi, S, base.cb)
        enc = O.encode(codec, k[None, :])
        # use the un-rounded norms so only the sketch is random
        u = k / np.linalg.norm(k)
        r = u - codec.crec[enc.idx[0]] @ codec.Pi
        L = O.logits_from_codes(codec, q[None, :], enc.idx, enc.qneg,
                                np.array([np.linalg.norm(k)]), np.array([np.linalg.norm(r)]))
        est.append(L[0, 0])
    est = np.array(est)
    err = est - q @ k
    sigma = err.std(ddof=1)
    assert abs(err.mean()) < 3 * sigma / math.sqrt(len(err))
    rhat = r / np.linalg.norm(r)
    var_cf = (k @ k) * (r @ r) * (math.pi / 2) / m * (q @ q - (2 / math.pi) * (q @ rhat) ** 2)
    chi2 = (len(err) - 1) * sigma ** 2 / var_cf
    lo, hi = stats.chi2.ppf([0.0005, 0.9995], len(err) - 1)
    assert lo < chi2 < hi


def test_unbiased_when_rotation_also_varies():
    d, b, m = 64, 2, 64
    rng = np.random.default_rng(6)
    k = rng.standard_normal(d)
    q = rng.standard_normal(d)
    errs = []
    for seed in range(400):
        codec = O.make_codec(d, b, m, 7000 + seed, 9000 + seed)
        enc = O.encode(codec, k[None, :])
        u = k / np.linalg.norm(k)
        r = u - codec.crec[enc.idx[0]] @ codec.Pi
        L = O.logits_from_codes(codec, q[None, :], enc.idx, enc.qneg,
                                np.array([np.linalg.norm(k)]), np.array([np.linalg.norm(r)]))
        errs.append(L[0, 0] - q @ k)
    errs = np.array(errs)
    assert abs(errs.mean()) < 3 * errs.std(ddof=1) / math.sqrt(len(errs))


def test_high_bit_width_recovers_exact_logits():
    # The estimate converges to the exact dot product as b grows: the residual
    # norm, and with it the error, halves with every extra bit (Lloyd-Max
    # distortion ~ 4^-b).  At b = 8 with m = 128 the rms error is below
    # 1e-3 ||q|| ||k||; what is left is the sketch's own standard deviation
    # ||r|| sqrt(pi / (2 m)) plus the fp16 rounding of the norms.
    d, m = 128, 128
    rng = np.random.default_rng(7)
    K = rng.standard_normal((256, d)) * 3.0
    Qv = rng.standard_normal((8, d))
    exact = O.exact_logits(Qv, K)
    scale = np.linalg.norm(Qv, axis=1)[:, None] * np.linalg.norm(K, axis=1)[None, :]
    rms = []
    for b in range(1, 9):
        codec = O.make_codec(d, b, m, 0x5EED0001, 0x5EED0002)
        enc = O.encode(codec, K)
        L = O.logits_from_codes(codec, Qv, enc.idx, enc.qneg, enc.norm16, enc.rnorm16)
        rel = (L - exact) / scale
        rms.append(math.sqrt(np.mean(rel ** 2)))
        pred = math.sqrt(d * codec.cb.distortion) * math.sqrt(math.pi / (2 * m))
        assert 0.7 * pred < rms[-1] < 1.3 * pred + 3e-4
    assert rms[-1] < 1e-3
    assert all(rms[i] / rms[i + 1] > 1.6 for i in range(6))


def test_mse_only_logits_equal_inner_product_with_reconstruction():
    # With m = 0 the logit is <q, v_hat>: rotating the query once (Pi q) and
    # dotting with crec[idx] is the same as dequantizing the key first.
    rng = np.random.default_rng(8)
    codec = O.make_codec(64, 3, 0, 21, 0)
    K = rng.standard_normal((50, 64))
    Qv = rng.standard_normal((5, 64))
    enc = O.encode(codec, K)
    L = O.logits_from_codes(codec, Qv, enc.idx, None, enc.norm16, None)
    Vh = O.dequantize(codec, enc.idx, enc.norm16)
    assert np.allclose(L, Qv @ Vh.T, rtol=1e-12, atol=1e-12)
    W = rng.random((5, 50))
    assert np.allclose(O.weighted_values(codec, W, enc.idx, enc.norm16), W @ Vh, rtol=1e-12, atol=1e-12)


def test_high_bit_width_values_reconstruct():
    rng = np.random.default_rng(9)
    codec = O.make_codec(128, 8, 0, 0x5EED0001, 0)
    V = rng.standard_normal((64, 128))
    enc = O.encode(codec, V)
    Vh = O.dequantize(codec, enc.idx, enc.norm16)
    rel = np.linalg.norm(Vh - V, axis=1) / np.linalg.norm(V, axis=1)
    assert rel.max() < 2e-2 and rel.mean() < math.sqrt(128 * codec.cb.distortion) * 1.2


def test_zero_vector():
    codec = O.make_codec(128, 3, 128, 1, 2)
    X = np.zeros((2, 128))
    X[1, 5] = 1.0
    enc = O.encode(codec, X)
    assert np.all(enc.idx[0] == 4) and float(enc.norm16[0]) == 0.0
    L = O.logits_from_codes(codec, np.ones((1, 128)), enc.idx, enc.qneg, enc.norm16, enc.rnorm16)
    assert L[0, 0] == 0.0


def test_norm_side_values_are_fp16():
    codec = O.make_codec(64, 2, 64, 1, 2)
    X = np.full((1, 64), 1.0 / 3.0)
    enc = O.encode(codec, X)
    assert enc.norm16.dtype == np.float16
    assert float(enc.norm16[0]) == float(np.float16(math.sqrt(64) / 3.0))


# --- packed layout -----------------------------------------------------------

@pytest.mark.parametrize("d,b,m", [(128, 3, 128), (128, 2, 128), (128, 4, 128), (128, 1, 128),
                                   (128, 3, 0), (64, 3, 64), (200, 2, 200), (200, 4, 200), (96, 3, 0)])
def test_pack_unpack_round_trip(d, b, m):
    rng = np.random.default_rng(10)
    lay = O.Layout(d, b, m, 64, 2)
    idx = rng.integers(0, 1 << b, size=(33, d))
    qneg = rng.random((33, m)) < 0.5 if m else None
    words = O.pack_codes(lay, idx, qneg)
    assert words.shape == (33, 4, lay.words)
    idx2, qneg2 = O.unpack_codes(lay, words)
    assert np.array_equal(idx, idx2)
    if m:
        assert np.array_equal(qneg, qneg2)


def test_record_sizes():
    # d = 128, m = 128: 3-bit keys are 64 code bytes + 4 norm bytes = 68 B,
    # 2-bit keys 52 B, 4-bit keys 84 B; 3-bit values (no QJL) 48 + 2 = 50 B.
    sizes = {(3, 128): 68, (2, 128): 52, (4, 128): 84, (3, 0): 50}
    for (b, m), total in sizes.items():
        lay = O.Layout(128, b, m, 64, 8)
        assert lay.code_bytes + lay.norm_bytes == total
    assert O.Layout(128, 3, 128, 64, 8).head_block_bytes == 64 * 68


def test_layout_hand_worked_bits():
    # d = 64, b = 3, m = 64: E = F = 16, so each chunk holds a trailing group of
    # 16 elements in 2 index words (code bit k of element l at word l//8, bit
    # 4 (l%8) + k) and one QJL word (row l at bit 8 (l%4) + (l%32)//4).
    #  coordinate 5  -> chunk 0, l = 5: code 1 -> word 0 bit 20.
    #  coordinate 17 -> chunk 1, l = 1: code 7 -> word 0 bits 4, 5, 6.
    #  coordinate 26 -> chunk 1, l = 10: code 6 -> word 1 bits 9, 10.
    #  projection 34 -> chunk 2, l = 2: bit 16; projection 63 -> chunk 3, l = 15: bit 27.
    lay = O.Layout(64, 3, 64, 64, 1)
    assert lay.n_idx == 2 and lay.words == 3
    idx = np.zeros((1, 64), dtype=np.int64)
    idx[0, 5] = 1
    idx[0, 17] = 7
    idx[0, 26] = 6
    qneg = np.zeros((1, 64), bool)
    qneg[0, 34] = True
    qneg[0, 63] = True
    w = O.pack_codes(lay, idx, qneg)[0]
    assert [int(v) for v in w[0]] == [1 << 20, 0, 0]
    assert [int(v) for v in w[1]] == [0b111 << 4, 0b11 << 9, 0]
    assert [int(v) for v in w[2]] == [0, 0, 1 << 16]
    assert [int(v) for v in w[3]] == [0, 0, 1 << 27]


def test_layout_hand_worked_bits_dense_groups():
    # b = 3, d = 128: E = 32, one full group of 3 words per chunk.
    #  element 9  (l' = 9 < 24): code 5 -> word 1, bits 4 + {0, 2}.
    #  element 26 (l' = 26 >= 24, e = 2): code 6 -> bit 1 in word 1 and bit 2
    #  in word 2, both at bit 4 e + 3 = 11.
    lay = O.Layout(128, 3, 0, 64, 1)
    assert lay.n_idx == 3
    idx = np.zeros((1, 128), dtype=np.int64)
    idx[0, 9] = 5
    idx[0, 26] = 6
    w = O.pack_codes(lay, idx, None)[0]
    assert [int(v) for v in w[0]] == [0, (1 << 4) | (1 << 6) | (1 << 11), 1 << 11]
    # b = 2, d = 128: E = 32, 2 words; element 13 (l%16 = 13): code 2 ->
    # word 0, bit 4 (13%8) + 2 (13//8) + 1 = 23.
    lay = O.Layout(128, 2, 0, 64, 1)
    idx = np.zeros((1, 128), dtype=np.int64)
    idx[0, 13] = 2
    idx[0, 32 + 20] = 3           # chunk 1, l = 20: word 1, bits 4*4 + 2*0 = 16, 17
    w = O.pack_codes(lay, idx, None)[0]
    assert [int(v) for v in w[0]] == [1 << 23, 0]
    assert [int(v) for v in w[1]] == [0, 0b11 << 16]
    # b = 1: element 11 (l%32 = 11): word 0, bit 4 (11%8) + 11//8 = 13.
    lay = O.Layout(128, 1, 0, 64, 1)
    idx = np.zeros((1, 128), dtype=np.int64)
    idx[0, 11] = 1
    assert [int(v) for v in O.pack_codes(lay, idx, None)[0, 0]] == [1 << 13]
    # b = 4 (sign-magnitude nibbles, H = 8), d = 128: coordinate 37 -> chunk 1,
    # l = 5: word 0, nibble at 4 ((5%8)//2 + 4 (5%2)) = 24; idx 2 -> neg 1,
    # mu 5 -> nibble 0b1101.
    lay = O.Layout(128, 4, 0, 64, 1)
    idx = np.full((1, 128), 8)
    idx[0, 37] = 2
    w = O.pack_codes(lay, idx, None)[0]
    assert [int(v) for v in w[1]] == [0b1101 << 24, 0, 0, 0]
    assert not w[0].any() and not w[2].any() and not w[3].any()


def test_pages_round_trip_with_block_table():
    rng = np.random.default_rng(11)
    lay = O.Layout(128, 3, 128, 64, 2)
    n_pages = 8
    pages = np.zeros(n_pages * lay.page_bytes, np.uint8)
    bt = rng.permutation(n_pages).reshape(2, 4).astype(np.int32)
    codec = O.make_codec(128, 3, 128, 5, 6)
    X = rng.standard_normal((150, 128))
    enc = O.encode(codec, X)
    pos = np.arange(30, 180)
    O.write_pages(lay, pages, bt, 1, 1, pos, enc.idx, enc.qneg, enc.norm16, enc.rnorm16)
    idx, qneg, n16, r16 = O.read_pages(lay, pages, bt, 1, 1, pos)
    assert np.array_equal(idx, enc.idx) and np.array_equal(qneg, enc.qneg)
    assert np.array_equal(n16, enc.norm16) and np.array_equal(r16, enc.rnorm16)
    # head 0 of sequence 1 and everything of sequence 0 stay untouched
    for p in bt[0]:
        assert not pages[p * lay.page_bytes:(p + 1) * lay.page_bytes].any()


def _attn_inputs(rng, d, n, bits_k=3, m=64, bits_v=3):
    kc = O.make_codec(d, bits_k, m, 31, 32)
    vc = O.make_codec(d, bits_v, 0, 33, 0)
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d)) * 2.0
    ke, ve = O.encode(kc, K), O.encode(vc, V)
    return kc, vc, K, (ke.idx, ke.qneg, ke.norm16, ke.rnorm16), (ve.idx, ve.norm16)


def test_attention_uniform_weights_give_the_mean_value():
    # a zero query (or scale 0) makes every logit equal: the output of every
    # query row is the plain mean of the reconstructed values
    rng = np.random.default_rng(40)
    kc, vc, K, ke, ve = _attn_inputs(rng, 32, 40)
    mean = O.dequantize(vc, *ve).mean(axis=0)
    o0 = O.attention_from_codes(kc, vc, np.zeros((3, 32)), ke, ve, 0.2)
    assert np.allclose(o0, mean[None, :], rtol=1e-12, atol=1e-12)
    Qv = rng.standard_normal((3, 32))
    o1 = O.attention_from_codes(kc, vc, Qv, ke, ve, 0.0)
    assert np.allclose(o1, mean[None, :], rtol=1e-12, atol=1e-12)


def test_attention_sharp_scale_selects_the_best_key():
    # with a large scale the softmax concentrates on the key of the largest
    # estimated logit: the output is that token's reconstructed value
    rng = np.random.default_rng(41)
    kc, vc, K, ke, ve = _attn_inputs(rng, 32, 40, bits_k=8, m=0)
    Qv = rng.standard_normal((4, 32))
    L = O.logits_from_codes(kc, Qv, ke[0], None, ke[2], None)
    o = O.attention_from_codes(kc, vc, Qv, ke, ve, 1e4)
    Vh = O.dequantize(vc, *ve)
    assert np.allclose(o, Vh[np.argmax(L, axis=1)], rtol=1e-9, atol=1e-9)
    # a query row's weights do not depend on the other rows
    o_single = O.attention_from_codes(kc, vc, Qv[2:3], ke, ve, 1e4)
    assert np.allclose(o_single[0], o[2], rtol=1e-12, atol=1e-12)


def test_attention_weights_sum_to_one_and_shift_invariant():
    # the output lies in the convex hull of the values: with all values equal
    # to one vector the output is that vector, for any query and scale
    rng = np.random.default_rng(42)
    kc, vc, K, ke, _ = _attn_inputs(rng, 16, 25)
    v = rng.standard_normal(16)
    ve = O.encode(vc, np.repeat(v[None, :], 25, axis=0))
    vh = O.dequantize(vc, ve.idx, ve.norm16)
    o = O.attention_from_codes(kc, vc, rng.standard_normal((5, 16)) * 3.0, ke, (ve.idx, ve.norm16), 0.7)
    assert np.allclose(o, vh[0][None, :], rtol=1e-12, atol=1e-12)


def test_attention_empty_context_is_zero():
    kc = O.make_codec(16, 3, 16, 31, 32)
    vc = O.make_codec(16, 3, 0, 33, 0)
    e = np.zeros((0, 16), dtype=np.int64)
    o = O.attention_from_codes(kc, vc, np.ones((2, 16)), (e, np.zeros((0, 16), bool), np.zeros(0), np.zeros(0)),
                               (e, np.zeros(0)), 0.25)
    assert o.shape == (2, 16) and not o.any()


def test_exact_top_k_against_brute_force_with_ties():
    rng = np.random.default_rng(61)
    S = rng.integers(0, 6, size=(20, 40)).astype(np.float64)   # many equal scores
    for k in (1, 3, 10, 40):
        got = O.exact_top_k(S, k)
        for row, g in zip(S, got):
            brute = [j for _, j in sorted((-row[j], j) for j in range(len(row)))][:k]
            assert list(g) == brute
    assert O.exact_top_k(S, 100).shape == (20, 40)


def test_recall_at_k():
    exact = np.array([[1, 2, 3, 4], [5, 6, 7, 8]])
    found = np.array([[4, 3, 9, 10], [5, 6, 7, 8]])
    assert O.recall_at_k(found, exact) == 0.75
    assert O.recall_at_k(exact, exact) == 1.0
