"""fp64 CPU oracle for the TurboQuant KV-cache codec (test infrastructure only).

This module is the slow, plain reference that the CUDA library is checked
against.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it; the product path never does.  It shares no code
with ``kv_cache_vector_rotate_b200`` and imports nothing from it.

Source of the method ("TQ" below): the web page "TurboQuant 설명: 무엇인지와
LLM 메모리 6배 절약 구현 방법" (TurboQuant explained: what it is and how to
implement 6x LLM memory savings), a2a-mcp.org.  Sections cited:

* TQ §Key summary -- online, data-oblivious vector quantization of the KV
  cache; random orthogonal rotation, a Lloyd-Max stage and a 1-bit QJL stage.
* TQ §Stage 1 (random rotation + PolarQuant) -- the rotation is the Q factor of
  a QR decomposition of a Gaussian matrix; after it every coordinate of a unit
  vector follows Beta((d-1)/2, (d-1)/2) on [-1, 1]; an MSE-optimal Lloyd-Max
  quantizer for that law maps each coordinate to a few bits; the vector is
  normalized first.
* TQ §Stage 2 (QJL residual correction) -- the residual left by stage 1 is
  sketched by the signs of a Gaussian (Johnson-Lindenstrauss) projection,
  which removes the inner-product bias.
* TQ §How it works / §How to implement -- attention logits are computed
  straight from the indices with the query rotated once, with no full
  dequantization.

Everything is float64 numpy.  The library routines used as single steps are
``numpy.linalg.qr`` (Householder QR), ``numpy.polynomial.legendre.leggauss``
(quadrature nodes) and matrix products.  Readings of points the page leaves
open are marked READING where they are taken.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against published values, closed forms, textbook special cases or brute force.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# ---------------------------------------------------------------------------
# Random numbers: SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) used as a
# counter-based generator, and the Box-Muller transform (Box & Muller 1958).
# READING: the page says only "Gaussian matrix"; the seeded generator is ours.
# ---------------------------------------------------------------------------

_GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Outputs number start..start+n-1 of SplitMix64 seeded with ``seed``.

    Output i is mix(seed + (i + 1) * gamma): the state after i + 1 steps of
    the published generator, so the stream can be cut anywhere.
    """
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GOLDEN_GAMMA
        z = (z ^ (z >> np.uint64(30))) * _MIX1
        z = (z ^ (z >> np.uint64(27))) * _MIX2
    return z ^ (z >> np.uint64(31))


def uniforms(seed: int, n: int) -> np.ndarray:
    """n doubles in [0, 1): the top 53 bits of each SplitMix64 output."""
    return (splitmix64(seed, n) >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def gaussians(seed: int, n: int) -> np.ndarray:
    """n standard normal doubles by Box-Muller on consecutive uniform pairs.

    Pair k uses uniforms (2k, 2k+1): rho = sqrt(-2 ln(1 - u_2k)),
    z_2k = rho cos(2 pi u_2k+1), z_2k+1 = rho sin(2 pi u_2k+1).
    """
    n_pairs = (n + 1) // 2
    u = uniforms(seed, 2 * n_pairs).reshape(n_pairs, 2)
    rho = np.sqrt(-2.0 * np.log1p(-u[:, 0]))
    ang = 2.0 * np.pi * u[:, 1]
    z = np.empty((n_pairs, 2))
    z[:, 0] = rho * np.cos(ang)
    z[:, 1] = rho * np.sin(ang)
    return z.reshape(-1)[:n]


def gaussian_matrix(seed: int, rows: int, cols: int) -> np.ndarray:
    """rows x cols matrix filled row-major from ``gaussians(seed, rows*cols)``."""
    return gaussians(seed, rows * cols).reshape(rows, cols)


# ---------------------------------------------------------------------------
# TQ §Stage 1: random orthogonal rotation from the QR of a Gaussian matrix.
# READING: Pi is the Q factor with the column signs fixed so that diag(R) > 0
# (this makes Q unique and Haar distributed); a vector is rotated as y = Pi x.
# ---------------------------------------------------------------------------


def rotation(d: int, seed_pi: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Returns (Pi, R, G) with G = Pi R, Pi orthogonal, diag(R) > 0."""
    G = gaussian_matrix(seed_pi, d, d)
    Q, R = np.linalg.qr(G)
    s = np.where(np.diag(R) < 0.0, -1.0, 1.0)
    return Q * s[None, :], R * s[:, None], G


def qjl_matrix(m: int, d: int, seed_s: int) -> np.ndarray:
    """TQ §Stage 2: the m x d Gaussian projection S of the QJL sketch."""
    return gaussian_matrix(seed_s, m, d)


# ---------------------------------------------------------------------------
# TQ §Stage 1: the coordinate law Beta((d-1)/2, (d-1)/2) on [-1, 1],
# density f(t) = C_d (1 - t^2)^((d-3)/2), C_d = Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)).
# Moments over a cell are integrated numerically in theta = asin(t), where the
# integrand C_d cos^(d-2)(theta) is smooth for every d >= 2 (for d = 2 the
# t-density is singular at +-1).  Composite Gauss-Legendre: 64 panels x 20 nodes.
# ---------------------------------------------------------------------------

_GL_X, _GL_W = np.polynomial.legendre.leggauss(20)
_PANELS = 64


def density_const(d: int) -> float:
    return math.exp(math.lgamma(d / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2.0))


def coord_density(t: np.ndarray, d: int) -> np.ndarray:
    """Normalized density of one coordinate of a uniform unit vector in R^d."""
    t = np.asarray(t, dtype=np.float64)
    return density_const(d) * np.power(np.clip(1.0 - t * t, 0.0, None), (d - 3) / 2.0)


def cell_moments(lo: np.ndarray, hi: np.ndarray, d: int) -> tuple[np.ndarray, ...]:
    """(P, M1, M2): integral over [lo, hi] of f, t f and t^2 f (vectorised over cells)."""
    a = np.arcsin(np.clip(np.asarray(lo, np.float64), -1.0, 1.0))
    b = np.arcsin(np.clip(np.asarray(hi, np.float64), -1.0, 1.0))
    edges = a[:, None] + (b - a)[:, None] * (np.arange(_PANELS + 1) / _PANELS)[None, :]
    mid = 0.5 * (edges[:, 1:] + edges[:, :-1])
    half = 0.5 * (edges[:, 1:] - edges[:, :-1])
    th = mid[:, :, None] + half[:, :, None] * _GL_X[None, None, :]
    w = half[:, :, None] * _GL_W[None, None, :]
    base = w * np.power(np.cos(th), d - 2)
    s = np.sin(th)
    c = density_const(d)
    P = c * base.sum(axis=(1, 2))
    M1 = c * (base * s).sum(axis=(1, 2))
    M2 = c * (base * s * s).sum(axis=(1, 2))
    return P, M1, M2


# ---------------------------------------------------------------------------
# TQ §Stage 1: Lloyd-Max quantizer for the coordinate law.  The MSE-optimal
# scalar quantizer satisfies two conditions (Lloyd 1957/1982, Max 1960):
# each boundary is the midpoint of its neighbouring centroids and each
# centroid is the conditional mean of its cell.  Lloyd's iteration alternates
# the two.  For many levels its linear convergence is slow, so once it has run
# ``lloyd_iters`` sweeps the same two conditions are finished by Newton's
# method on the centroid equations (tridiagonal Jacobian); the fixed point is
# unique for this log-concave density, so the answer does not depend on that
# switch.  READING: the page gives no initialisation or stopping rule.
# ---------------------------------------------------------------------------


@dataclass
class Codebook:
    d: int
    bits: int
    centroids: np.ndarray      # 2^b ascending, exactly antisymmetric
    boundaries: np.ndarray     # 2^b - 1 interior boundaries (midpoints)
    distortion: float          # per-coordinate MSE E[(T - c(T))^2]
    lloyd_sweeps: int
    newton_steps: int


def _midpoints(c: np.ndarray) -> np.ndarray:
    return 0.5 * (c[1:] + c[:-1])


def _edges(c: np.ndarray) -> np.ndarray:
    return np.concatenate(([-1.0], _midpoints(c), [1.0]))


def _equiprobable_start(d: int, K: int) -> np.ndarray:
    """Means of the K equal-probability cells (a start point for the iteration)."""
    th = np.linspace(-np.pi / 2, np.pi / 2, 200001)
    g = np.power(np.cos(th), d - 2)
    cdf = np.concatenate(([0.0], np.cumsum(0.5 * (g[1:] + g[:-1]) * np.diff(th))))
    cdf /= cdf[-1]
    q = np.interp(np.arange(1, K) / K, cdf, th)
    e = np.concatenate(([-1.0], np.sin(q), [1.0]))
    P, M1, _ = cell_moments(e[:-1], e[1:], d)
    return M1 / P


def lloyd_max(d: int, bits: int, tol: float = 1e-15, lloyd_iters: int = 200,
              newton_iters: int = 60) -> Codebook:
    if d < 2 or bits < 1:
        raise ValueError("need d >= 2 and bits >= 1")
    K = 1 << bits
    c = _equiprobable_start(d, K)
    sweeps = 0
    for sweeps in range(1, lloyd_iters + 1):
        e = _edges(c)
        P, M1, _ = cell_moments(e[:-1], e[1:], d)
        c_new = M1 / P
        step = np.max(np.abs(c_new - c))
        c = c_new
        if step < tol:
            break
    newton = 0
    e = _edges(c)
    P, M1, _ = cell_moments(e[:-1], e[1:], d)
    resid = c - M1 / P
    while np.max(np.abs(resid)) >= tol and newton < newton_iters:
        newton += 1
        mu = M1 / P
        with np.errstate(divide="ignore"):      # the end points +-1 are fixed
            f_lo = coord_density(e[:-1], d)
            f_hi = coord_density(e[1:], d)
        f_lo[0] = 0.0          # t_0 = -1 is fixed
        f_hi[-1] = 0.0         # t_K = +1 is fixed
        d_lo = f_lo * (mu - e[:-1]) / P    # d mu_i / d t_i
        d_hi = f_hi * (e[1:] - mu) / P     # d mu_i / d t_{i+1}
        J = np.eye(K)
        idx = np.arange(K)
        J[idx, idx] -= 0.5 * (d_lo + d_hi)
        J[idx[1:], idx[:-1]] -= 0.5 * d_lo[1:]
        J[idx[:-1], idx[1:]] -= 0.5 * d_hi[:-1]
        c = c - np.linalg.solve(J, resid)
        e = _edges(c)
        P, M1, _ = cell_moments(e[:-1], e[1:], d)
        resid = c - M1 / P
    # The law is symmetric, so the optimum is antisymmetric: make it exactly so.
    c = 0.5 * (c - c[::-1])
    t = _midpoints(c)
    if K % 2 == 0:
        t[K // 2 - 1] = 0.0
    e = np.concatenate(([-1.0], t, [1.0]))
    P, M1, M2 = cell_moments(e[:-1], e[1:], d)
    D = float(np.sum(M2 - 2.0 * c * M1 + c * c * P))
    return Codebook(d, bits, c, t, D, sweeps, newton)


def fp16(x) -> np.ndarray:
    """Round to IEEE binary16, nearest-even, directly from float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16)


def reconstruction_levels(c: np.ndarray) -> tuple[np.ndarray, int | None]:
    """The reconstruction levels of a Lloyd-Max codebook.

    READING (TQ §Stage 1 gives the centroids as real numbers, not how they
    are stored): a codebook of at most 8 levels (b <= 3) keeps its levels in
    8-bit fixed point on one power-of-two scale -- every centroid rounded
    (half to even) to an integer multiple of 2^-f, f the largest integer with
    max|c| 2^f <= 127 -- so that a decoded coordinate is one signed byte; the
    levels are then exact in fp16 and fp32 too, and the rounding moves each
    by at most 2^-(f+1) (about 0.1 % more distortion at b = 3, d = 128; pinned
    in tests/test_oracle_codec.py).  Larger codebooks keep their levels in
    fp16 (8 bits would merge neighbouring levels).  Returns (levels, f), with
    f = None for fp16 levels.  The boundaries stay the float64 midpoints of
    the unrounded centroids."""
    c = np.asarray(c, dtype=np.float64)
    if len(c) > 8:
        return fp16(c).astype(np.float64), None
    f = int(math.floor(math.log2(127.0 / float(np.max(np.abs(c))))))
    return np.round(c * 2.0 ** f) / 2.0 ** f, f


# ---------------------------------------------------------------------------
# The codec.  TQ §Stage 1: normalize, rotate, quantize each coordinate.
# TQ §Stage 2: 1-bit signs of a Gaussian projection of the residual.
# READINGS:
#  * the norm ||x|| and the residual norm ||r|| are side values stored as fp16;
#  * reconstruction uses the levels crec = reconstruction_levels(c) (also in
#    the residual), the boundaries stay float64;
#  * a tie y == t_i goes to the upper cell; sign(0) = +1;
#  * the zero vector is quantized as u = 0 (every index is the cell holding 0);
#  * the QJL sketch keeps one sign per projection row (m bits per key).
# ---------------------------------------------------------------------------


@dataclass
class Codec:
    d: int
    bits: int
    m: int
    Pi: np.ndarray          # d x d
    S: np.ndarray | None    # m x d, None for MSE-only (values)
    cb: Codebook

    @property
    def crec(self) -> np.ndarray:
        return reconstruction_levels(self.cb.centroids)[0]


def make_codec(d: int, bits: int, m: int, seed_pi: int, seed_s: int) -> Codec:
    Pi, _, _ = rotation(d, seed_pi)
    S = qjl_matrix(m, d, seed_s) if m > 0 else None
    return Codec(d, bits, m, Pi, S, lloyd_max(d, bits))


@dataclass
class Encoded:
    idx: np.ndarray          # [N, d] int, level index 0..2^b-1
    qneg: np.ndarray | None  # [N, m] bool, True where (S r)_i < 0
    norm16: np.ndarray       # [N] float16, ||x||
    rnorm16: np.ndarray | None  # [N] float16, ||r||
    y: np.ndarray            # [N, d] rotated unit coordinates (for windows)
    proj: np.ndarray | None  # [N, m] S r (for windows)


def unit_and_norm(X: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    X = np.asarray(X, dtype=np.float64)
    n = np.sqrt(np.sum(X * X, axis=1))
    safe = np.where(n > 0.0, n, 1.0)
    U = np.where(n[:, None] > 0.0, X / safe[:, None], 0.0)
    return U, n


def quantize_indices(Y: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """idx_j = number of interior boundaries t_i with t_i <= y_j."""
    return np.sum(Y[..., None] >= boundaries[None, None, :], axis=-1)


def qjl_sketch(codec: Codec, U: np.ndarray, idx: np.ndarray):
    """TQ §Stage 2 for unit rows U coded by idx: (S r, r < 0 bits, fp16 ||r||)
    with the residual r = u - Pi^T crec[idx] taken in the original space."""
    R = U - codec.crec[idx] @ codec.Pi
    proj = R @ codec.S.T
    return proj, proj < 0.0, fp16(np.sqrt(np.sum(R * R, axis=1)))


def encode(codec: Codec, X: np.ndarray) -> Encoded:
    U, n = unit_and_norm(X)
    Y = U @ codec.Pi.T
    idx = quantize_indices(Y, codec.cb.boundaries)
    qneg = rnorm16 = proj = None
    if codec.m > 0:
        proj, qneg, rnorm16 = qjl_sketch(codec, U, idx)
    return Encoded(idx, qneg, fp16(n), rnorm16, Y, proj)


def qjl_scale(m: int) -> float:
    return math.sqrt(math.pi / 2.0) / m


def logits_from_codes(codec: Codec, Qv: np.ndarray, idx: np.ndarray, qneg: np.ndarray,
                      norm16: np.ndarray, rnorm16: np.ndarray) -> np.ndarray:
    """Estimated <q, k> for every (query, key) pair, float64.

    L = ||k|| ( sum_j (Pi q)_j crec[idx_j]
                + sqrt(pi/2)/m ||r|| sum_i (S q)_i sign_i )
    with sign_i = -1 where the stored QJL bit says (S r)_i < 0, else +1.
    """
    Qv = np.asarray(Qv, dtype=np.float64)
    q_rot = Qv @ codec.Pi.T                       # [nq, d]
    mse = q_rot @ codec.crec[idx].T                # [nq, N]
    out = mse
    if codec.m > 0:
        q_s = Qv @ codec.S.T                      # [nq, m]
        signs = np.where(qneg, -1.0, 1.0)         # [N, m]
        qjl = q_s @ signs.T                       # [nq, N]
        out = mse + qjl_scale(codec.m) * rnorm16.astype(np.float64)[None, :] * qjl
    return norm16.astype(np.float64)[None, :] * out


def dequantize(codec: Codec, idx: np.ndarray, norm16: np.ndarray) -> np.ndarray:
    """v_hat = ||v|| Pi^T crec[idx]  (MSE reconstruction, one row per token)."""
    return norm16.astype(np.float64)[:, None] * (codec.crec[idx] @ codec.Pi)


def weighted_values(codec: Codec, W: np.ndarray, idx: np.ndarray, norm16: np.ndarray) -> np.ndarray:
    """o_h = sum_t W[h, t] v_hat_t for every row h of W."""
    return np.asarray(W, dtype=np.float64) @ dequantize(codec, idx, norm16)


def attention_from_codes(kcodec: Codec, vcodec: Codec, Qv: np.ndarray, kenc, venc,
                         scale: float) -> np.ndarray:
    """Decode attention from the codes (TQ §How it works: attention logits
    from the compressed keys, values from their codes), written out as its
    definition: o_h = sum_t softmax_t(scale * L[h, t]) v_hat_t with L the
    estimated logits of ``logits_from_codes`` and v_hat the reconstruction of
    ``dequantize``.  READING: the softmax is the standard one over the valid
    positions (the page names attention, not its normalization); an empty
    context gives a zero row.  ``kenc`` / ``venc`` are (idx, qneg, norm16,
    rnorm16) / (idx, norm16) of the same tokens."""
    Qv = np.asarray(Qv, dtype=np.float64)
    idx, qneg, n16, r16 = kenc
    vidx, vn16 = venc
    if len(idx) == 0:
        return np.zeros((Qv.shape[0], vcodec.d))
    L = scale * logits_from_codes(kcodec, Qv, idx, qneg, n16, r16)   # [nq, N]
    L = L - L.max(axis=1, keepdims=True)
    P = np.exp(L)
    P /= P.sum(axis=1, keepdims=True)
    return weighted_values(vcodec, P, vidx, vn16)


def exact_logits(Qv: np.ndarray, K: np.ndarray) -> np.ndarray:
    """Brute force <q, k> in float64."""
    return np.asarray(Qv, np.float64) @ np.asarray(K, np.float64).T


def exact_top_k(scores: np.ndarray, k: int) -> np.ndarray:
    """[rows, k] column indices of the k largest scores of each row, best
    first; equal scores go to the lower index.  READING: the page names no
    tie rule for nearest-neighbour search."""
    scores = np.asarray(scores, dtype=np.float64)
    cols = np.arange(scores.shape[1])
    # lexsort sorts by the last key first: score descending, then index ascending
    order = np.array([np.lexsort((cols, -row))[:k] for row in scores], dtype=np.int64)
    return order.reshape(scores.shape[0], min(k, scores.shape[1]))


def recall_at_k(found: np.ndarray, exact: np.ndarray) -> float:
    """Mean over rows of |found_row & exact_row| / k (TQ §Benchmarks, recall@k)."""
    return float(np.mean([len(set(a.tolist()) & set(b.tolist())) / len(b) for a, b in zip(found, exact)]))


# ---------------------------------------------------------------------------
# Packed record layout, version 3 (the byte format the CUDA library reads and
# writes; written here from its specification, independently of the library).
#
# d_pad = 64 ceil(d/64), m_pad = 64 ceil(m/64); E = d_pad/4, F = m_pad/4.
# Coordinate j lives in chunk t = j // E at local position l = j % E;
# projection i lives in chunk t = i // F at local position l = i % F.
# Words of one chunk (32-bit little endian): index words, then ceil(F/32) QJL
# words (bit = 1 where (S r)_i < 0).  Stored code of an element: its level
# index for b <= 3; for b = 4 the sign-magnitude nibble neg << 3 | mu (with
# H = 8: idx >= H -> neg 0, mu = idx - H; idx < H -> neg 1, mu = H - 1 - idx).
# Bit k of the code of local element l lives at (index word, bit):
#   b = 1 : (l//32, 4 (l%8) + (l%32)//8)                       ceil(E/32) words
#   b = 2 : (l//16, 4 (l%8) + 2 ((l%16)//8) + k)               E/16 words
#   b = 3 : 32-element groups of 3 words; with g = l//32, l' = l%32:
#           l' < 24 -> (3g + l'//8, 4 (l'%8) + k);
#           l' >= 24 -> (3g + k, 4 (l' - 24) + 3);
#           a last group of 16 (E % 32 == 16) takes 2 words:
#           (3 (E//32) + l'//8, 4 (l'%8) + k)
#   b = 4 : (l//8, 4 ((l%8)//2 + 4 (l%2)) + k)                E/8 words
#   QJL   : row l at (l//32, 8 (l%4) + (l%32)//4) of the QJL words
# Padding coordinates and projections store code 0 and sign bit 0.
# A record is the 4 chunks back to back (CB = 16 W bytes).  A page holds P
# tokens for each of n_kv_heads heads; a head block is P records followed by P
# norm slots (fp16 ||x|| then, when m > 0, fp16 ||r||), padded to 16 bytes.
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Layout:
    d: int
    bits: int
    m: int
    page_tokens: int
    n_kv_heads: int

    @property
    def d_pad(self) -> int:
        return 64 * ((self.d + 63) // 64)

    @property
    def m_pad(self) -> int:
        return 64 * ((self.m + 63) // 64)

    @property
    def E(self) -> int:
        return self.d_pad // 4

    @property
    def F(self) -> int:
        return self.m_pad // 4

    @property
    def n_idx(self) -> int:
        E = self.E
        return {1: (E + 31) // 32, 2: E // 16, 3: 3 * (E // 32) + 2 * ((E % 32) // 16), 4: E // 8}[self.bits]

    @property
    def n_qjl(self) -> int:
        return (self.F + 31) // 32

    @property
    def words(self) -> int:
        return self.n_idx + self.n_qjl

    @property
    def code_bytes(self) -> int:
        return 16 * self.words

    @property
    def norm_bytes(self) -> int:
        return 4 if self.m > 0 else 2

    @property
    def head_block_bytes(self) -> int:
        raw = self.page_tokens * (self.code_bytes + self.norm_bytes)
        return 16 * ((raw + 15) // 16)

    @property
    def page_bytes(self) -> int:
        return self.n_kv_heads * self.head_block_bytes


def code_bit_position(lay: Layout, l: int, k: int) -> tuple[int, int]:
    """(index word, bit) of bit k of the stored code of local element l."""
    E, b = lay.E, lay.bits
    if b == 1:
        return l // 32, 4 * (l % 8) + (l % 32) // 8
    if b == 2:
        return l // 16, 4 * (l % 8) + 2 * ((l % 16) // 8) + k
    if b == 3:
        g, lp = divmod(l, 32)
        if g < E // 32:
            if lp < 24:
                return 3 * g + lp // 8, 4 * (lp % 8) + k
            return 3 * g + k, 4 * (lp - 24) + 3
        return 3 * (E // 32) + lp // 8, 4 * (lp % 8) + k
    return l // 8, 4 * ((l % 8) // 2 + 4 * (l % 2)) + k


def qjl_bit_position(l: int) -> tuple[int, int]:
    """(QJL word, bit) of local projection row l."""
    return l // 32, 8 * (l % 4) + (l % 32) // 4


def _stored_code(idx: np.ndarray, bits: int) -> np.ndarray:
    if bits < 4:
        return idx.astype(np.uint64)
    H = 8
    neg = idx < H
    mu = np.where(neg, H - 1 - idx, idx - H)
    return ((neg.astype(np.uint64) << np.uint64(3)) | mu.astype(np.uint64))


def _level_index(code: np.ndarray, bits: int) -> np.ndarray:
    code = code.astype(np.int64)
    if bits < 4:
        return code
    neg, mu = code >> 3, code & 7
    return np.where(neg == 1, 7 - mu, 8 + mu)


def pack_codes(lay: Layout, idx: np.ndarray, qneg: np.ndarray | None) -> np.ndarray:
    """[N, d] indices (+ [N, m] QJL bits) -> [N, 4, W] uint32 words."""
    N = idx.shape[0]
    full = np.zeros((N, lay.d_pad), dtype=np.int64)
    full[:, :lay.d] = idx
    code = _stored_code(full, lay.bits)
    code[:, lay.d:] = 0                       # padding stores code 0
    words = np.zeros((N, 4, lay.words), dtype=np.uint64)
    one = np.uint64(1)
    for j in range(lay.d_pad):
        t, l = divmod(j, lay.E)
        for k in range(lay.bits):
            w, p = code_bit_position(lay, l, k)
            words[:, t, w] |= ((code[:, j] >> np.uint64(k)) & one) << np.uint64(p)
    if lay.m > 0:
        for i in range(lay.m):
            t, l = divmod(i, lay.F)
            w, p = qjl_bit_position(l)
            words[:, t, lay.n_idx + w] |= qneg[:, i].astype(np.uint64) << np.uint64(p)
    return words.astype(np.uint32)


def unpack_codes(lay: Layout, words: np.ndarray) -> tuple[np.ndarray, np.ndarray | None]:
    """Inverse of ``pack_codes``: [N, 4, W] uint32 -> ([N, d] idx, [N, m] qneg)."""
    w64 = words.astype(np.uint64)
    N = w64.shape[0]
    one = np.uint64(1)
    code = np.zeros((N, lay.d), dtype=np.uint64)
    for j in range(lay.d):
        t, l = divmod(j, lay.E)
        for k in range(lay.bits):
            w, p = code_bit_position(lay, l, k)
            code[:, j] |= ((w64[:, t, w] >> np.uint64(p)) & one) << np.uint64(k)
    idx = _level_index(code, lay.bits)
    qneg = None
    if lay.m > 0:
        qneg = np.zeros((N, lay.m), dtype=bool)
        for i in range(lay.m):
            t, l = divmod(i, lay.F)
            w, p = qjl_bit_position(l)
            qneg[:, i] = ((w64[:, t, lay.n_idx + w] >> np.uint64(p)) & one) == one
    return idx, qneg


def token_offsets(lay: Layout, block_table: np.ndarray, b: int, h: int, pos: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Byte offsets (record, norm slot) of tokens ``pos`` of sequence b, head h."""
    pos = np.asarray(pos, dtype=np.int64)
    page = block_table[b, pos // lay.page_tokens].astype(np.int64)
    slot = pos % lay.page_tokens
    head = page * lay.page_bytes + h * lay.head_block_bytes
    rec = head + slot * lay.code_bytes
    nrm = head + lay.page_tokens * lay.code_bytes + slot * lay.norm_bytes
    return rec, nrm


def write_pages(lay: Layout, pages: np.ndarray, block_table: np.ndarray, b: int, h: int,
                pos: np.ndarray, enc_idx: np.ndarray, enc_qneg: np.ndarray | None,
                norm16: np.ndarray, rnorm16: np.ndarray | None) -> None:
    """Stores the records of tokens ``pos`` (one row each) into the byte array ``pages``."""
    words = pack_codes(lay, enc_idx, enc_qneg).reshape(len(pos), -1)
    raw = words.view(np.uint8).reshape(len(pos), lay.code_bytes)
    rec, nrm = token_offsets(lay, block_table, b, h, pos)
    cols = np.arange(lay.code_bytes)
    pages[rec[:, None] + cols[None, :]] = raw
    nb = norm16.astype(np.float16).view(np.uint8).reshape(-1, 2)
    pages[nrm[:, None] + np.arange(2)[None, :]] = nb
    if lay.m > 0:
        rb = rnorm16.astype(np.float16).view(np.uint8).reshape(-1, 2)
        pages[nrm[:, None] + 2 + np.arange(2)[None, :]] = rb


def read_pages(lay: Layout, pages: np.ndarray, block_table: np.ndarray, b: int, h: int,
               pos: np.ndarray):
    """Reads tokens ``pos`` back: (idx, qneg, norm16, rnorm16)."""
    rec, nrm = token_offsets(lay, block_table, b, h, pos)
    raw = pages[rec[:, None] + np.arange(lay.code_bytes)[None, :]]
    words = np.ascontiguousarray(raw).view(np.uint32).reshape(len(pos), 4, lay.words)
    idx, qneg = unpack_codes(lay, words)
    n16 = np.ascontiguousarray(pages[nrm[:, None] + np.arange(2)[None, :]]).view(np.float16).reshape(-1)
    r16 = None
    if lay.m > 0:
        r16 = np.ascontiguousarray(pages[nrm[:, None] + 2 + np.arange(2)[None, :]]).view(np.float16).reshape(-1)
    return idx, qneg, n16, r16
