"""fp64 CPU oracle for the recursive polar form of stage 1 (test infrastructure only).

Same rules as ``tq_oracle``: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it; it shares no code with
``kv_cache_vector_rotate_b200`` and imports nothing from it.

Source: "TurboQuant explained" (a2a-mcp.org), §Stage 1, its PolarQuant
paragraph.  The vector is normalized; its coordinates are paired recursively
and every pair is turned from Cartesian into polar form; the radii carry the
magnitude and the angles the direction; the angles' laws are concentrated and
known in advance, which is why no per-block scale has to be stored.

The page gives only that outline.  READINGS taken here, each the plainest one
the rest of the page supports:

* P1 The transform acts on the rotated unit vector u = Pi x / ||x||: the
  random rotation of §Stage 1 comes first, and ||x|| is the fp16 side value,
  as in the scalar codec.
* P2 n = d is a power of two.  Level 1 pairs (u[2i], u[2i+1]); level l > 1
  pairs the radii of level l - 1 the same way.  The recursion ends with one
  radius, ||u|| = 1, which is not stored: n - 1 angles in all.
* P3 Level-1 angles are atan2(u[2i+1], u[2i]) in [-pi, pi]; deeper angles are
  atan2(rho[2i+1], rho[2i]) in [0, pi/2] (radii are never negative).
* P4 For u uniform on the sphere (what the rotation makes of any fixed x),
  level-1 angles are uniform on [-pi, pi], and a level-l angle, whose two
  radii each cover k = 2^(l-1) coordinates, has the density
  2 (sin phi cos phi)^(k-1) / B(k/2, k/2) on [0, pi/2] (sin^2 phi follows
  Beta(k/2, k/2)).  These laws fix every codebook in advance.
* P5 Every angle is coded with b bits by the Lloyd-Max quantizer of its
  level's law: the scalar codec's budget of b bits per coordinate, less one.
  A tie goes to the upper cell.  The angle tables are kept in float64.
* P6 Decoding runs the recursion backwards from radius 1 with the centroids
  in place of the angles.  The key is ||x|| Pi^T u_hat and its logit against
  a query q is ||x|| <Pi q, u_hat>; the zero vector decodes to zero.
* P7 Stage 2 (§Stage 2) applies unchanged on top: the residual
  r = u - Pi^T u_hat (original space) keeps the signs of S r and the fp16
  ||r||, and the logit gains ||x|| sqrt(pi/2)/m ||r|| <S q, sign(S r)>.

Parity status: every function here is pinned by ``tests/test_oracle_polar.py``
against closed forms, a library's Beta law and integrals, special vectors and
brute force.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from .tq_oracle import fp16, qjl_matrix, qjl_scale, rotation, unit_and_norm

# ---------------------------------------------------------------------------
# The recursive polar transform (P2, P3) and its inverse (P6).
# ---------------------------------------------------------------------------


def n_levels(n: int) -> int:
    """Levels of the recursion for n coordinates (n a power of two >= 2)."""
    if n < 2 or n & (n - 1):
        raise ValueError("the polar transform needs a power-of-two length >= 2")
    return n.bit_length() - 1


def polar_forward(U: np.ndarray) -> tuple[list[np.ndarray], np.ndarray]:
    """Rows of U [N, n] -> (angles, radius): angles[l - 1] is level l,
    shape [N, n / 2^l]; radius [N] is the last level's radius (= ||row||)."""
    rho = np.asarray(U, dtype=np.float64)
    n_levels(rho.shape[1])
    angles = []
    while rho.shape[1] > 1:
        a, b = rho[:, 0::2], rho[:, 1::2]
        angles.append(np.arctan2(b, a))
        rho = np.sqrt(a * a + b * b)
    return angles, rho[:, 0]


def polar_inverse(angles: list[np.ndarray], radius: np.ndarray) -> np.ndarray:
    """Inverse of ``polar_forward``: each level's radii split into
    (rho cos phi, rho sin phi), deepest level first."""
    rho = np.asarray(radius, dtype=np.float64)[:, None]
    for ang in reversed(angles):
        ang = np.asarray(ang, dtype=np.float64)
        out = np.empty((rho.shape[0], 2 * rho.shape[1]))
        out[:, 0::2] = rho * np.cos(ang)
        out[:, 1::2] = rho * np.sin(ang)
        rho = out
    return rho


# ---------------------------------------------------------------------------
# The angle laws (P4).
# ---------------------------------------------------------------------------


def angle_support(level: int) -> tuple[float, float]:
    if level < 1:
        raise ValueError("levels start at 1")
    return (-math.pi, math.pi) if level == 1 else (0.0, math.pi / 2.0)


def angle_density(level: int, phi) -> np.ndarray:
    """Normalized density of a level-`level` angle of a uniform unit vector."""
    phi = np.asarray(phi, dtype=np.float64)
    lo, hi = angle_support(level)
    inside = (phi >= lo) & (phi <= hi)
    if level == 1:
        return np.where(inside, 1.0 / (2.0 * math.pi), 0.0)
    k = 1 << (level - 1)
    # 2 / B(k/2, k/2) = 2 Gamma(k) / Gamma(k/2)^2
    log_c = math.log(2.0) + math.lgamma(k) - 2.0 * math.lgamma(k / 2.0)
    s = np.clip(np.sin(phi) * np.cos(phi), 0.0, None)
    return np.where(inside, np.exp(log_c) * np.power(s, k - 1), 0.0)


# ---------------------------------------------------------------------------
# Lloyd-Max quantizer of an angle law (P5).  The two optimality conditions
# (Lloyd 1957/1982, Max 1960): boundaries are midpoints of neighbouring
# centroids, centroids are the conditional means of their cells.  Lloyd's
# iteration alternates them from the equal-probability cells; every law here
# is log-concave on its support, so the fixed point is unique.  Cell moments
# by composite Gauss-Legendre quadrature (the densities are smooth on the
# support).
# ---------------------------------------------------------------------------

_GL_X, _GL_W = np.polynomial.legendre.leggauss(20)
_PANELS = 64


def _cell_moments(level: int, lo: np.ndarray, hi: np.ndarray) -> tuple[np.ndarray, ...]:
    """(P, M1, M2): integrals over [lo, hi] of f, phi f and phi^2 f per cell."""
    edges = lo[:, None] + (hi - lo)[:, None] * (np.arange(_PANELS + 1) / _PANELS)[None, :]
    mid = 0.5 * (edges[:, 1:] + edges[:, :-1])
    half = 0.5 * (edges[:, 1:] - edges[:, :-1])
    x = mid[:, :, None] + half[:, :, None] * _GL_X[None, None, :]
    fw = half[:, :, None] * _GL_W[None, None, :] * angle_density(level, x)
    return fw.sum(axis=(1, 2)), (fw * x).sum(axis=(1, 2)), (fw * x * x).sum(axis=(1, 2))


@dataclass
class AngleCodebook:
    level: int
    bits: int
    centroids: np.ndarray      # 2^b ascending
    boundaries: np.ndarray     # 2^b - 1 interior boundaries (midpoints)
    distortion: float          # E[(phi - c(phi))^2] under the level's law
    sweeps: int


def angle_lloyd_max(level: int, bits: int, tol: float = 1e-13, max_sweeps: int = 20000) -> AngleCodebook:
    if bits < 1:
        raise ValueError("bits >= 1")
    lo, hi = angle_support(level)
    K = 1 << bits
    grid = np.linspace(lo, hi, 200001)
    f = angle_density(level, grid)
    cdf = np.concatenate(([0.0], np.cumsum(0.5 * (f[1:] + f[:-1]) * np.diff(grid))))
    cdf /= cdf[-1]
    e = np.concatenate(([lo], np.interp(np.arange(1, K) / K, cdf, grid), [hi]))
    P, M1, _ = _cell_moments(level, e[:-1], e[1:])
    c = M1 / P
    sweeps = 0
    for sweeps in range(1, max_sweeps + 1):
        e = np.concatenate(([lo], 0.5 * (c[1:] + c[:-1]), [hi]))
        P, M1, _ = _cell_moments(level, e[:-1], e[1:])
        c_new = M1 / P
        step = float(np.max(np.abs(c_new - c)))
        c = c_new
        if step < tol:
            break
    # every law is symmetric about the middle of its support: make the
    # centroids exactly symmetric
    centre = 0.5 * (lo + hi)
    c = 0.5 * (c + (2.0 * centre - c[::-1]))
    t = 0.5 * (c[1:] + c[:-1])
    e = np.concatenate(([lo], t, [hi]))
    P, M1, M2 = _cell_moments(level, e[:-1], e[1:])
    D = float(np.sum(M2 - 2.0 * c * M1 + c * c * P))
    return AngleCodebook(level, bits, c, t, D, sweeps)


# ---------------------------------------------------------------------------
# The codec (P1, P5, P6).
# ---------------------------------------------------------------------------


@dataclass
class PolarCodec:
    d: int
    bits: int
    Pi: np.ndarray                 # d x d, the rotation of the scalar codec
    books: list[AngleCodebook]     # level 1 first
    m: int = 0                     # QJL rows (0: stage 1 only)
    S: np.ndarray | None = None    # m x d


def make_polar_codec(d: int, bits: int, seed_pi: int, m: int = 0, seed_s: int = 0) -> PolarCodec:
    L = n_levels(d)
    Pi, _, _ = rotation(d, seed_pi)
    S = qjl_matrix(m, d, seed_s) if m > 0 else None
    return PolarCodec(d, bits, Pi, [angle_lloyd_max(level, bits) for level in range(1, L + 1)], m, S)


@dataclass
class PolarEncoded:
    idx: list[np.ndarray]      # level l: [N, d / 2^l] int, 0 .. 2^b - 1
    norm16: np.ndarray         # [N] float16 ||x||
    angles: list[np.ndarray]   # the exact angles (for boundary windows)
    qneg: np.ndarray | None = None     # [N, m] bool, True where (S r)_i < 0
    rnorm16: np.ndarray | None = None  # [N] float16 ||r||


def quantize_angles(angles: list[np.ndarray], books: list[AngleCodebook]) -> list[np.ndarray]:
    """idx = number of interior boundaries t_i with t_i <= phi, per level."""
    return [np.sum(a[..., None] >= book.boundaries, axis=-1) for a, book in zip(angles, books)]


def polar_encode(codec: PolarCodec, X: np.ndarray) -> PolarEncoded:
    U, n = unit_and_norm(X)
    angles, _ = polar_forward(U @ codec.Pi.T)
    idx = quantize_angles(angles, codec.books)
    enc = PolarEncoded(idx, fp16(n), angles)
    if codec.m > 0:
        R = U - polar_decode_unit(codec, idx) @ codec.Pi     # residual, original space (P7)
        enc.qneg = (R @ codec.S.T) < 0.0
        enc.rnorm16 = fp16(np.sqrt(np.sum(R * R, axis=1)))
    return enc


def polar_decode_unit(codec: PolarCodec, idx: list[np.ndarray]) -> np.ndarray:
    """u_hat in the rotated space: the inverse recursion from radius 1."""
    angles = [book.centroids[i] for book, i in zip(codec.books, idx)]
    return polar_inverse(angles, np.ones(idx[0].shape[0]))


def polar_decode(codec: PolarCodec, enc: PolarEncoded) -> np.ndarray:
    """x_hat = ||x|| Pi^T u_hat, rows."""
    return enc.norm16.astype(np.float64)[:, None] * (polar_decode_unit(codec, enc.idx) @ codec.Pi)


def polar_logits(codec: PolarCodec, Qv: np.ndarray, enc: PolarEncoded) -> np.ndarray:
    """[n_queries, N]: ||x|| (<Pi q, u_hat> + sqrt(pi/2)/m ||r|| <S q, sign(S r)>),
    the query rotated (and sketched) once; the second term only when m > 0."""
    Qv = np.asarray(Qv, dtype=np.float64)
    out = (Qv @ codec.Pi.T) @ polar_decode_unit(codec, enc.idx).T
    if codec.m > 0:
        signs = np.where(enc.qneg, -1.0, 1.0)
        out = out + qjl_scale(codec.m) * enc.rnorm16.astype(np.float64)[None, :] * ((Qv @ codec.S.T) @ signs.T)
    return out * enc.norm16.astype(np.float64)[None, :]
