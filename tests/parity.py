"""Helpers shared by the GPU parity tests: oracle-side page construction and
the comparison rules for codes, logits and values.

Tolerances (stated once, used everywhere):
  * level indices and sign bits are bit-exact, except for a coordinate whose
    rotated unit value lies within 1e-5 of a cell boundary, or a projection
    (S r)_i within 1e-5 of zero; all mismatches together must stay below
    1e-4 of the symbols compared;
  * a token whose indices differ inside a boundary window has its signs and
    ||r|| checked for validity against the GPU's own (equally valid) indices;
  * fp16 side values (||x||, ||r||) differ by at most one fp16 unit in the
    last place (the GPU rounds an fp32 value, the oracle a float64 one);
  * logits from identical codes: |L_gpu - L| / max(|L|, ||q|| ||k|| / sqrt(d))
    <= 1e-3;
  * values: |v_gpu - v| <= 1e-3 max(||v||_inf, natural scale).
"""

from __future__ import annotations

import numpy as np

from oracle import tq_oracle as O

WINDOW = 1e-5
MISMATCH_RATE = 1e-4
LOGIT_TOL = 1e-3
VALUE_TOL = 1e-3


def fp16_ulp(x: np.ndarray) -> np.ndarray:
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -14)))
    return 2.0 ** (e - 10)


def oracle_pages(lay: O.Layout, n_pages: int, block_table: np.ndarray, encs: dict) -> np.ndarray:
    """Byte image of a cache holding the oracle's records.
    encs[(b, h)] = (positions, Encoded)."""
    pages = np.zeros(n_pages * lay.page_bytes, dtype=np.uint8)
    for (b, h), (pos, enc) in encs.items():
        if len(pos):                           # an empty sequence has no records
            O.write_pages(lay, pages, block_table, b, h, pos, enc.idx, enc.qneg, enc.norm16, enc.rnorm16)
    return pages


def compare_codes(codec: O.Codec, X: np.ndarray, ora: O.Encoded, idx, qneg, n16, r16) -> dict:
    """Checks GPU codes of the rows X against the oracle's; returns statistics."""
    N, d = ora.idx.shape
    t = codec.cb.boundaries
    near_b = np.min(np.abs(ora.y[..., None] - t[None, None, :]), axis=-1) < WINDOW
    imis = idx != ora.idx
    assert not np.any(imis & ~near_b), "index mismatch outside the boundary window"
    # a differing index must be the neighbouring cell
    assert np.all(np.abs(idx[imis] - ora.idx[imis]) == 1)
    n_sym = N * d
    n_bad = int(imis.sum())
    # norms within one fp16 ulp
    dn = np.abs(n16.astype(np.float64) - ora.norm16.astype(np.float64))
    assert np.all(dn <= fp16_ulp(ora.norm16) + 1e-30), "||x|| differs by more than 1 ulp"
    stats = {"idx_mismatch": n_bad, "near_boundary": int(near_b.sum())}
    if codec.m > 0:
        same = ~imis.any(axis=1)
        near_s = np.abs(ora.proj) < WINDOW
        smis = (qneg != ora.qneg) & same[:, None]
        assert not np.any(smis & ~near_s), "QJL sign mismatch outside the zero window"
        dr = np.abs(r16.astype(np.float64) - ora.rnorm16.astype(np.float64))
        assert np.all((dr <= fp16_ulp(ora.rnorm16) + 1e-30)[same]), "||r|| differs by more than 1 ulp"
        n_sym += N * codec.m
        n_bad += int(smis.sum())
        flipped = np.nonzero(~same)[0]
        if len(flipped):
            U, _ = O.unit_and_norm(X[flipped])
            proj, qn, rn = O.qjl_sketch(codec, U, idx[flipped])
            vmis = (qneg[flipped] != qn) & (np.abs(proj) >= WINDOW)
            assert not np.any(vmis), "signs of a re-coded token are not those of its indices"
            dr = np.abs(r16[flipped].astype(np.float64) - rn.astype(np.float64))
            assert np.all(dr <= fp16_ulp(rn) + 1e-30)
            n_bad += int((qneg[flipped] != ora.qneg[flipped]).sum())
        stats["sign_mismatch"] = int(smis.sum())
        stats["recoded_tokens"] = int(len(flipped))
    stats["rate"] = n_bad / n_sym
    assert stats["rate"] <= MISMATCH_RATE, stats
    return stats


def logit_error(L_gpu: np.ndarray, L_ora: np.ndarray, qnorm: np.ndarray, knorm16: np.ndarray, d: int) -> float:
    """max |L_gpu - L| / max(|L|, ||q|| ||k|| / sqrt(d)) over all pairs."""
    scale = np.maximum(np.abs(L_ora), qnorm[:, None] * knorm16.astype(np.float64)[None, :] / np.sqrt(d))
    diff = np.abs(L_gpu.astype(np.float64) - L_ora)
    ok = scale > 0
    assert np.all(diff[~ok] == 0)
    return float(np.max(diff[ok] / scale[ok])) if ok.any() else 0.0
