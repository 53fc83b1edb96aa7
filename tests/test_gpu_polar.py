"""GPU parity of the recursive polar form (tq_polar_encode, tq_polar_logits)
against oracle/polar_oracle.py.

The records are unpacked here from their documented layout (include/tq.h):
angle codes, sign bits, fp16 norms.  Checked:
  * ||x|| within one fp16 ulp of the oracle's;
  * angle indices equal to the oracle's except where the oracle's angle lies
    within a window of a boundary; the window grows as 1 / rho for the pair's
    radius rho (fp32 atan2 of a pair with a small radius moves by ~1e-7 / rho),
    and such mismatches stay below a 1e-3 rate;
  * given the GPU's indices, the sign bits equal those of the oracle's
    residual except where |(S r)_i| < 1e-4, and fp16 ||r|| within 1e-3;
  * logits given identical codes within the logit tolerance of tests/parity.py
    (1e-3 of ||q|| ||x|| / sqrt(d)).
"""

import numpy as np
import pytest

from kv_cache_vector_rotate_b200 import synth
from oracle import polar_oracle as PO
from oracle import tq_oracle as O
from parity import LOGIT_TOL

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tqm():
    from kv_cache_vector_rotate_b200 import tq as tqmod
    tqmod.load_library()
    return tqmod


def _unpack(records: np.ndarray, d: int, bits: int, m: int):
    """records uint8 [n, RB] -> (idx per level, qneg [n, m] | None, norm16, rnorm16)."""
    n = records.shape[0]
    words = np.ascontiguousarray(records).view(np.uint32)
    cw = ((d - 1) * bits + 31) // 32
    sbits = np.unpackbits(words[:, :cw].view(np.uint8), axis=1, bitorder="little")   # [n, 32 cw]
    codes = np.zeros((n, d - 1), dtype=np.int64)
    for k in range(bits):
        codes |= sbits[:, np.arange(d - 1) * bits + k].astype(np.int64) << k
    idx, off = [], 0
    half = d // 2
    while half >= 1:
        idx.append(codes[:, off:off + half])
        off += half
        half //= 2
    qneg = None
    if m > 0:
        sb = np.unpackbits(words[:, cw:cw + m // 32].view(np.uint8), axis=1, bitorder="little")
        qneg = sb[:, :m].astype(bool)
    nw = words[:, cw + m // 32]
    n16 = (nw & 0xFFFF).astype(np.uint16).view(np.float16)
    r16 = (nw >> 16).astype(np.uint16).view(np.float16)
    return idx, qneg, n16, r16


def _level_radii(U_rot: np.ndarray):
    """The radius of every angle's pair, level 1 first (float64)."""
    rho, out = U_rot, []
    while rho.shape[1] > 1:
        a, b = rho[:, 0::2], rho[:, 1::2]
        r = np.sqrt(a * a + b * b)
        out.append(r)
        rho = r
    return out


def _inputs(seed: int, n: int, d: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d)) * np.exp(rng.uniform(-1, 1, size=(1, d)))
    X[rng.random((n, d)) < 0.01] *= 30.0       # outliers
    X[0] = 0.0                                  # the zero vector
    X[1] = 1e-3 * rng.standard_normal(d)        # a small vector
    return X.astype(np.float32)


@pytest.mark.parametrize("d,bits,m", [(128, 3, 128), (128, 1, 0), (128, 4, 0), (64, 2, 64), (256, 3, 256),
                                      (256, 4, 128), (64, 4, 32)])
def test_polar_encode_matches_oracle(tqm, d, bits, m):
    n = 3000
    X = _inputs(500 + d + bits + m, n, d)
    pc = tqm.PolarCodec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rec = tqm.polar_encode(pc, torch.from_numpy(X).cuda(), error_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    idx, qneg, n16, r16 = _unpack(rec.cpu().numpy(), d, bits, m)
    codec = PO.make_polar_codec(d, bits, synth.SEED_PI, m, synth.SEED_S)
    enc = PO.polar_encode(codec, X.astype(np.float64))
    # norms
    ref = enc.norm16.astype(np.float64)
    ulp = np.spacing(np.abs(enc.norm16)).astype(np.float64)
    assert np.all(np.abs(n16.astype(np.float64) - ref) <= ulp)
    # angle indices, outside the windows
    U, _ = O.unit_and_norm(X.astype(np.float64))
    radii = _level_radii(U @ codec.Pi.T)
    total, bad = 0, 0
    for lvl, (gi, oi, ang, rho, book) in enumerate(zip(idx, enc.idx, enc.angles, radii, codec.books), start=1):
        dist = np.min(np.abs(ang[..., None] - book.boundaries[None, None, :]), axis=-1)
        window = 1e-5 + 4e-7 / np.maximum(rho, 1e-30)
        mism = gi != oi
        assert np.all(dist[mism] <= window[mism]), (lvl, np.max(np.abs(gi - oi)))
        total += gi.size
        bad += int(mism.sum())
    assert bad <= 1e-3 * total, (bad, total)
    if m > 0:
        # the residual of the GPU's own indices
        Uh = PO.polar_decode_unit(codec, [np.asarray(g) for g in idx])
        R = U - Uh @ codec.Pi
        proj = R @ codec.S.T
        ok = (proj < 0) == qneg
        assert np.all(ok | (np.abs(proj) < 1e-4)), np.max(np.abs(proj[~ok]))
        rn = np.sqrt(np.sum(R * R, axis=1))
        assert np.all(np.abs(r16.astype(np.float64) - rn) <= 1e-3 * np.maximum(rn, 1e-3) + np.spacing(np.float16(rn)))
    pc.close()


@pytest.mark.parametrize("d,bits,m,nq,qdtype", [(128, 3, 128, 4, "bf16"), (128, 2, 0, 70, "f32"),
                                                (64, 4, 64, 9, "f32"), (256, 3, 256, 33, "bf16"),
                                                (256, 1, 0, 4, "f16")])
def test_polar_logits_match_oracle_given_codes(tqm, d, bits, m, nq, qdtype):
    n = 1500
    X = _inputs(600 + d + bits, n, d)
    rng = np.random.default_rng(601 + d)
    qf = rng.standard_normal((nq, d)).astype(np.float32)
    if qdtype == "bf16":
        Q = synth.to_bf16(qf)[1].astype(np.float64)
        qt = torch.from_numpy(Q.astype(np.float32)).cuda().to(torch.bfloat16)
    elif qdtype == "f16":
        Q = qf.astype(np.float16).astype(np.float64)
        qt = torch.from_numpy(qf.astype(np.float16)).cuda()
    else:
        Q = qf.astype(np.float64)
        qt = torch.from_numpy(qf).cuda()
    pc = tqm.PolarCodec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    rec = tqm.polar_encode(pc, torch.from_numpy(X).cuda())
    L = tqm.polar_logits(pc, rec, qt)
    torch.cuda.synchronize()
    idx, qneg, n16, r16 = _unpack(rec.cpu().numpy(), d, bits, m)
    codec = PO.make_polar_codec(d, bits, synth.SEED_PI, m, synth.SEED_S)
    enc = PO.PolarEncoded([np.asarray(g) for g in idx], n16, [], qneg if m > 0 else None, r16 if m > 0 else None)
    Lo = PO.polar_logits(codec, Q, enc)
    scale = np.linalg.norm(Q, axis=1)[:, None] * n16.astype(np.float64)[None, :] / np.sqrt(d)
    err = np.abs(L.cpu().numpy() - Lo)
    assert np.all(err <= LOGIT_TOL * scale + 1e-30), np.max(err / np.maximum(scale, 1e-30))
    assert np.all(L.cpu().numpy()[:, 0] == 0.0)      # the zero vector
    pc.close()


def test_polar_unsupported_shapes(tqm):
    for d, bits, m in [(100, 3, 0), (128, 5, 0), (128, 3, 16), (64, 2, 128)]:
        with pytest.raises(tqm.TqError):
            tqm.PolarCodec(d, bits, m, 1, 2)
