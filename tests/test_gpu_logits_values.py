"""GPU parity of tq_logits and tq_dequant_values against the fp64 oracle.

The caches are written by the ORACLE (oracle/ packs the records); the GPU
reads them through the C ABI, so the logits and values are compared given
identical codes.  Tolerances are those of tests/parity.py.
"""

import numpy as np
import pytest

from kv_cache_vector_rotate_b200 import synth
from oracle import tq_oracle as O
from gpu_cases import _check_logits, _oracle_cache, _q_tensor
from parity import LOGIT_TOL, VALUE_TOL, compare_codes, logit_error

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tqm():
    from kv_cache_vector_rotate_b200 import tq as tqmod
    tqmod.load_library()
    return tqmod


def test_tiny_config_logits(tqm):
    # 4096 fp32 keys with outlier channels, 16 fp32 queries on one KV head.
    K, Q, _ = synth.tiny_keys()
    d, bits, m, pt = 128, 3, 128, 64
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, 1)
    keys = K.astype(np.float64)[None, None]
    cb, cache, encs, _ = _oracle_cache(tqm, codec, lay, keys, [4096], pt, 21)
    q = Q.astype(np.float64)[None]
    ctx = torch.tensor([4096], dtype=torch.int32, device="cuda")
    L = tqm.logits(cb, cache, _q_tensor(q, "f32"), ctx, 4096)
    torch.cuda.synchronize()
    _check_logits(codec, q, encs, L.cpu().numpy(), [4096], 1, 16)
    assert cache.errors() == 0


@pytest.mark.parametrize("d,bits,m,G,dtype", [
    (128, 3, 128, 4, "bf16"), (128, 2, 128, 4, "bf16"), (128, 4, 128, 4, "f16"),
    (128, 1, 128, 2, "f32"), (128, 3, 0, 4, "bf16"), (64, 3, 64, 5, "bf16"),
    (200, 2, 200, 3, "f32"), (256, 4, 256, 8, "bf16"), (192, 3, 192, 1, "bf16"),
])
def test_logits_ragged_context(tqm, d, bits, m, G, dtype):
    batch, heads, pt = 2, 2, 32
    ctx = [1000, 333]
    rng = np.random.default_rng(22)
    keys = rng.standard_normal((batch, heads, max(ctx), d)) * np.exp(rng.uniform(-2, 2, size=(1, heads, 1, d)))
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, heads)
    cb, cache, encs, _ = _oracle_cache(tqm, codec, lay, keys, ctx, pt, 23)
    qf = rng.standard_normal((batch, heads * G, d)).astype(np.float32)
    if dtype == "bf16":
        _, q = synth.to_bf16(qf)
    elif dtype == "f16":
        q = qf.astype(np.float16).astype(np.float64)
    else:
        q = qf.astype(np.float64)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    out = torch.full((batch, heads * G, max(ctx)), float("nan"), device="cuda")
    tqm.logits(cb, cache, _q_tensor(q, dtype), ctx_t, max(ctx), out=out)
    torch.cuda.synchronize()
    L = out.cpu().numpy()
    _check_logits(codec, q, encs, L, ctx, heads, G)
    assert np.all(np.isnan(L[1, :, ctx[1]:]))          # positions past ctx_len untouched
    assert cache.errors() == 0


def test_logits_decode_config_full_size(tqm):
    # batch 1, 8 KV heads / 32 query heads, d = 128, context 32768, bf16 keys
    # with per-channel log-uniform scales; b = 3 + QJL m = 128.
    batch, hkv, hq, ctx, d, pt = 1, 8, 32, 32768, 128, 64
    data = synth.decode_step(1002, batch, hkv, hq, ctx, d)
    codec = O.make_codec(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, 3, 128, pt, hkv)
    cb, cache, encs, _ = _oracle_cache(tqm, codec, lay, data["k"][1], [ctx], pt, 24)
    qbits, q = data["q"]
    qt = torch.from_numpy(qbits.view(np.int16)).view(torch.bfloat16).cuda()
    L = tqm.logits(cb, cache, qt, torch.tensor([ctx], dtype=torch.int32, device="cuda"), ctx)
    torch.cuda.synchronize()
    _check_logits(codec, q, encs, L.cpu().numpy(), [ctx], hkv, hq // hkv)


def test_logits_empty_context(tqm):
    cb = tqm.Codebook(128, 3, 128, synth.SEED_PI, synth.SEED_S)
    cache = tqm.PagedCache.allocate(cb, 1, 64, 1, torch.zeros(2, 1, dtype=torch.int32))
    q = torch.ones(2, 4, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.full((2, 4, 64), 7.0, device="cuda")
    tqm.logits(cb, cache, q, torch.tensor([0, 0], dtype=torch.int32, device="cuda"), 64, out=out)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


@pytest.mark.parametrize("d,bits,pt", [(128, 3, 64), (128, 2, 64), (200, 4, 64), (64, 1, 64),
                                       (128, 3, 16), (128, 3, 256)])
def test_values_mode_a_and_b(tqm, d, bits, pt):
    # pt = 16: 32-token units straddle pages (the kernels' per-half copies);
    # pt = 256: several units per page
    batch, heads, G = 2, 2, 4
    ctx = [700, 129]
    rng = np.random.default_rng(31)
    vals = rng.standard_normal((batch, heads, max(ctx), d)) * 2.0
    codec = O.make_codec(d, bits, 0, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, 0, pt, heads)
    cb, cache, encs, _ = _oracle_cache(tqm, codec, lay, vals, ctx, pt, 32)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    # mode A
    outA = tqm.dequant_values(cb, cache, ctx_t, max(ctx), batch)
    # mode B
    W = synth.softmax_like_weights(33, batch, heads * G, max(ctx))
    outB = tqm.dequant_values(cb, cache, ctx_t, max(ctx), batch, weights=torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    A = outA.cpu().numpy()
    B = outB.cpu().numpy()
    for (b, h), (pos, enc) in encs.items():
        Vh = O.dequantize(codec, enc.idx, enc.norm16)
        err = np.abs(A[b, h, : ctx[b]] - Vh)
        assert np.all(err <= VALUE_TOL * np.max(np.abs(Vh), axis=1, keepdims=True) + 1e-30)
        assert not A[b, h, ctx[b]:].any()
        Wg = W[b, h * G:(h + 1) * G, : ctx[b]].astype(np.float64)
        o = Wg @ Vh
        scale = np.maximum(np.abs(o).max(axis=1), (np.abs(Wg) @ np.linalg.norm(Vh, axis=1)) / np.sqrt(d))
        assert np.all(np.abs(B[b, h * G:(h + 1) * G] - o) <= VALUE_TOL * scale[:, None])
    assert cache.errors() == 0


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_long_context_config_sampled(tqm, bits):
    """Long-context decode: batch 4, 8 KV / 32 query heads, d = 128, context
    131072, keys b + QJL m = 128, written by the GPU append.  On 256 sampled
    positions of every (sequence, KV head): the codes against the oracle's
    encoding of the same vectors, and the GPU logits at those positions
    against the oracle estimator given the codes read back."""
    batch, hkv, hq, ctx, d, m, pt = 4, 8, 32, 131072, 128, 128, 64
    G = hq // hkv
    K, q = synth.decode_keys_device(1003 + bits, batch, hkv, hq, ctx, d)
    pps = ctx // pt
    bt = synth.block_table(25 + bits, batch, pps)
    cb = tqm.Codebook(d, bits, m, synth.SEED_PI, synth.SEED_S)
    cache = tqm.PagedCache.allocate(cb, batch * pps, pt, hkv, torch.from_numpy(bt))
    tqm.quantize_append(cb, K, torch.zeros(batch, dtype=torch.int32, device="cuda"), cache)
    ctx_t = torch.full((batch,), ctx, dtype=torch.int32, device="cuda")
    L = tqm.logits(cb, cache, q, ctx_t, ctx)
    torch.cuda.synchronize()
    assert cache.errors() == 0
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, hkv)
    pages = cache.pages.cpu().numpy()
    rng = np.random.default_rng(26 + bits)
    qf = q.float().cpu().numpy().astype(np.float64)
    worst = 0.0
    got = {"X": [], "idx": [], "qneg": [], "n16": [], "r16": []}
    for b in range(batch):
        for h in range(hkv):
            pos = np.sort(rng.choice(ctx, 256, replace=False))
            X = K[b, h, torch.from_numpy(pos).cuda()].float().cpu().numpy().astype(np.float64)
            idx, qneg, n16, r16 = O.read_pages(lay, pages, bt, b, h, pos)
            for k_, v_ in zip(got, (X, idx, qneg, n16, r16)):
                got[k_].append(v_)
            Qg = qf[b, h * G:(h + 1) * G]
            Lo = O.logits_from_codes(codec, Qg, idx, qneg, n16, r16)
            Lg = L[b, h * G:(h + 1) * G][:, torch.from_numpy(pos).cuda()].cpu().numpy()
            worst = max(worst, logit_error(Lg, Lo, np.linalg.norm(Qg, axis=1), n16, d))
    assert worst <= LOGIT_TOL, worst
    # the mismatch rate is a statistic of the whole sample (8192 vectors)
    X = np.concatenate(got["X"])
    compare_codes(codec, X, O.encode(codec, X), *(np.concatenate(got[k_]) for k_ in ("idx", "qneg", "n16", "r16")))


def _small_case(tqm, batch, heads, G, ctx, pt, seed, d=128, bits=3, m=128):
    rng = np.random.default_rng(seed)
    keys = rng.standard_normal((batch, heads, max(ctx), d))
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, heads)
    cb, cache, encs, _ = _oracle_cache(tqm, codec, lay, keys, ctx, pt, seed + 1)
    _, q = synth.to_bf16(rng.standard_normal((batch, heads * G, d)).astype(np.float32))
    return codec, cb, cache, encs, q


def test_logits_workspace_reused_across_shapes(tqm):
    # One workspace serves calls of three shapes in turn (stale fragments of
    # a larger shape left in it); each call is exact against the oracle.
    cases = [(2, 2, 4, [700, 129], 32), (1, 4, 8, [1500], 64), (3, 1, 2, [64, 1, 300], 16)]
    built = [_small_case(tqm, *c, seed=40 + i) for i, c in enumerate(cases)]
    need = max(tqm.logits_workspace_bytes(cb, len(c[3]), c[1], c[1] * c[2])
               for c, (_, cb, _, _, _) in zip(cases, built))
    ws = torch.full((need,), 0x5A, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for (batch, heads, G, ctx, pt), (codec, cb, cache, encs, q) in zip(cases, built):
            ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
            L = tqm.logits(cb, cache, _q_tensor(q, "bf16"), ctx_t, max(ctx), workspace=ws)
            torch.cuda.synchronize()
            _check_logits(codec, q, encs, L.cpu().numpy(), ctx, heads, G)
            assert cache.errors() == 0


def test_logits_more_query_tiles_than_cta_slots(tqm):
    # 128 sequences x 8 KV heads = 1024 query tiles, short ragged contexts:
    # more tiles than CTA slots on the GPU (148 SMs x 5), one CTA per tile.
    ctx = [40 + (i * 7) % 25 for i in range(128)]
    codec, cb, cache, encs, q = _small_case(tqm, 128, 8, 4, ctx, 16, 50)
    L = tqm.logits(cb, cache, _q_tensor(q, "bf16"), torch.tensor(ctx, dtype=torch.int32, device="cuda"),
                   max(ctx))
    torch.cuda.synchronize()
    _check_logits(codec, q, encs, L.cpu().numpy(), ctx, 8, 4)
    assert cache.errors() == 0
