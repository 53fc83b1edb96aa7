"""GPU tests of tq_attend against the oracle's attention: the fused split-K
path (d <= 128, equal page sizes) and the composed path (logits, cluster row
softmax, value pass), full decode-step size, bad pages; and what the value
pass and tq_attend write for empty contexts and read past the context."""

import numpy as np
import pytest

from kv_cache_vector_rotate_b200 import synth
from oracle import tq_oracle as O
from parity import VALUE_TOL
from gpu_cases import _oracle_cache, _q_tensor

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tqm():
    from kv_cache_vector_rotate_b200 import tq as tqmod
    tqmod.load_library()
    return tqmod


def _attend_case(tqm, d, kbits, m, vbits, kpt, vpt, ctx, heads, G, seed, qdtype="bf16", vscale=2.0):
    """Both caches written by the oracle, tq_attend on the GPU, and the
    oracle's softmax attention given the same codes.  The logit tolerance
    (1e-3 of ||q|| ||k|| / sqrt(d)) moves the softmax weights by at most
    about scale x that, so the output is checked to 2e-3 of its row scale."""
    batch = len(ctx)
    rng = np.random.default_rng(seed)
    keys = rng.standard_normal((batch, heads, max(ctx), d)) * np.exp(rng.uniform(-1, 1, size=(1, heads, 1, d)))
    vals = rng.standard_normal((batch, heads, max(ctx), d)) * vscale
    kcodec = O.make_codec(d, kbits, m, synth.SEED_PI, synth.SEED_S)
    vcodec = O.make_codec(d, vbits, 0, synth.SEED_PI, synth.SEED_S)
    kcb, kcache, kencs, _ = _oracle_cache(tqm, kcodec, O.Layout(d, kbits, m, kpt, heads), keys, ctx, kpt, seed + 1)
    vcb, vcache, vencs, _ = _oracle_cache(tqm, vcodec, O.Layout(d, vbits, 0, vpt, heads), vals, ctx, vpt, seed + 2)
    qf = rng.standard_normal((batch, heads * G, d)).astype(np.float32)
    q = synth.to_bf16(qf)[1] if qdtype == "bf16" else qf.astype(np.float64)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    scale = 1.0 / np.sqrt(d)
    out = tqm.attend(kcb, kcache, vcb, vcache, _q_tensor(q, qdtype), ctx_t, max(ctx), scale=scale)
    torch.cuda.synchronize()
    O_gpu = out.cpu().numpy()
    for b in range(batch):
        for h in range(heads):
            if ctx[b] == 0:
                assert not O_gpu[b, h * G:(h + 1) * G].any()
                continue
            _check_attention(kcodec, vcodec, q[b, h * G:(h + 1) * G], kencs[(b, h)][1], vencs[(b, h)][1],
                             scale, O_gpu[b, h * G:(h + 1) * G], (b, h))
    assert kcache.errors() == 0 and vcache.errors() == 0


def _check_attention(kcodec, vcodec, Qg, ke, ve, scale, got, where, keep=None):
    if keep is not None:
        ke = O.Encoded(*(None if x is None else np.asarray(x)[keep] for x in
                         (ke.idx, ke.qneg, ke.norm16, ke.rnorm16, ke.y, ke.proj)))
        ve = O.Encoded(*(None if x is None else np.asarray(x)[keep] for x in
                         (ve.idx, ve.qneg, ve.norm16, ve.rnorm16, ve.y, ve.proj)))
    o = O.attention_from_codes(kcodec, vcodec, Qg, (ke.idx, ke.qneg, ke.norm16, ke.rnorm16),
                               (ve.idx, ve.norm16), scale)
    vh = O.dequantize(vcodec, ve.idx, ve.norm16)
    row_scale = np.maximum(np.abs(o).max(axis=1), np.linalg.norm(vh, axis=1).mean() / np.sqrt(kcodec.d))
    err = np.abs(got - o).max(axis=1)
    assert np.all(err <= 2e-3 * row_scale), (where, err / row_scale)


# The fused split-K path: d <= 128 and equal page sizes.  Contexts of 700
# (ragged last unit), 129 (one token past two units) and 0 (a zero row);
# 16-token pages (units straddle pages), 256-token pages (several units per
# page); GQA groups of 1, 2, 4 and 8 query heads (two query tiles).
@pytest.mark.parametrize("d,kbits,m,vbits,pt,G", [
    (128, 3, 128, 3, 32, 4), (128, 2, 128, 4, 32, 4), (128, 4, 0, 2, 32, 4), (128, 3, 128, 3, 16, 4),
    (128, 3, 128, 3, 256, 4), (128, 3, 128, 3, 64, 8), (64, 2, 64, 2, 64, 4), (96, 3, 96, 3, 64, 2),
    (128, 1, 128, 1, 128, 1), (64, 4, 0, 4, 16, 4)])
def test_attend_matches_oracle_attention(tqm, d, kbits, m, vbits, pt, G):
    _attend_case(tqm, d, kbits, m, vbits, pt, pt, [700, 129, 0], 2, G, 34 + kbits + vbits + G)


# The composed path (logits, row softmax, value pass): d > 128, or key and
# value caches with different page sizes.
@pytest.mark.parametrize("d,kpt,vpt", [(200, 64, 64), (256, 32, 32), (128, 32, 64)])
def test_attend_composed_path_matches_oracle(tqm, d, kpt, vpt):
    _attend_case(tqm, d, 3, d, 3, kpt, vpt, [700, 129, 0], 2, 4, 60 + d)


@pytest.mark.parametrize("G,kbits,vbits", [(6, 3, 2), (3, 2, 4), (12, 4, 3)])
def test_attend_ragged_query_tiles(tqm, G, kbits, vbits):
    """GQA groups that are not a multiple of 4 (the last query tile of a line
    is ragged) on the fused path, at 4000 / 2500 tokens, mixed key and value
    widths."""
    _attend_case(tqm, 128, kbits, 128, vbits, 64, 64, [4000, 2500], 2, G, 70 + G)


def test_attend_many_units_per_cta(tqm):
    """Two sequences x 8 KV heads x 32 query heads at 8192 / 7777 tokens: CTAs
    with many units, shares that span two lines (the consumer warps split
    between them), refills of every ring slot."""
    _attend_case(tqm, 128, 3, 128, 3, 64, 64, [8192, 7777], 8, 4, 61)


def test_attend_small_value_norms(tqm):
    """Value norms near 1e-5 over 8192 tokens (p ||v|| far below fp16's normal
    range): the fused kernel's B operand carries a power-of-two scale."""
    _attend_case(tqm, 128, 3, 128, 3, 64, 64, [8192, 3000], 2, 4, 64, vscale=1e-5 / np.sqrt(128))


def test_attend_decode_config_full_size(tqm):
    """The decode step at full size (batch 1, 8 KV / 32 query heads, d 128,
    context 32768, keys b = 3 + QJL m = 128, values b = 3) with the bench's
    inputs, against the oracle on every head."""
    batch, hkv, hq, ctx, d, pt = 1, 8, 32, 32768, 128, 64
    data = synth.decode_step(1002, batch, hkv, hq, ctx, d)
    kcodec = O.make_codec(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    vcodec = O.make_codec(d, 3, 0, synth.SEED_PI, synth.SEED_S)
    kcb, kcache, kencs, _ = _oracle_cache(tqm, kcodec, O.Layout(d, 3, 128, pt, hkv), data["k"][1], [ctx], pt, 24)
    vcb, vcache, vencs, _ = _oracle_cache(tqm, vcodec, O.Layout(d, 3, 0, pt, hkv), data["v"][1], [ctx], pt, 25)
    qbits, q = data["q"]
    qt = torch.from_numpy(qbits.view(np.int16)).view(torch.bfloat16).cuda()
    scale = 1.0 / np.sqrt(d)
    out = tqm.attend(kcb, kcache, vcb, vcache, qt, torch.tensor([ctx], dtype=torch.int32, device="cuda"), ctx,
                     scale=scale)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    G = hq // hkv
    for h in range(hkv):
        _check_attention(kcodec, vcodec, q[0, h * G:(h + 1) * G], kencs[(0, h)][1], vencs[(0, h)][1], scale,
                         got[0, h * G:(h + 1) * G], h)
    assert kcache.errors() == 0 and vcache.errors() == 0


@pytest.mark.parametrize("which", ["key", "value"])
def test_attend_bad_page_is_skipped_and_reported(tqm, which):
    """A block-table entry out of range inside the context: the call
    completes, the cache's error word has the page bit, and the tokens of
    that page leave the softmax (the rest match the oracle's attention over
    the remaining tokens)."""
    d, pt, heads, G, ctx = 128, 32, 2, 4, [2048]
    rng = np.random.default_rng(62)
    keys = rng.standard_normal((1, heads, ctx[0], d))
    vals = rng.standard_normal((1, heads, ctx[0], d)) * 2.0
    kcodec = O.make_codec(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    vcodec = O.make_codec(d, 3, 0, synth.SEED_PI, synth.SEED_S)
    kcb, kcache, kencs, kbt = _oracle_cache(tqm, kcodec, O.Layout(d, 3, 128, pt, heads), keys, ctx, pt, 63)
    vcb, vcache, vencs, vbt = _oracle_cache(tqm, vcodec, O.Layout(d, 3, 0, pt, heads), vals, ctx, pt, 63)
    cache = kcache if which == "key" else vcache
    bad_page = 17
    cache.block_table[0, bad_page] = 10 ** 6
    qf = rng.standard_normal((1, heads * G, d)).astype(np.float32)
    q = synth.to_bf16(qf)[1]
    scale = 1.0 / np.sqrt(d)
    out = tqm.attend(kcb, kcache, vcb, vcache, _q_tensor(q, "bf16"), torch.tensor(ctx, dtype=torch.int32,
                     device="cuda"), ctx[0], scale=scale)
    torch.cuda.synchronize()
    assert cache.errors() & tqm.DEV_ERR_PAGE
    got = out.cpu().numpy()
    pos = np.arange(ctx[0])
    keep = (pos // pt) != bad_page
    for h in range(heads):
        _check_attention(kcodec, vcodec, q[0, h * G:(h + 1) * G], kencs[(0, h)][1], vencs[(0, h)][1], scale,
                         got[0, h * G:(h + 1) * G], h, keep=keep)

def test_attend_with_no_context_clears_out(tqm):
    """max_ctx = 0: every context is empty, so tq_attend writes zero rows over
    whatever out held."""
    d, pt, heads, G, batch = 128, 32, 2, 4, 2
    kcb = tqm.Codebook(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    vcb = tqm.Codebook(d, 3, 0, synth.SEED_PI, synth.SEED_S)
    bt = torch.from_numpy(synth.block_table(37, batch, 1))
    kcache = tqm.PagedCache.allocate(kcb, batch, pt, heads, bt)
    vcache = tqm.PagedCache.allocate(vcb, batch, pt, heads, bt)
    q = torch.randn(batch, heads * G, d, device="cuda").to(torch.bfloat16)
    out = torch.full((batch, heads * G, d), float("nan"), device="cuda")
    ctx_t = torch.zeros(batch, dtype=torch.int32, device="cuda")
    tqm.attend(kcb, kcache, vcb, vcache, q, ctx_t, 0, out=out)
    torch.cuda.synchronize()
    assert bool((out == 0).all())

def test_values_mode_b_with_no_context_clears_out(tqm):
    """Mode B with max_ctx = 0: every weighted sum is over an empty context,
    so out becomes zeros whatever it held."""
    d, pt, heads, G, batch = 128, 32, 2, 4, 2
    cb = tqm.Codebook(d, 3, 0, synth.SEED_PI, synth.SEED_S)
    cache = tqm.PagedCache.allocate(cb, batch, pt, heads, torch.from_numpy(synth.block_table(38, batch, 1)))
    w = torch.zeros(batch, heads * G, 1, device="cuda")
    out = torch.full((batch, heads * G, d), float("nan"), device="cuda")
    ctx_t = torch.zeros(batch, dtype=torch.int32, device="cuda")
    tqm.dequant_values(cb, cache, ctx_t, 0, batch, weights=w, out=out)
    torch.cuda.synchronize()
    assert bool((out == 0).all())

def test_values_mode_b_ignores_bytes_past_the_context(tqm):
    """Slots past a sequence's context may hold any bytes (here 0xFF: NaN
    norms): mode B must not let them reach the sums (zero weight times a
    NaN norm would)."""
    d, bits, pt, batch, heads, G, n = 128, 3, 64, 2, 2, 4, 700
    ctx = [700, 129]
    cb = tqm.Codebook(d, bits, 0, synth.SEED_PI, synth.SEED_S)
    pps = (n + pt - 1) // pt
    bt = synth.block_table(39, batch, pps)
    cache = tqm.PagedCache.allocate(cb, batch * pps, pt, heads, torch.from_numpy(bt))
    cache.pages.fill_(0xFF)
    V = np.random.default_rng(40).standard_normal((batch, heads, n, d)).astype(np.float32)
    tqm.quantize_append(cb, torch.from_numpy(V).cuda(), torch.zeros(batch, dtype=torch.int32, device="cuda"), cache)
    W = synth.softmax_like_weights(41, batch, heads * G, n)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    out = tqm.dequant_values(cb, cache, ctx_t, n, batch, weights=torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    B = out.cpu().numpy()
    assert np.all(np.isfinite(B))
    codec = O.make_codec(d, bits, 0, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, 0, pt, heads)
    pages = cache.pages.cpu().numpy()
    for b in range(batch):
        for h in range(heads):
            idx, _, n16, _ = O.read_pages(lay, pages, bt, b, h, np.arange(ctx[b]))
            Vh = O.dequantize(codec, idx, n16)
            Wg = W[b, h * G:(h + 1) * G, : ctx[b]].astype(np.float64)
            o = Wg @ Vh
            scale = np.maximum(np.abs(o).max(axis=1), (np.abs(Wg) @ np.linalg.norm(Vh, axis=1)) / np.sqrt(d))
            assert np.all(np.abs(B[b, h * G:(h + 1) * G] - o) <= VALUE_TOL * scale[:, None])
    assert cache.errors() == 0


def test_values_mode_b_small_norms_long_context(tqm):
    """Mode B at context 32768 with value norms near 1e-3 and softmax-like
    weights (w ||v|| near 3e-8, below fp16's normal range): the B operand
    carries a power-of-two scale, so the sums keep their precision."""
    d, bits, pt, heads, G, n = 128, 3, 64, 2, 4, 32768
    rng = np.random.default_rng(90)
    V = (rng.standard_normal((1, heads, n, d)) * (1e-3 / np.sqrt(d))).astype(np.float32)
    codec = O.make_codec(d, bits, 0, synth.SEED_PI, synth.SEED_S)
    cb, cache, encs, _ = _oracle_cache(tqm, codec, O.Layout(d, bits, 0, pt, heads), V.astype(np.float64), [n], pt, 91)
    W = synth.softmax_like_weights(92, 1, heads * G, n)
    out = tqm.dequant_values(cb, cache, torch.tensor([n], dtype=torch.int32, device="cuda"), n, 1,
                             weights=torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    B = out.cpu().numpy()
    for h in range(heads):
        _, e = encs[(0, h)]
        Vh = O.dequantize(codec, e.idx, e.norm16)
        Wg = W[0, h * G:(h + 1) * G].astype(np.float64)
        o = Wg @ Vh
        scale = np.maximum(np.abs(o).max(axis=1), (np.abs(Wg) @ np.linalg.norm(Vh, axis=1)) / np.sqrt(d))
        assert np.all(np.abs(B[0, h * G:(h + 1) * G] - o) <= VALUE_TOL * scale[:, None]), h
    assert cache.errors() == 0


@pytest.mark.parametrize("d,bits,pt,G,batch,heads", [(128, 3, 32, 6, 3, 3), (64, 4, 16, 3, 2, 5),
                                                     (128, 1, 128, 9, 1, 2)])
def test_values_mode_b_ragged_groups_bad_page(tqm, d, bits, pt, G, batch, heads):
    """Mode B on the fused pass (d <= 128): query groups that are not a
    multiple of 4 (a ragged second query tile), several (sequence, KV head)
    lines per CTA, contexts 1500 / 0 / 333, and one out-of-range block-table
    entry inside sequence 0's context: the page is reported and its tokens
    are left out of the sums."""
    ctx = [1500, 0, 333][:batch]
    rng = np.random.default_rng(300 + d + bits + G)
    vals = rng.standard_normal((batch, heads, max(ctx), d)) * 2.0
    codec = O.make_codec(d, bits, 0, synth.SEED_PI, synth.SEED_S)
    cb, cache, encs, bt = _oracle_cache(tqm, codec, O.Layout(d, bits, 0, pt, heads), vals, ctx, pt, 301 + G)
    bad_page = 3
    cache.block_table[0, bad_page] = 10 ** 6
    W = synth.softmax_like_weights(302 + G, batch, heads * G, max(ctx))
    out = tqm.dequant_values(cb, cache, torch.tensor(ctx, dtype=torch.int32, device="cuda"), max(ctx), batch,
                             weights=torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    assert cache.errors() & tqm.DEV_ERR_PAGE
    B = out.cpu().numpy()
    for b in range(batch):
        for h in range(heads):
            if ctx[b] == 0:
                assert not B[b, h * G:(h + 1) * G].any()
                continue
            _, e = encs[(b, h)]
            Vh = O.dequantize(codec, e.idx, e.norm16)
            Wg = W[b, h * G:(h + 1) * G, : ctx[b]].astype(np.float64).copy()
            if b == 0:
                Wg[:, (np.arange(ctx[b]) // pt) == bad_page] = 0.0
            o = Wg @ Vh
            scale = np.maximum(np.abs(o).max(axis=1), (np.abs(Wg) @ np.linalg.norm(Vh, axis=1)) / np.sqrt(d))
            assert np.all(np.abs(B[b, h * G:(h + 1) * G] - o) <= VALUE_TOL * scale[:, None]), (b, h)
