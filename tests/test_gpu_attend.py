"""GPU tests of tq_attend (logits, cluster row softmax, value pass) against the
oracle's attention, and of what the value pass and tq_attend write for empty
contexts and read past the context.  Collected after every other test file.
"""

import numpy as np
import pytest

from kv_cache_vector_rotate_b200 import synth
from oracle import tq_oracle as O
from parity import VALUE_TOL
from test_gpu_logits_values import _oracle_cache, _q_tensor

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tqm():
    from kv_cache_vector_rotate_b200 import tq as tqmod
    tqmod.load_library()
    return tqmod


@pytest.mark.parametrize("kbits,m,vbits,pt", [(3, 128, 3, 32), (2, 128, 4, 32), (4, 0, 2, 32), (3, 128, 3, 16),
                                              (3, 128, 3, 256)])
def test_attend_matches_oracle_attention(tqm, kbits, m, vbits, pt):
    """tq_attend (logits from the key codes, row softmax, values from their
    codes) against the oracle's softmax attention given the same codes; a
    sequence with an empty context gives a zero row.  The logit tolerance
    (1e-3 of ||q|| ||k|| / sqrt(d)) moves the softmax weights by at most about
    scale x that, so the output is checked to 2e-3 of its row scale."""
    batch, heads, G, d = 3, 2, 4, 128
    ctx = [700, 129, 0]
    rng = np.random.default_rng(34 + kbits + vbits)
    keys = rng.standard_normal((batch, heads, max(ctx), d)) * np.exp(rng.uniform(-1, 1, size=(1, heads, 1, d)))
    vals = rng.standard_normal((batch, heads, max(ctx), d)) * 2.0
    kcodec = O.make_codec(d, kbits, m, synth.SEED_PI, synth.SEED_S)
    vcodec = O.make_codec(d, vbits, 0, synth.SEED_PI, synth.SEED_S)
    kcb, kcache, kencs, _ = _oracle_cache(tqm, kcodec, O.Layout(d, kbits, m, pt, heads), keys, ctx, pt, 35)
    vcb, vcache, vencs, _ = _oracle_cache(tqm, vcodec, O.Layout(d, vbits, 0, pt, heads), vals, ctx, pt, 36)
    _, q = synth.to_bf16(rng.standard_normal((batch, heads * G, d)).astype(np.float32))
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    scale = 1.0 / np.sqrt(d)
    out = tqm.attend(kcb, kcache, vcb, vcache, _q_tensor(q, "bf16"), ctx_t, max(ctx), scale=scale)
    torch.cuda.synchronize()
    O_gpu = out.cpu().numpy()
    for b in range(batch):
        for h in range(heads):
            Qg = q[b, h * G:(h + 1) * G]
            if ctx[b] == 0:
                assert not O_gpu[b, h * G:(h + 1) * G].any()
                continue
            _, ke = kencs[(b, h)]
            _, ve = vencs[(b, h)]
            o = O.attention_from_codes(kcodec, vcodec, Qg, (ke.idx, ke.qneg, ke.norm16, ke.rnorm16),
                                       (ve.idx, ve.norm16), scale)
            vh = O.dequantize(vcodec, ve.idx, ve.norm16)
            row_scale = np.maximum(np.abs(o).max(axis=1), np.linalg.norm(vh, axis=1).mean() / np.sqrt(d))
            err = np.abs(O_gpu[b, h * G:(h + 1) * G] - o).max(axis=1)
            assert np.all(err <= 2e-3 * row_scale), (b, h, err / row_scale)
    assert kcache.errors() == 0 and vcache.errors() == 0

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
