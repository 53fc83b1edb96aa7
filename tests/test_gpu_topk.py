"""GPU parity of tq_logits_topk (many-query scoring on the tensor cores with a
fused top-k) against the fp64 oracle given the GPU's codes.

The oracle ranks its own estimate (O.logits_from_codes of the codes read back
from the pages) with O.exact_top_k.  Scores within the logit tolerance of one
another may rank either way, so the check is: every returned score equals
the oracle's estimate at the returned position (LOGIT_TOL of ||q|| ||k|| /
sqrt(d)); the returned positions are distinct, in range and ranked best
first; and the returned set is a top-k of the oracle's scores up to twice
that tolerance (no returned score is clearly below the oracle's k-th, no
position left out is clearly above the returned k-th).
"""

import numpy as np
import pytest

from gpu_cases import _q_tensor
from kv_cache_vector_rotate_b200 import synth
from oracle import tq_oracle as O
from parity import LOGIT_TOL

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tqm():
    from kv_cache_vector_rotate_b200 import tq as tqmod
    tqmod.load_library()
    return tqmod


def _gpu_cache(tqm, X, d, bits, m, pt, ctx, seed):
    """X [batch, heads, n, d] float32 quantized on the GPU into a paged cache."""
    batch, heads, n, _ = X.shape
    cb = tqm.Codebook(d, bits, m, synth.SEED_PI, synth.SEED_S)
    pps = (n + pt - 1) // pt
    bt = synth.block_table(seed, batch, pps)
    cache = tqm.PagedCache.allocate(cb, batch * pps, pt, heads, torch.from_numpy(bt))
    tqm.quantize_append(cb, torch.from_numpy(np.ascontiguousarray(X)).cuda(),
                        torch.zeros(batch, dtype=torch.int32, device="cuda"), cache)
    return cb, cache, bt


def _check_topk(codec, lay, pages, bt, Q, ctx, heads, k, scores, idx, sample_rows=None, skip=None):
    """Q [batch, n_q_heads, d] float64; scores / idx [batch, n_q_heads, k] from the GPU."""
    batch, hq, d = Q.shape
    G = hq // heads
    rng = np.random.default_rng(5)
    for b in range(batch):
        for h in range(heads):
            pos = np.arange(ctx[b])
            if skip is not None:
                pos = pos[~skip(b, h, pos)]
            idx_o, qneg, n16, r16 = O.read_pages(lay, pages, bt, b, h, pos)
            rows = np.arange(G) if sample_rows is None else np.sort(rng.choice(G, sample_rows, replace=False))
            Qg = Q[b, h * G + rows]
            L = O.logits_from_codes(codec, Qg, idx_o, qneg, n16, r16)          # [rows, len(pos)]
            qn = np.linalg.norm(Qg, axis=1)
            kk = min(k, len(pos))
            # the oracle's k-th best score of each row (O.exact_top_k ranks the
            # same scores; the k-th value is all the set check needs)
            kth_all = -np.partition(-L, kk - 1, axis=1)[:, kk - 1] if kk > 0 else None
            for r, row in enumerate(rows):
                s_g = scores[b, h * G + row]
                i_g = idx[b, h * G + row]
                assert np.all(i_g[kk:] == -1) and np.all(np.isneginf(s_g[kk:])), (b, h, row)
                if kk == 0:
                    continue
                i_g, s_g = i_g[:kk], s_g[:kk]
                assert len(set(i_g.tolist())) == kk and np.all(np.isin(i_g, pos)), (b, h, row, i_g)
                col = np.searchsorted(pos, i_g)
                tol = LOGIT_TOL * qn[r] * n16[col].astype(np.float64) / np.sqrt(d)
                assert np.all(np.abs(s_g - L[r, col]) <= tol), (b, h, row, np.max(np.abs(s_g - L[r, col]) / tol))
                assert np.all(np.diff(s_g) <= 0), (b, h, row)
                scale = LOGIT_TOL * qn[r] * np.max(n16.astype(np.float64)) / np.sqrt(d)
                assert np.all(L[r, col] >= kth_all[r] - 2 * scale), (b, h, row)
                rest = np.ones(len(pos), dtype=bool)
                rest[col] = False
                assert np.all(L[r, rest] <= s_g[-1] + 2 * scale), (b, h, row)


def test_topk_vector_search_1000_queries_d200(tqm):
    """The vector-search shape: d = 200 (E = F = 64 after padding), one
    sequence of one KV head, 1000 query heads (16 tiles of 64, the last
    ragged), unit rows ~ N(0, diag(1/i)), b = 2 and QJL m = 200, k = 10."""
    n, nq, d, bits, m, pt, k = 40000, 1000, 200, 2, 200, 64, 10
    X = synth.anisotropic_unit(2105, n, d).reshape(1, 1, n, d)
    Q = synth.anisotropic_unit(3105, nq, d)
    cb, cache, bt = _gpu_cache(tqm, X, d, bits, m, pt, [n], 2106)
    s, i = tqm.logits_topk(cb, cache, torch.from_numpy(Q).cuda().view(1, nq, d),
                           torch.tensor([n], dtype=torch.int32, device="cuda"), n, k)
    torch.cuda.synchronize()
    assert cache.errors() == 0
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    _check_topk(codec, O.Layout(d, bits, m, pt, 1), cache.pages.cpu().numpy(), bt,
                Q.astype(np.float64).reshape(1, nq, d), [n], 1, k, s.cpu().numpy(), i.cpu().numpy())


@pytest.mark.parametrize("d,bits,m,pt,G,k,qdtype", [
    (128, 3, 128, 64, 100, 10, "bf16"), (128, 4, 128, 16, 64, 32, "f16"), (128, 1, 0, 256, 70, 5, "f32"),
    (64, 2, 64, 32, 130, 16, "bf16"), (192, 3, 192, 64, 64, 1, "bf16"), (256, 4, 0, 128, 65, 8, "f32")])
def test_topk_shapes_and_ragged_contexts(tqm, d, bits, m, pt, G, k, qdtype):
    """Two sequences x two KV heads with contexts 3001 and 1200 (ragged
    128-key tiles, a shorter sequence inside the longest's tiles), query
    groups of 64-130 (ragged 64-query tiles), every chunk width E = 16..64,
    with and without the sketch, pages of 16-256 tokens, k from 1 to 32."""
    ctx, heads, batch = [3001, 1200], 2, 2
    rng = np.random.default_rng(200 + d + bits)
    X = rng.standard_normal((batch, heads, max(ctx), d)).astype(np.float32)
    X *= np.exp(rng.uniform(-1, 1, size=(1, heads, 1, d))).astype(np.float32)
    cb, cache, bt = _gpu_cache(tqm, X, d, bits, m, pt, ctx, 300 + d)
    qf = rng.standard_normal((batch, heads * G, d)).astype(np.float32)
    Q = synth.to_bf16(qf)[1] if qdtype == "bf16" else qf.astype(np.float16 if qdtype == "f16" else np.float32)
    Q = Q.astype(np.float64)
    s, i = tqm.logits_topk(cb, cache, _q_tensor(Q, qdtype), torch.tensor(ctx, dtype=torch.int32, device="cuda"),
                           max(ctx), k)
    torch.cuda.synchronize()
    assert cache.errors() == 0
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    _check_topk(codec, O.Layout(d, bits, m, pt, heads), cache.pages.cpu().numpy(), bt, Q, ctx, heads, k,
                s.cpu().numpy(), i.cpu().numpy(), sample_rows=min(G, 24))


def test_topk_context_shorter_than_k_and_empty(tqm):
    """A sequence with 5 keys and k = 8 (three empty entries), one with none."""
    d, bits, m, pt, G, k = 128, 3, 128, 64, 64, 8
    ctx, heads, batch = [5, 0], 1, 2
    rng = np.random.default_rng(77)
    X = rng.standard_normal((batch, heads, 64, d)).astype(np.float32)
    cb, cache, bt = _gpu_cache(tqm, X, d, bits, m, pt, ctx, 78)
    Q = synth.to_bf16(rng.standard_normal((batch, heads * G, d)).astype(np.float32))[1].astype(np.float64)
    s, i = tqm.logits_topk(cb, cache, _q_tensor(Q, "bf16"), torch.tensor(ctx, dtype=torch.int32, device="cuda"),
                           64, k)
    torch.cuda.synchronize()
    s, i = s.cpu().numpy(), i.cpu().numpy()
    assert np.all(i[1] == -1) and np.all(np.isneginf(s[1]))
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    _check_topk(codec, O.Layout(d, bits, m, pt, heads), cache.pages.cpu().numpy(), bt, Q[:1], ctx[:1], heads, k,
                s[:1], i[:1])


def test_topk_bad_page_is_skipped_and_reported(tqm):
    """A block-table entry out of range inside the context: the cache's error
    word has the page bit and the page's keys are not ranked."""
    d, bits, m, pt, G, k, n = 128, 3, 128, 32, 64, 10, 2048
    rng = np.random.default_rng(79)
    X = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    cb, cache, bt = _gpu_cache(tqm, X, d, bits, m, pt, [n], 80)
    bad_page = 17
    cache.block_table[0, bad_page] = 10 ** 6
    Q = synth.to_bf16(rng.standard_normal((1, G, d)).astype(np.float32))[1].astype(np.float64)
    s, i = tqm.logits_topk(cb, cache, _q_tensor(Q, "bf16"), torch.tensor([n], dtype=torch.int32, device="cuda"),
                           n, k)
    torch.cuda.synchronize()
    assert cache.errors() & tqm.DEV_ERR_PAGE
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    _check_topk(codec, O.Layout(d, bits, m, pt, 1), cache.pages.cpu().numpy(), bt, Q, [n], 1, k,
                s.cpu().numpy(), i.cpu().numpy(), skip=lambda b, h, pos: (pos // pt) == bad_page)
