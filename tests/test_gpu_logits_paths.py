"""GPU parity of tq_logits against the fp64 oracle on the logits kernel's
work-division paths: CTAs whose share spans two (sequence, head) lines,
CTAs with more units than copy slots (slot refills), CTAs of 4 warps when
the work is small, units that straddle pages (16-token pages), pages of
up to 256 tokens, every bit width with and without the sketch, GQA groups of
1 - 8 queries, bf16 / fp16 / fp32 queries, and bad block-table entries.
Caches are written by the oracle; tolerances are those of tests/parity.py.
"""

import numpy as np
import pytest

from gpu_cases import _check_logits, _oracle_cache, _q_tensor
from kv_cache_vector_rotate_b200 import synth
from oracle import tq_oracle as O
from parity import LOGIT_TOL, logit_error

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tqm():
    from kv_cache_vector_rotate_b200 import tq as tqmod
    tqmod.load_library()
    return tqmod


def _queries(rng, batch, hq, d, dtype):
    qf = rng.standard_normal((batch, hq, d)).astype(np.float32)
    if dtype == "bf16":
        return synth.to_bf16(qf)[1]
    if dtype == "f16":
        return qf.astype(np.float16).astype(np.float64)
    return qf.astype(np.float64)


@pytest.mark.parametrize("d,bits,m,G,dtype,pt", [
    (128, 3, 128, 4, "bf16", 64), (128, 2, 128, 4, "bf16", 32), (128, 4, 128, 4, "f16", 64),
    (128, 1, 128, 2, "f32", 16), (128, 3, 0, 4, "bf16", 256), (64, 3, 64, 5, "bf16", 64),
    (64, 4, 0, 8, "f32", 16), (128, 3, 128, 1, "bf16", 64), (128, 2, 0, 3, "f16", 128),
    (96, 3, 96, 4, "bf16", 32),
])
def test_ragged_context_shapes(tqm, d, bits, m, G, dtype, pt):
    batch, heads = 2, 2
    ctx = [1000, 333]
    rng = np.random.default_rng(60 + d + bits + m + G)
    keys = rng.standard_normal((batch, heads, max(ctx), d)) * np.exp(rng.uniform(-2, 2, size=(1, heads, 1, d)))
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, heads)
    cb, cache, encs, _ = _oracle_cache(tqm, codec, lay, keys, ctx, pt, 61)
    q = _queries(rng, batch, heads * G, d, dtype)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    out = torch.full((batch, heads * G, max(ctx)), float("nan"), device="cuda")
    tqm.logits(cb, cache, _q_tensor(q, dtype), ctx_t, max(ctx), out=out)
    torch.cuda.synchronize()
    L = out.cpu().numpy()
    _check_logits(codec, q, encs, L, ctx, heads, G)
    assert np.all(np.isnan(L[1, :, ctx[1]:]))          # positions past ctx_len untouched
    assert cache.errors() == 0


def test_many_units_per_cta(tqm):
    # 2 sequences x 8 KV heads x 8192 keys: ~110 units per CTA, so every warp
    # refills its copy slots (more units than slots)
    batch, heads, G, pt, d = 2, 8, 4, 64, 128
    ctx = [8192, 7777]
    rng = np.random.default_rng(70)
    keys = rng.standard_normal((batch, heads, max(ctx), d))
    codec = O.make_codec(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, 3, 128, pt, heads)
    cb, cache, encs, _ = _oracle_cache(tqm, codec, lay, keys, ctx, pt, 71)
    q = _queries(rng, batch, heads * G, d, "bf16")
    L = tqm.logits(cb, cache, _q_tensor(q, "bf16"), torch.tensor(ctx, dtype=torch.int32, device="cuda"), max(ctx))
    torch.cuda.synchronize()
    _check_logits(codec, q, encs, L.cpu().numpy(), ctx, heads, G)
    assert cache.errors() == 0


def test_bad_page_is_skipped_and_reported(tqm):
    # one block-table entry inside the context points past the cache: its
    # positions are not written, the error word says so, the rest is exact
    batch, heads, G, pt, d = 1, 2, 4, 32, 128
    ctx = [2048]
    rng = np.random.default_rng(72)
    keys = rng.standard_normal((batch, heads, ctx[0], d))
    codec = O.make_codec(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, 3, 128, pt, heads)
    cb, cache, encs, bt = _oracle_cache(tqm, codec, lay, keys, ctx, pt, 73)
    bad_page = 17
    bt_bad = bt.copy()
    bt_bad[0, bad_page] = 10 ** 6
    cache.block_table.copy_(torch.from_numpy(bt_bad))
    q = _queries(rng, batch, heads * G, d, "bf16")
    out = torch.full((batch, heads * G, ctx[0]), float("nan"), device="cuda")
    tqm.logits(cb, cache, _q_tensor(q, "bf16"), torch.tensor(ctx, dtype=torch.int32, device="cuda"), ctx[0],
               out=out)
    torch.cuda.synchronize()
    assert cache.errors() & tqm.DEV_ERR_PAGE
    L = out.cpu().numpy()
    lo, hi = bad_page * pt, (bad_page + 1) * pt
    assert np.all(np.isnan(L[0, :, lo:hi]))
    keep = np.r_[0:lo, hi:ctx[0]]
    for (b, h), (pos, enc) in encs.items():
        Qg = q[b, h * G:(h + 1) * G]
        Lo = O.logits_from_codes(codec, Qg, enc.idx[keep], enc.qneg[keep], enc.norm16[keep], enc.rnorm16[keep])
        err = logit_error(L[b, h * G:(h + 1) * G][:, keep], Lo, np.linalg.norm(Qg, axis=1), enc.norm16[keep], d)
        assert err <= LOGIT_TOL, err


def test_wide_ctas_ragged_groups_lines_bad_page(tqm):
    """About 34 units per CTA (15 consumer warps, two-launch form): 2
    sequences x 4 KV heads x 6 query heads (a ragged second query tile),
    contexts 20000 and 13000 (the second sequence's lines end early), CTA
    shares that straddle lines, and one out-of-range block-table entry."""
    batch, heads, G, pt, d = 2, 4, 6, 64, 128
    ctx = [20000, 13000]
    rng = np.random.default_rng(74)
    keys = rng.standard_normal((batch, heads, max(ctx), d)) * np.exp(rng.uniform(-1, 1, size=(1, heads, 1, d)))
    codec = O.make_codec(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, 3, 128, pt, heads)
    cb, cache, encs, bt = _oracle_cache(tqm, codec, lay, keys, ctx, pt, 75)
    bad_page = 40
    bt_bad = bt.copy()
    bt_bad[1, bad_page] = 10 ** 6
    cache.block_table.copy_(torch.from_numpy(bt_bad))
    q = _queries(rng, batch, heads * G, d, "bf16")
    out = torch.full((batch, heads * G, max(ctx)), float("nan"), device="cuda")
    tqm.logits(cb, cache, _q_tensor(q, "bf16"), torch.tensor(ctx, dtype=torch.int32, device="cuda"), max(ctx),
               out=out)
    torch.cuda.synchronize()
    assert cache.errors() & tqm.DEV_ERR_PAGE
    L = out.cpu().numpy()
    lo, hi = bad_page * pt, (bad_page + 1) * pt
    assert np.all(np.isnan(L[1, :, lo:hi]))
    assert np.all(np.isnan(L[1, :, ctx[1]:]))
    for (b, h), (pos, enc) in encs.items():
        keep = np.arange(ctx[b]) if b == 0 else np.r_[0:lo, hi:ctx[b]]
        Qg = q[b, h * G:(h + 1) * G]
        Lo = O.logits_from_codes(codec, Qg, enc.idx[keep], enc.qneg[keep], enc.norm16[keep], enc.rnorm16[keep])
        err = logit_error(L[b, h * G:(h + 1) * G][:, keep], Lo, np.linalg.norm(Qg, axis=1), enc.norm16[keep], d)
        assert err <= LOGIT_TOL, (b, h, err)
