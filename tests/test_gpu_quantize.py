"""GPU parity of tq_quantize_append against the fp64 oracle (through the C ABI).

Inputs come from kv_cache_vector_rotate_b200.synth; expected values only from
oracle/.  Tolerances are those of tests/parity.py.
"""

import numpy as np
import pytest

from kv_cache_vector_rotate_b200 import synth
from oracle import tq_oracle as O
from parity import compare_codes, fp16_ulp

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _dev_tensor(bits_or_vals, dtype):
    if dtype == "bf16":
        return torch.from_numpy(bits_or_vals.view(np.int16)).view(torch.bfloat16).cuda()
    if dtype == "f16":
        return torch.from_numpy(bits_or_vals.astype(np.float16)).cuda()
    return torch.from_numpy(bits_or_vals.astype(np.float32)).cuda()


def _run_append(tqm, d, bits, m, x_dev, start_pos, n_pages, page_tokens, bt, cb=None):
    cb = cb or tqm.Codebook(d, bits, m, synth.SEED_PI, synth.SEED_S)
    cache = tqm.PagedCache.allocate(cb, n_pages, page_tokens, x_dev.shape[1], torch.from_numpy(bt))
    tqm.quantize_append(cb, x_dev, torch.tensor(start_pos, dtype=torch.int32, device="cuda"), cache)
    torch.cuda.synchronize()
    return cb, cache


def _read_back(lay, cache, bt, b, h, pos):
    pages = cache.pages.cpu().numpy()
    return O.read_pages(lay, pages, bt, b, h, pos)


@pytest.fixture(scope="module")
def tqm():
    from kv_cache_vector_rotate_b200 import tq as tqmod
    tqmod.load_library()
    return tqmod


def test_tiny_config_fp32_with_outliers(tqm):
    # d = 128, 4096 fp32 keys ~ N(0,1) with 4 outlier channels x20, b = 3 + QJL m = 128.
    K, _, _ = synth.tiny_keys()
    d, bits, m, pt = 128, 3, 128, 64
    bt = synth.block_table(7, 1, 4096 // pt)
    x = torch.from_numpy(K).cuda().view(1, 1, 4096, d)
    cb, cache = _run_append(tqm, d, bits, m, x, [0], 4096 // pt, pt, bt)
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, 1)
    idx, qneg, n16, r16 = _read_back(lay, cache, bt, 0, 0, np.arange(4096))
    ora = O.encode(codec, K.astype(np.float64))
    stats = compare_codes(codec, K.astype(np.float64), ora, idx, qneg, n16, r16)
    assert cache.errors() == 0
    print(stats)


@pytest.mark.parametrize("d,bits,m,dtype", [
    (128, 2, 128, "bf16"), (128, 4, 128, "f16"), (128, 3, 0, "bf16"), (128, 1, 128, "f32"),
    (64, 3, 64, "bf16"), (200, 2, 200, "bf16"), (256, 3, 256, "f32"), (96, 4, 0, "bf16"),
    (192, 3, 192, "bf16"),
])
def test_shapes_bits_dtypes_ragged_midpage(tqm, d, bits, m, dtype):
    batch, heads, n_new, pt = 2, 3, 101, 32
    start = [5, 70]                      # appends that begin inside a page
    pages_per_seq = (max(start) + n_new + pt - 1) // pt
    bt = synth.block_table(11, batch, pages_per_seq)
    rng = np.random.default_rng(12)
    xf = rng.standard_normal((batch, heads, n_new, d)).astype(np.float32) * 3.0
    if dtype == "bf16":
        bits16, vals = synth.to_bf16(xf)
        x = _dev_tensor(bits16, "bf16")
    elif dtype == "f16":
        vals = xf.astype(np.float16).astype(np.float64)
        x = _dev_tensor(vals, "f16")
    else:
        vals = xf.astype(np.float64)
        x = _dev_tensor(vals, "f32")
    cb, cache = _run_append(tqm, d, bits, m, x, start, batch * pages_per_seq, pt, bt)
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, heads)
    for b in range(batch):
        for h in range(heads):
            pos = start[b] + np.arange(n_new)
            idx, qneg, n16, r16 = _read_back(lay, cache, bt, b, h, pos)
            X = vals[b, h]
            compare_codes(codec, X, O.encode(codec, X), idx, qneg, n16, r16)
    # slots before the start positions were never written
    pages = cache.pages.cpu().numpy()
    rec, nrm = O.token_offsets(lay, bt, 1, 0, np.arange(start[1]))
    assert not pages[rec[:, None] + np.arange(lay.code_bytes)[None, :]].any()
    assert cache.errors() == 0


def test_two_appends_equal_one(tqm):
    d, bits, m, pt = 128, 3, 128, 64
    rng = np.random.default_rng(13)
    bits16, vals = synth.to_bf16(rng.standard_normal((1, 2, 127, d)).astype(np.float32))
    bt = synth.block_table(14, 1, 2)
    x = _dev_tensor(bits16, "bf16")
    cb, one = _run_append(tqm, d, bits, m, x, [0], 2, pt, bt)
    two = tqm.PagedCache.allocate(cb, 2, pt, 2, torch.from_numpy(bt))
    tqm.quantize_append(cb, x[:, :, :37].contiguous(), torch.tensor([0], dtype=torch.int32, device="cuda"), two)
    tqm.quantize_append(cb, x[:, :, 37:].contiguous(), torch.tensor([37], dtype=torch.int32, device="cuda"), two)
    torch.cuda.synchronize()
    assert torch.equal(one.pages, two.pages)


def test_zero_vectors_and_norm_overflow(tqm):
    d, bits, m, pt = 128, 3, 128, 16
    x = np.zeros((1, 1, 32, d), np.float32)
    x[0, 0, 1, 3] = 1.0
    x[0, 0, 2, :] = 7000.0        # ||x|| = 79195 > 65504: stored as +inf, error bit set
    bt = np.arange(2, dtype=np.int32).reshape(1, 2)
    cb, cache = _run_append(tqm, d, bits, m, torch.from_numpy(x).cuda(), [0], 2, pt, bt)
    lay = O.Layout(d, bits, m, pt, 1)
    idx, qneg, n16, r16 = _read_back(lay, cache, bt, 0, 0, np.arange(32))
    assert np.all(idx[0] == 4) and float(n16[0]) == 0.0
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    ora = O.encode(codec, x[0, 0].astype(np.float64))
    assert np.array_equal(idx[0], ora.idx[0])
    assert np.isinf(n16[2])
    assert cache.errors() & tqm.DEV_ERR_RANGE


def test_out_of_range_page_is_skipped_and_reported(tqm):
    d, bits, m, pt = 128, 3, 128, 16
    rng = np.random.default_rng(15)
    x = torch.from_numpy(rng.standard_normal((1, 1, 48, d)).astype(np.float32)).cuda()
    bt = np.array([[0, 99, 1]], dtype=np.int32)   # page 99 does not exist (3 pages)
    cb, cache = _run_append(tqm, d, bits, m, x, [0], 3, pt, bt)
    assert cache.errors() & tqm.DEV_ERR_PAGE
    lay = O.Layout(d, bits, m, pt, 1)
    pages = cache.pages.cpu().numpy().reshape(3, lay.page_bytes)
    assert pages[0].any() and pages[1].any() and not pages[2].any()


def test_empty_append_is_a_no_op(tqm):
    cb = tqm.Codebook(128, 3, 128, synth.SEED_PI, synth.SEED_S)
    cache = tqm.PagedCache.allocate(cb, 1, 64, 1, torch.zeros(1, 1, dtype=torch.int32))
    x = torch.zeros(1, 1, 0, 128, dtype=torch.bfloat16, device="cuda")
    tqm.quantize_append(cb, x, torch.zeros(1, dtype=torch.int32, device="cuda"), cache)
    torch.cuda.synchronize()
    assert not cache.pages.any()


@pytest.mark.parametrize("bits,m", [(3, 128), (3, 0), (4, 128), (1, 128)])
def test_prefill_batch_tensor_core_path(tqm, bits, m):
    """A prefill-shaped append (bf16, d = 128, thousands of vectors: the
    tensor-core kernel) against the oracle on every vector of 2 of the 16
    (sequence, head) pairs and on the norms of all of them."""
    d, pt = 128, 64
    batch, heads, n_new = 4, 4, 1024
    rng = np.random.default_rng(16 + bits + m)
    xf = rng.standard_normal((batch, heads, n_new, d)).astype(np.float32)
    xf[rng.random(xf.shape) < 0.01] *= 30.0             # outliers, as in the append workload
    bits16, vals = synth.to_bf16(xf)
    bt = synth.block_table(17, batch, n_new // pt)
    cb, cache = _run_append(tqm, d, bits, m, _dev_tensor(bits16, "bf16"), [0] * batch, batch * n_new // pt, pt, bt)
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, heads)
    for b, h in [(0, 0), (3, 2)]:
        pos = np.arange(n_new)
        idx, qneg, n16, r16 = _read_back(lay, cache, bt, b, h, pos)
        X = vals[b, h]
        compare_codes(codec, X, O.encode(codec, X), idx, qneg, n16, r16)
    for b in range(batch):
        for h in range(heads):
            _, _, n16, _ = _read_back(lay, cache, bt, b, h, np.arange(n_new))
            ref = O.fp16(np.linalg.norm(vals[b, h], axis=-1))
            dn = np.abs(n16.astype(np.float64) - ref.astype(np.float64))
            assert np.all(dn <= fp16_ulp(ref) + 1e-30)     # fp32 vs fp64 sums: within one fp16 ulp
    assert cache.errors() == 0


def test_tensor_core_path_matches_small_appends(tqm):
    """The same 2048 bf16 vectors appended at once (tensor-core kernel) and in
    appends of 8 (CUDA-core kernel) give records that agree except where both
    are within the oracle's windows."""
    d, bits, m, pt = 128, 3, 128, 64
    rng = np.random.default_rng(18)
    bits16, vals = synth.to_bf16(rng.standard_normal((1, 2, 1024, d)).astype(np.float32))
    bt = synth.block_table(19, 1, 1024 // pt)
    x = _dev_tensor(bits16, "bf16")
    cb, big = _run_append(tqm, d, bits, m, x, [0], 1024 // pt, pt, bt)
    small = tqm.PagedCache.allocate(cb, 1024 // pt, pt, 2, torch.from_numpy(bt))
    for s in range(0, 1024, 8):
        tqm.quantize_append(cb, x[:, :, s:s + 8].contiguous(), torch.tensor([s], dtype=torch.int32, device="cuda"),
                            small)
    torch.cuda.synchronize()
    lay = O.Layout(d, bits, m, pt, 2)
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    for h in range(2):
        pos = np.arange(1024)
        a = O.read_pages(lay, big.pages.cpu().numpy(), bt, 0, h, pos)
        c = O.read_pages(lay, small.pages.cpu().numpy(), bt, 0, h, pos)
        ora = O.encode(codec, vals[0, h])
        for got in (a, c):
            compare_codes(codec, vals[0, h], ora, *got)
        same_idx = (a[0] == c[0]).mean()
        assert same_idx > 0.9999


def test_tensor_core_many_tiles_ragged(tqm):
    """4 x 8 x 1999 bf16 vectors: 500 tiles of 128 (the last one 96 rows), so
    each persistent CTA walks 3-4 tiles through both X buffers and both
    tensor-memory Y buffers; 3 (sequence, head) pairs against the oracle,
    every norm within one fp16 ulp."""
    d, bits, m, pt = 128, 3, 128, 64
    batch, heads, n_new = 4, 8, 1999
    rng = np.random.default_rng(26)
    xf = rng.standard_normal((batch, heads, n_new, d)).astype(np.float32)
    xf[rng.random(xf.shape) < 0.01] *= 30.0
    bits16, vals = synth.to_bf16(xf)
    pps = (n_new + pt - 1) // pt
    bt = synth.block_table(27, batch, pps)
    cb, cache = _run_append(tqm, d, bits, m, _dev_tensor(bits16, "bf16"), [0] * batch, batch * pps, pt, bt)
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, heads)
    pages = cache.pages.cpu().numpy()
    for b, h in [(0, 0), (1, 5), (3, 7)]:
        idx, qneg, n16, r16 = O.read_pages(lay, pages, bt, b, h, np.arange(n_new))
        compare_codes(codec, vals[b, h], O.encode(codec, vals[b, h]), idx, qneg, n16, r16)
    for b in range(batch):
        for h in range(heads):
            _, _, n16, _ = O.read_pages(lay, pages, bt, b, h, np.arange(n_new))
            ref = O.fp16(np.linalg.norm(vals[b, h], axis=-1))
            assert np.all(np.abs(n16.astype(np.float64) - ref.astype(np.float64)) <= fp16_ulp(ref) + 1e-30)
    assert cache.errors() == 0


def test_append_workload_full_size_sampled(tqm):
    """The online-append workload at full size (16 x 8 KV heads x 4096 new
    bf16 tokens, 1% outliers x30, 64-token pages, b = 3 + QJL m = 128), in
    the launch the benchmark times: 2048 sampled records against the
    oracle."""
    d, bits, m, pt = 128, 3, 128, 64
    batch, heads, n_new = 16, 8, 4096
    bits16, vals = synth.append_batch(1005, batch, heads, n_new, d)
    pps = n_new // pt
    bt = synth.block_table(1006, batch, pps)
    cb, cache = _run_append(tqm, d, bits, m, _dev_tensor(bits16, "bf16"), [0] * batch, batch * pps, pt, bt)
    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, heads)
    pages = cache.pages.cpu().numpy()
    rng = np.random.default_rng(28)
    X, got = [], [[], [], [], []]
    for _ in range(16):
        b, h = int(rng.integers(batch)), int(rng.integers(heads))
        pos = np.sort(rng.choice(n_new, 128, replace=False))
        for acc, part in zip(got, O.read_pages(lay, pages, bt, b, h, pos)):
            acc.append(part)
        X.append(vals[b, h, pos].astype(np.float64))
    X = np.concatenate(X)
    idx, qneg, n16, r16 = (np.concatenate(a) for a in got)
    compare_codes(codec, X, O.encode(codec, X), idx, qneg, n16, r16)
    assert cache.errors() == 0


def test_bounded_wait_runs_out_and_reports(tqm):
    """The failure path of every streaming kernel: a wait on an mbarrier that
    nothing completes gives up after about a second, reports
    TQ_DEV_ERR_TIMEOUT in the error word and returns (the context stays
    usable: an append afterwards is exact)."""
    import time
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    tqm.selftest_wait_timeout(err)
    torch.cuda.synchronize()
    dt = time.time() - t0
    assert int(err.item()) & tqm.DEV_ERR_TIMEOUT
    assert 0.05 < dt < 30.0, dt
    rng = np.random.default_rng(29)
    bits16, vals = synth.to_bf16(rng.standard_normal((1, 1, 64, 128)).astype(np.float32))
    cb, cache = _run_append(tqm, 128, 3, 128, _dev_tensor(bits16, "bf16"), [0], 1, 64, synth.block_table(30, 1, 1))
    codec = O.make_codec(128, 3, 128, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(128, 3, 128, 64, 1)
    got = _read_back(lay, cache, synth.block_table(30, 1, 1), 0, 0, np.arange(64))
    compare_codes(codec, vals[0, 0], O.encode(codec, vals[0, 0]), *got)
    assert cache.errors() == 0


@pytest.mark.parametrize("kbits,vbits,dtype,batch,heads,n_new", [
    (3, 3, "bf16", 1, 8, 1), (4, 2, "f16", 4, 8, 1), (1, 4, "f32", 3, 4, 5), (2, 1, "bf16", 32, 8, 1),
    (3, 3, "bf16", 2, 8, 64)])
def test_append_kv_equals_two_appends(tqm, kbits, vbits, dtype, batch, heads, n_new):
    """tq_quantize_append_kv (keys b + QJL m = 128, values b without a sketch,
    d = 128) writes the same page bytes as tq_quantize_append of the keys and
    then of the values: decode steps at ragged mid-page positions (one
    launch for both), and a 1024-vector append that takes the two calls.
    The keys of the first case are also checked against the oracle."""
    d, pt = 128, 16
    rng = np.random.default_rng(40 + kbits + 4 * vbits + batch)
    start = rng.integers(0, 200, size=batch).astype(np.int32)
    pps = (int(start.max()) + n_new + pt - 1) // pt
    bt = synth.block_table(41 + batch, batch, pps)
    xs = []
    for _ in range(2):
        xf = rng.standard_normal((batch, heads, n_new, d)).astype(np.float32)
        xf[rng.random(xf.shape) < 0.01] *= 30.0
        if dtype == "bf16":
            bits16, vals = synth.to_bf16(xf)
            xs.append((_dev_tensor(bits16, "bf16"), vals))
        else:
            xs.append((_dev_tensor(xf, dtype), xf.astype(np.float16 if dtype == "f16" else np.float32)))
    (k, kv), (v, _) = xs
    kcb = tqm.Codebook(d, kbits, 128, synth.SEED_PI, synth.SEED_S)
    vcb = tqm.Codebook(d, vbits, 0, synth.SEED_PI, synth.SEED_S)
    sp = torch.from_numpy(start).cuda()
    caches = [tqm.PagedCache.allocate(cb, batch * pps, pt, heads, torch.from_numpy(bt)) for cb in (kcb, vcb) * 2]
    tqm.quantize_append_kv(kcb, k, vcb, v, sp, caches[0], caches[1])
    tqm.quantize_append(kcb, k, sp, caches[2])
    tqm.quantize_append(vcb, v, sp, caches[3])
    torch.cuda.synchronize()
    assert all(c.errors() == 0 for c in caches)
    assert torch.equal(caches[0].pages, caches[2].pages)
    assert torch.equal(caches[1].pages, caches[3].pages)
    if batch == 1 and heads == 8:
        codec = O.make_codec(d, kbits, 128, synth.SEED_PI, synth.SEED_S)
        lay = O.Layout(d, kbits, 128, pt, heads)
        for h in range(heads):
            got = _read_back(lay, caches[0], bt, 0, h, start[0] + np.arange(n_new))
            x64 = kv[0, h].astype(np.float64)
            compare_codes(codec, x64, O.encode(codec, x64), *got)


@pytest.mark.parametrize("km,vm,d", [(0, 0, 128), (128, 128, 128), (64, 0, 64)])
def test_append_kv_other_codebooks_take_two_appends(tqm, km, vm, d):
    """Codebooks the one-launch form does not take (keys without a sketch,
    values with one, d = 64): tq_quantize_append_kv writes what the two
    single-cache appends write."""
    pt, batch, heads = 16, 2, 4
    rng = np.random.default_rng(60 + km + vm + d)
    start = rng.integers(0, 60, size=batch).astype(np.int32)
    pps = (int(start.max()) + 1 + pt - 1) // pt
    bt = synth.block_table(61, batch, pps)
    k = _dev_tensor(synth.to_bf16(rng.standard_normal((batch, heads, 1, d)).astype(np.float32))[0], "bf16")
    v = _dev_tensor(synth.to_bf16(rng.standard_normal((batch, heads, 1, d)).astype(np.float32))[0], "bf16")
    kcb = tqm.Codebook(d, 3, km, synth.SEED_PI, synth.SEED_S)
    vcb = tqm.Codebook(d, 2, vm, synth.SEED_PI, synth.SEED_S)
    sp = torch.from_numpy(start).cuda()
    caches = [tqm.PagedCache.allocate(cb, batch * pps, pt, heads, torch.from_numpy(bt)) for cb in (kcb, vcb) * 2]
    tqm.quantize_append_kv(kcb, k, vcb, v, sp, caches[0], caches[1])
    tqm.quantize_append(kcb, k, sp, caches[2])
    tqm.quantize_append(vcb, v, sp, caches[3])
    torch.cuda.synchronize()
    assert all(c.errors() == 0 for c in caches)
    assert torch.equal(caches[0].pages, caches[2].pages)
    assert torch.equal(caches[1].pages, caches[3].pages)


def test_append_kv_rejects_mismatched_heads(tqm):
    d, pt = 128, 16
    kcb = tqm.Codebook(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    vcb = tqm.Codebook(d, 3, 0, synth.SEED_PI, synth.SEED_S)
    bt = torch.zeros(1, 1, dtype=torch.int32)
    kc = tqm.PagedCache.allocate(kcb, 1, pt, 8, bt)
    vc = tqm.PagedCache.allocate(vcb, 1, pt, 4, bt)
    x = torch.zeros(1, 8, 1, d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tqm.TqError):
        tqm.quantize_append_kv(kcb, x, vcb, x, torch.zeros(1, dtype=torch.int32, device="cuda"), kc, vc)
