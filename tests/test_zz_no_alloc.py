"""tq_logits_noalloc (through the C ABI) against tq_logits.

Some callers cannot allocate device memory where they call the library: a
serving loop whose memory is an arena carved up at start-up, a framework or
plugin interface that gives an operator no workspace, or a hot path that must
not call cudaMalloc/cudaFree because they can block or synchronize the
device.  tq_logits_noalloc serves them from a static 1 MiB device array.  This
file is collected after the kernels' parity tests on purpose; it passes alone
in a fresh process and after the other tests.
"""

import ctypes

import numpy as np
import pytest

from kv_cache_vector_rotate_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

LOGIT_TOL = 1e-3     # the relative tolerance of the other logits tests


def _close(a, b, q, knorm_max, d):
    scale = torch.maximum(b.abs(), (q.float().norm(dim=-1, keepdim=True) * knorm_max / np.sqrt(d)))
    return bool(torch.all((a - b).abs() <= LOGIT_TOL * scale))


def test_noalloc_matches_tq_logits_twice_in_a_row():
    from kv_cache_vector_rotate_b200 import tq
    tq.load_library()
    batch, hkv, G, d, pt = 2, 2, 4, 128, 64
    ctx = [700, 257]
    rng = np.random.default_rng(41)
    kbits, kvals = synth.to_bf16(rng.standard_normal((batch, hkv, max(ctx), d)).astype(np.float32) * 2)
    K = torch.from_numpy(kbits.view(np.int16)).view(torch.bfloat16).cuda()
    pps = (max(ctx) + pt - 1) // pt
    cb = tq.Codebook(d, 3, 128, synth.SEED_PI, synth.SEED_S)
    cache = tq.PagedCache.allocate(cb, batch * pps, pt, hkv, torch.from_numpy(synth.block_table(42, batch, pps)))
    tq.quantize_append(cb, K, torch.zeros(batch, dtype=torch.int32, device="cuda"), cache)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    knorm_max = float(np.linalg.norm(kvals, axis=-1).max())
    for call in range(2):
        _, qv = synth.to_bf16(rng.standard_normal((batch, hkv * G, d)).astype(np.float32))
        q = torch.from_numpy(qv.astype(np.float32)).cuda().to(torch.bfloat16)
        ref = tq.logits(cb, cache, q, ctx_t, max(ctx))
        got = torch.full_like(ref, float("nan"))
        tq.logits_noalloc(cb, cache, q, ctx_t, max(ctx), out=got)
        torch.cuda.synchronize()
        for b in range(batch):
            assert _close(got[b, :, : ctx[b]], ref[b, :, : ctx[b]], q[b], knorm_max, d), call
            assert torch.all(torch.isnan(got[b, :, ctx[b]:]))
    assert cache.errors() == 0


def test_noalloc_rejects_requests_beyond_the_static_scratch():
    from kv_cache_vector_rotate_b200 import tq
    lib = tq.load_library()
    limit = lib.tq_logits_noalloc_scratch_bytes()
    assert limit == 1 << 20
    cb = tq.Codebook(128, 3, 128, synth.SEED_PI, synth.SEED_S)
    batch = 4096                   # 4096 x 8 KV heads of query fragments: well over 1 MiB
    assert tq.logits_workspace_bytes(cb, batch, 8, 32) > limit
    cache = tq.PagedCache.allocate(cb, 1, 64, 8, torch.zeros(batch, 1, dtype=torch.int32))
    q = torch.zeros(batch, 32, 128, dtype=torch.bfloat16, device="cuda")
    ctx_t = torch.zeros(batch, dtype=torch.int32, device="cuda")
    out = torch.zeros(batch, 32, 64, device="cuda")
    cs = cache.struct()
    st = lib.tq_logits_noalloc(cb.handle, ctypes.byref(cs), q.data_ptr(), tq.TQ_BF16, batch, 32,
                               ctx_t.data_ptr(), 64, out.data_ptr(), 64, None)
    assert st == tq.TQ_EINVAL
    assert b"static scratch" in lib.tq_last_error()
