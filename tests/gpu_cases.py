"""Case builders shared by the GPU parity tests of the logits path: caches
written by the ORACLE (oracle/ packs the records) and read by the GPU
through the C ABI, and the logit check against the oracle estimator given
identical codes (tolerances of tests/parity.py)."""

import numpy as np
import torch

from kv_cache_vector_rotate_b200 import synth
from oracle import tq_oracle as O
from parity import LOGIT_TOL, logit_error, oracle_pages


def _oracle_cache(tqm, codec, lay, keys, ctx, pt, seed):
    """keys [batch, heads, ctx_max, d] float64; ctx [batch] -> (cb, cache, encs, bt)."""
    batch, heads, cmax, d = keys.shape
    pps = (cmax + pt - 1) // pt
    bt = synth.block_table(seed, batch, pps)
    encs = {}
    for b in range(batch):
        for h in range(heads):
            pos = np.arange(ctx[b])
            encs[(b, h)] = (pos, O.encode(codec, keys[b, h, : ctx[b]]))
    pages = oracle_pages(lay, batch * pps, bt, encs)
    cb = tqm.Codebook(codec.d, codec.bits, codec.m, synth.SEED_PI, synth.SEED_S)
    cache = tqm.PagedCache.allocate(cb, batch * pps, pt, heads, torch.from_numpy(bt))
    cache.pages.copy_(torch.from_numpy(pages))
    return cb, cache, encs, bt


def _q_tensor(q_vals, dtype):
    t = torch.from_numpy(q_vals.astype(np.float32)).cuda()
    return t.to({"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dtype])


def _check_logits(codec, q, encs, L_gpu, ctx, heads, G):
    worst = 0.0
    for (b, h), (pos, enc) in encs.items():
        Qg = q[b, h * G:(h + 1) * G]
        L = O.logits_from_codes(codec, Qg, enc.idx, enc.qneg, enc.norm16, enc.rnorm16)
        err = logit_error(L_gpu[b, h * G:(h + 1) * G, : ctx[b]], L, np.linalg.norm(Qg, axis=1),
                          enc.norm16, codec.d)
        worst = max(worst, err)
    assert worst <= LOGIT_TOL, worst
    return worst
