"""Vector search from the codes (TQ §Benchmarks: nearest-neighbour search at
d = 200, top-10 recall against exact brute force).

Synthetic stand-in for the page's GloVe d = 200 evaluation (not available
here): unit rows ~ N(0, diag(1/i)) from kv_cache_vector_rotate_b200.synth. The
database is one sequence of one KV head; the queries are its query heads, so
the scores are tq_logits from the packed records (d = 200 pads to 256: the
E = F = 64 kernels). Checked here: the records against the oracle's encoding,
the scores against the oracle's logits given the GPU's codes, and recall@10
of the code scores against the fp64 brute-force top 10.
"""

import numpy as np
import pytest

from kv_cache_vector_rotate_b200 import synth
from oracle import tq_oracle as O
from parity import LOGIT_TOL, compare_codes, logit_error

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

RECALL = {}


@pytest.fixture(scope="module")
def tqm():
    from kv_cache_vector_rotate_b200 import tq as tqmod
    tqmod.load_library()
    return tqmod


@pytest.mark.parametrize("bits", [2, 4])
def test_search_codes_scores_and_recall(tqm, bits):
    n, nq, d, m, pt = 98304, 64, 200, 200, 64
    X = synth.anisotropic_unit(2005, n, d)
    Q = synth.anisotropic_unit(3005, nq, d)
    cb = tqm.Codebook(d, bits, m, synth.SEED_PI, synth.SEED_S)
    pps = n // pt
    bt = synth.block_table(2006, 1, pps)
    cache = tqm.PagedCache.allocate(cb, pps, pt, 1, torch.from_numpy(bt))
    tqm.quantize_append(cb, torch.from_numpy(X).cuda().view(1, 1, n, d),
                        torch.zeros(1, dtype=torch.int32, device="cuda"), cache)
    L = tqm.logits(cb, cache, torch.from_numpy(Q).cuda().view(1, nq, d),
                   torch.tensor([n], dtype=torch.int32, device="cuda"), n)
    torch.cuda.synchronize()
    assert cache.errors() == 0
    scores = L[0].cpu().numpy()

    codec = O.make_codec(d, bits, m, synth.SEED_PI, synth.SEED_S)
    lay = O.Layout(d, bits, m, pt, 1)
    rng = np.random.default_rng(2007)
    pos = np.sort(rng.choice(n, 1024, replace=False))
    idx, qneg, n16, r16 = O.read_pages(lay, cache.pages.cpu().numpy(), bt, 0, 0, pos)
    Xs = X[pos].astype(np.float64)
    compare_codes(codec, Xs, O.encode(codec, Xs), idx, qneg, n16, r16)
    Q64 = Q.astype(np.float64)
    Lo = O.logits_from_codes(codec, Q64, idx, qneg, n16, r16)
    assert logit_error(scores[:, pos], Lo, np.linalg.norm(Q64, axis=1), n16, d) <= LOGIT_TOL

    exact = Q64 @ X.astype(np.float64).T                       # [nq, n]
    top_exact = np.argpartition(-exact, 10, axis=1)[:, :10]
    top_codes = np.argpartition(-scores, 10, axis=1)[:, :10]
    recall = np.mean([len(set(a) & set(b)) / 10 for a, b in zip(top_exact, top_codes)])
    best = np.argmax(exact, axis=1)
    one_at_10 = np.mean([best[i] in set(top_codes[i]) for i in range(nq)])
    RECALL[bits] = recall
    print(f"b={bits}: recall@10 {recall:.3f}, 1@10 {one_at_10:.3f}")
    assert recall >= {2: 0.35, 4: 0.70}[bits], recall
    assert one_at_10 >= {2: 0.60, 4: 0.90}[bits], one_at_10


def test_search_recall_grows_with_bits():
    if len(RECALL) < 2:
        pytest.skip("needs both bit widths of the search test")
    assert RECALL[4] > RECALL[2]
