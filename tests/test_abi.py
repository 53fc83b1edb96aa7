"""The C-ABI library loads, exports every entry point of include/tq.h, and its
host-side codebook tables agree with the oracle (no GPU needed)."""

import ctypes
import os
import re

import numpy as np
import pytest

from kv_cache_vector_rotate_b200 import tq
from oracle import tq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = tq.load_library()
    names = _header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(tq.EXPORTS)


def test_layout_version():
    assert tq.load_library().tq_layout_version() == 3


@pytest.mark.parametrize("d,bits,m", [(128, 3, 128), (128, 2, 128), (128, 4, 0), (64, 1, 64), (200, 4, 200)])
def test_host_tables_match_oracle(d, bits, m):
    cb = tq.Codebook(d, bits, m, 0x5EED0001, 0x5EED0002, device=False)
    t = cb.export()
    Pi, _, _ = O.rotation(d, 0x5EED0001)
    assert np.max(np.abs(t["pi"] - Pi)) < 1e-12
    if m:
        S = O.qjl_matrix(m, d, 0x5EED0002)
        assert np.max(np.abs(t["s"] - S)) < 1e-13
    ob = O.lloyd_max(d, bits)
    assert np.max(np.abs(t["centroids"] - ob.centroids)) < 1e-12
    assert np.max(np.abs(t["boundaries"] - ob.boundaries)) < 1e-12
    assert np.array_equal(O.fp16(t["centroids"]), O.fp16(ob.centroids))


@pytest.mark.parametrize("d,bits,m,pt,h", [(128, 3, 128, 64, 8), (128, 3, 0, 64, 8), (128, 2, 128, 32, 2),
                                           (128, 4, 128, 64, 1), (200, 2, 200, 64, 1), (64, 1, 64, 16, 3)])
def test_layout_sizes_match_oracle(d, bits, m, pt, h):
    cb = tq.Codebook(d, bits, m, 1, 2, device=False)
    info = cb.layout(pt, h)
    lay = O.Layout(d, bits, m, pt, h)
    assert info.d_pad == lay.d_pad and info.words_per_chunk == lay.words
    assert info.code_bytes == lay.code_bytes and info.norm_bytes == lay.norm_bytes
    assert info.head_block_bytes == lay.head_block_bytes and info.page_bytes == lay.page_bytes


@pytest.mark.parametrize("d,bits,m,status", [(100, 3, 128, tq.TQ_EINVAL), (128, 5, 128, tq.TQ_EUNSUPPORTED),
                                             (128, 0, 128, tq.TQ_EUNSUPPORTED), (264, 3, 0, tq.TQ_EINVAL),
                                             (128, 3, 64, tq.TQ_EUNSUPPORTED), (128, 3, -1, tq.TQ_EINVAL)])
def test_bad_params_rejected_on_host(d, bits, m, status):
    with pytest.raises(tq.TqError) as e:
        tq.Codebook(d, bits, m, 1, 2, device=False)
    assert e.value.status == status
    assert tq.load_library().tq_last_error()


def test_host_only_codebook_refuses_kernels():
    cb = tq.Codebook(128, 3, 128, 1, 2, device=False)
    lib = tq.load_library()
    cs = tq.CacheStruct(None, 1, 64, 1, None, 1, None)
    st = lib.tq_quantize_append(cb.handle, None, 0, 1, 1, 1, None, ctypes.byref(cs), None)
    assert st == tq.TQ_EINVAL
    assert b"host-only" in lib.tq_last_error()


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_reconstruction_levels_match_oracle_for_every_supported_d(bits):
    # The levels the kernels decode with (8-bit fixed point for b <= 3, fp16
    # for b = 4), built by the library's host code, equal the oracle's
    # reconstruction_levels of its own Lloyd-Max centroids, scale included.
    for d in range(8, 257, 8):
        cb = tq.Codebook(d, bits, 0, 3, 4, device=False)
        lev, f = cb.levels()
        ref, fr = O.reconstruction_levels(O.lloyd_max(d, bits).centroids)
        cb.close()
        assert f == fr, d
        assert np.array_equal(lev, ref), d


def test_attend_workspace_covers_both_paths():
    # tq_attend's workspace covers its two paths (the page sizes, which pick
    # the path, are not arguments): the composed path's fp32 scores [batch,
    # n_q_heads, max_ctx] then the logits and values workspaces, and the
    # fused path's query fragments then fp32 partials [n_cta][2][4][4E + 2],
    # n_cta = the largest grid over page sizes 16 .. 1024 (CTAs: at least one
    # per SM -- 148 without a GPU -- and per line, at most 127 units each for
    # 16-token pages, at most one per unit); each part rounded up to 256 bytes.
    kcb = tq.Codebook(128, 3, 128, 1, 2, device=False)
    vcb = tq.Codebook(128, 3, 0, 3, 4, device=False)
    lib = tq.load_library()
    al = lambda n: (n + 255) // 256 * 256
    for batch, hkv, hq, ctx in [(1, 8, 32, 32768), (3, 2, 8, 700), (2, 4, 4, 17), (1, 1, 4, 10 ** 6)]:
        composed = (al(batch * hq * ctx * 4) + al(lib.tq_logits_workspace_bytes(kcb.handle, batch, hkv, hq))
                    + al(lib.tq_values_workspace_bytes(vcb.handle, batch, hkv, hq, ctx)))
        lines = batch * hkv * ((hq // hkv + 3) // 4)
        items = lines * ((ctx + 63) // 64)
        n_cta = max(1, min(max(148, lines, -(-items // 127)), items))
        fused = al(lib.tq_logits_workspace_bytes(kcb.handle, batch, hkv, hq)) + al(n_cta * 2 * 4 * 130 * 4)
        assert lib.tq_attend_workspace_bytes(kcb.handle, vcb.handle, batch, hkv, hq, ctx) == max(composed, fused)
    for args in [(1, 8, 30, 64), (1, 0, 8, 64), (-1, 2, 8, 64), (1, 2, 8, -1)]:
        assert lib.tq_attend_workspace_bytes(kcb.handle, vcb.handle, *args) == 0
    assert lib.tq_attend_workspace_bytes(None, vcb.handle, 1, 2, 8, 64) == 0


def test_attend_refuses_host_only_codebooks():
    kcb = tq.Codebook(128, 3, 128, 1, 2, device=False)
    vcb = tq.Codebook(128, 3, 0, 3, 4, device=False)
    lib = tq.load_library()
    cs = tq.CacheStruct(None, 1, 64, 1, None, 1, None)
    st = lib.tq_attend(kcb.handle, ctypes.byref(cs), vcb.handle, ctypes.byref(cs), None, 0, 1, 4, None, 64,
                       0.1, None, None, 0, None)
    assert st == tq.TQ_EINVAL
    assert b"host-only" in lib.tq_last_error()


@pytest.mark.parametrize("level", [1, 2, 3, 5, 7, 8])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_polar_angle_tables_match_oracle(level, bits):
    from oracle import polar_oracle as P
    c, t, dist = tq.polar_angle_codebook(level, bits)
    ref = P.angle_lloyd_max(level, bits)
    assert np.allclose(c, ref.centroids, rtol=0, atol=1e-11)
    assert np.allclose(t, ref.boundaries, rtol=0, atol=1e-11)
    assert abs(dist - ref.distortion) <= 1e-12 + 1e-9 * ref.distortion


def test_polar_angle_codebook_refuses_bad_arguments():
    lib = tq.load_library()
    buf = (ctypes.c_double * 512)()
    assert lib.tq_polar_angle_codebook(0, 2, buf, None, None) == tq.TQ_EINVAL
    assert lib.tq_polar_angle_codebook(9, 2, buf, None, None) == tq.TQ_EINVAL
    assert lib.tq_polar_angle_codebook(2, 9, buf, None, None) == tq.TQ_EUNSUPPORTED
    assert lib.tq_polar_angle_codebook(2, 2, None, None, None) == tq.TQ_EINVAL
