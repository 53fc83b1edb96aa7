"""Python binding of libtq (include/tq.h): argument marshalling only.

Every step of the codec runs inside libtq's CUDA kernels; this module turns
torch tensors into device pointers and the current CUDA stream into the
stream argument, and raises on a non-zero status.  If libtq.so is missing the
import of the library fails loudly: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libtq.so")

TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ERANGE, TQ_ETIMEOUT, TQ_ECUDA, TQ_ENOMEM = range(7)
TQ_BF16, TQ_F16, TQ_F32 = 0, 1, 2
DEV_ERR_PAGE, DEV_ERR_RANGE, DEV_ERR_TIMEOUT, DEV_ERR_CONFIG = 1, 2, 4, 8

# Every entry point declared in include/tq.h.
EXPORTS = (
    "tq_codebook_build", "tq_codebook_build_host", "tq_codebook_free", "tq_codebook_export",
    "tq_layout", "tq_quantize_append", "tq_logits_workspace_bytes", "tq_logits",
    "tq_values_workspace_bytes", "tq_dequant_values", "tq_last_error", "tq_layout_version",
    "tq_logits_noalloc", "tq_logits_noalloc_scratch_bytes", "tq_selftest_wait_timeout",
    "tq_logits_topk_workspace_bytes", "tq_logits_topk",
    "tq_quantize_append_kv", "tq_polar_build", "tq_polar_free", "tq_polar_record_bytes", "tq_polar_encode",
    "tq_polar_logits_workspace_bytes", "tq_polar_logits",
    "tq_attend_workspace_bytes", "tq_attend", "tq_polar_angle_codebook", "tq_codebook_levels",
)


class TqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libtq status {status}: {msg}")
        self.status = status


class Params(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("bits", ctypes.c_int32), ("m", ctypes.c_int32),
                ("seed_pi", ctypes.c_uint64), ("seed_s", ctypes.c_uint64)]


class LayoutInfo(ctypes.Structure):
    _fields_ = [("d_pad", ctypes.c_int32), ("m_pad", ctypes.c_int32),
                ("words_per_chunk", ctypes.c_int32), ("code_bytes", ctypes.c_int32),
                ("norm_bytes", ctypes.c_int32), ("head_block_bytes", ctypes.c_int32),
                ("page_bytes", ctypes.c_int64)]


class CacheStruct(ctypes.Structure):
    _fields_ = [("pages", ctypes.c_void_p), ("n_pages", ctypes.c_int64),
                ("page_tokens", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("block_table", ctypes.c_void_p), ("max_pages_per_seq", ctypes.c_int64),
                ("error_word", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libtq.so and declares the C signatures (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m kv_cache_vector_rotate_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    dp = ctypes.POINTER(ctypes.c_double)
    sig = {
        "tq_codebook_build": (i32, [ctypes.POINTER(Params), ctypes.POINTER(vp)]),
        "tq_codebook_build_host": (i32, [ctypes.POINTER(Params), ctypes.POINTER(vp)]),
        "tq_codebook_free": (None, [vp]),
        "tq_codebook_export": (i32, [vp, dp, dp, dp, dp]),
        "tq_codebook_levels": (i32, [vp, dp, ctypes.POINTER(i32)]),
        "tq_layout": (i32, [vp, i32, i32, ctypes.POINTER(LayoutInfo)]),
        "tq_quantize_append": (i32, [vp, vp, i32, i64, i32, i64, vp, ctypes.POINTER(CacheStruct), vp]),
        "tq_logits_workspace_bytes": (sz, [vp, i64, i32, i32]),
        "tq_logits": (i32, [vp, ctypes.POINTER(CacheStruct), vp, i32, i64, i32, vp, i64, vp, i64, vp, sz, vp]),
        "tq_values_workspace_bytes": (sz, [vp, i64, i32, i32, i64]),
        "tq_dequant_values": (i32, [vp, ctypes.POINTER(CacheStruct), vp, i64, i64, i32, vp, i64,
                                    vp, i32, i64, vp, sz, vp]),
        "tq_logits_noalloc": (i32, [vp, ctypes.POINTER(CacheStruct), vp, i32, i64, i32, vp, i64, vp, i64, vp]),
        "tq_logits_noalloc_scratch_bytes": (sz, []),
        "tq_logits_topk_workspace_bytes": (sz, [vp, i64, i32, i32, i64, i32]),
        "tq_quantize_append_kv": (i32, [vp, vp, vp, vp, i32, i64, i32, i64, vp, ctypes.POINTER(CacheStruct),
                                        ctypes.POINTER(CacheStruct), vp]),
        "tq_polar_build": (i32, [i32, i32, i32, ctypes.c_uint64, ctypes.c_uint64, ctypes.POINTER(vp)]),
        "tq_polar_free": (None, [vp]),
        "tq_polar_record_bytes": (i32, [vp]),
        "tq_polar_encode": (i32, [vp, vp, i32, i64, vp, vp, vp]),
        "tq_polar_logits_workspace_bytes": (sz, [vp, i32]),
        "tq_polar_logits": (i32, [vp, vp, i64, vp, i32, i32, vp, i64, vp, sz, vp]),
        "tq_logits_topk": (i32, [vp, ctypes.POINTER(CacheStruct), vp, i32, i64, i32, vp, i64, i32, vp, vp, vp, sz,
                                 vp]),
        "tq_selftest_wait_timeout": (i32, [vp, vp]),
        "tq_attend_workspace_bytes": (sz, [vp, vp, i64, i32, i32, i64]),
        "tq_attend": (i32, [vp, ctypes.POINTER(CacheStruct), vp, ctypes.POINTER(CacheStruct), vp, i32, i64, i32,
                            vp, i64, ctypes.c_float, vp, vp, sz, vp]),
        "tq_polar_angle_codebook": (i32, [i32, i32, vp, vp, vp]),
        "tq_last_error": (ctypes.c_char_p, []),
        "tq_layout_version": (i32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != TQ_OK:
        raise TqError(status, load_library().tq_last_error().decode())


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _dtype_code(t) -> int:
    import torch
    codes = {torch.bfloat16: TQ_BF16, torch.float16: TQ_F16, torch.float32: TQ_F32}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _stream(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class Codebook:
    """Handle of tq_codebook: Pi, S and the Lloyd-Max tables for (d, bits, m)."""

    def __init__(self, d: int, bits: int, m: int, seed_pi: int, seed_s: int, device: bool = True):
        lib = load_library()
        self.d, self.bits, self.m = d, bits, m
        self.seed_pi, self.seed_s = seed_pi, seed_s
        self._p = Params(d, bits, m, seed_pi, seed_s)
        h = ctypes.c_void_p()
        fn = lib.tq_codebook_build if device else lib.tq_codebook_build_host
        _check(fn(ctypes.byref(self._p), ctypes.byref(h)))
        self.handle = h

    def close(self) -> None:
        if getattr(self, "handle", None):
            load_library().tq_codebook_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def export(self):
        import numpy as np
        K = 1 << self.bits
        pi = np.zeros(self.d * self.d)
        s = np.zeros(max(self.m, 1) * self.d)
        c = np.zeros(K)
        t = np.zeros(K - 1)
        dp = ctypes.POINTER(ctypes.c_double)
        _check(load_library().tq_codebook_export(
            self.handle, pi.ctypes.data_as(dp), s.ctypes.data_as(dp), c.ctypes.data_as(dp),
            t.ctypes.data_as(dp)))
        return {"pi": pi.reshape(self.d, self.d), "s": s[: self.m * self.d].reshape(self.m, self.d),
                "centroids": c, "boundaries": t}

    def levels(self):
        """tq_codebook_levels: (reconstruction levels, scale exponent f or None)."""
        import numpy as np
        lev = np.zeros(1 << self.bits)
        f = ctypes.c_int32(0)
        _check(load_library().tq_codebook_levels(self.handle, lev.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                                 ctypes.byref(f)))
        return lev, (None if f.value == -(1 << 31) else f.value)

    def layout(self, page_tokens: int, n_kv_heads: int) -> LayoutInfo:
        info = LayoutInfo()
        _check(load_library().tq_layout(self.handle, page_tokens, n_kv_heads, ctypes.byref(info)))
        return info


@dataclass
class PagedCache:
    """Caller-owned paged cache (torch device tensors) in the tq_cache form."""

    pages: object           # torch.uint8 [n_pages * page_bytes]
    n_pages: int
    page_tokens: int
    n_kv_heads: int
    block_table: object     # torch.int32 [batch, max_pages_per_seq]
    error_word: object      # torch.int32 [1] (bits of TQ_DEV_ERR_*)

    @staticmethod
    def allocate(cb: Codebook, n_pages: int, page_tokens: int, n_kv_heads: int, block_table, device="cuda"):
        import torch
        info = cb.layout(page_tokens, n_kv_heads)
        pages = torch.zeros(n_pages * info.page_bytes, dtype=torch.uint8, device=device)
        err = torch.zeros(1, dtype=torch.int32, device=device)
        bt = block_table.to(device=device, dtype=torch.int32).contiguous()
        return PagedCache(pages, n_pages, page_tokens, n_kv_heads, bt, err)

    def struct(self) -> CacheStruct:
        return CacheStruct(self.pages.data_ptr(), self.n_pages, self.page_tokens, self.n_kv_heads,
                           self.block_table.data_ptr(), self.block_table.shape[1],
                           self.error_word.data_ptr())

    def errors(self) -> int:
        return int(self.error_word.item()) & 0xFFFFFFFF


def quantize_append(cb: Codebook, x, start_pos, cache: PagedCache, stream=None) -> None:
    """tq_quantize_append: x [batch, n_kv_heads, n_new, d] -> records in `cache`."""
    assert x.is_cuda and x.is_contiguous() and x.dim() == 4
    b, h, n, d = x.shape
    assert d == cb.d
    cs = cache.struct()
    _check(load_library().tq_quantize_append(cb.handle, _ptr(x), _dtype_code(x), b, h, n,
                                              _ptr(start_pos), ctypes.byref(cs), _stream(stream)))


def quantize_append_kv(key_cb: Codebook, k, value_cb: Codebook, v, start_pos, key_cache: PagedCache,
                       value_cache: PagedCache, stream=None) -> None:
    """tq_quantize_append_kv: the keys k and the values v [batch, n_kv_heads, n_new, d]
    of one cache update, into their two caches."""
    assert k.is_cuda and k.is_contiguous() and k.dim() == 4 and v.is_cuda and v.is_contiguous()
    assert k.shape == v.shape and k.dtype == v.dtype
    b, h, n, d = k.shape
    assert d == key_cb.d and d == value_cb.d
    ks, vs = key_cache.struct(), value_cache.struct()
    _check(load_library().tq_quantize_append_kv(key_cb.handle, _ptr(k), value_cb.handle, _ptr(v), _dtype_code(k),
                                                 b, h, n, _ptr(start_pos), ctypes.byref(ks), ctypes.byref(vs),
                                                 _stream(stream)))


def logits_workspace_bytes(cb: Codebook, batch: int, n_kv_heads: int, n_q_heads: int) -> int:
    return int(load_library().tq_logits_workspace_bytes(cb.handle, batch, n_kv_heads, n_q_heads))


def logits(cb: Codebook, cache: PagedCache, q, ctx_len, max_ctx: int, out=None, workspace=None,
           stream=None):
    """tq_logits: q [batch, n_q_heads, d] -> out fp32 [batch, n_q_heads, max_ctx]."""
    import torch
    assert q.is_cuda and q.is_contiguous() and q.dim() == 3
    b, hq, d = q.shape
    if out is None:
        out = torch.empty(b, hq, max_ctx, dtype=torch.float32, device=q.device)
    if workspace is None:
        n = logits_workspace_bytes(cb, b, cache.n_kv_heads, hq)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    cs = cache.struct()
    _check(load_library().tq_logits(cb.handle, ctypes.byref(cs), _ptr(q), _dtype_code(q), b, hq,
                                     _ptr(ctx_len), max_ctx, _ptr(out), out.stride(1),
                                     _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def logits_topk_workspace_bytes(cb: Codebook, batch: int, n_kv_heads: int, n_q_heads: int, max_ctx: int,
                                k: int) -> int:
    return int(load_library().tq_logits_topk_workspace_bytes(cb.handle, batch, n_kv_heads, n_q_heads, max_ctx, k))


def logits_topk(cb: Codebook, cache: PagedCache, q, ctx_len, max_ctx: int, k: int, scores=None, idx=None,
                workspace=None, stream=None):
    """tq_logits_topk: q [batch, n_q_heads, d] -> (scores fp32, idx int32), each [batch, n_q_heads, k]."""
    import torch
    assert q.is_cuda and q.is_contiguous() and q.dim() == 3
    b, hq, d = q.shape
    if scores is None:
        scores = torch.empty(b, hq, k, dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty(b, hq, k, dtype=torch.int32, device=q.device)
    if workspace is None:
        n = logits_topk_workspace_bytes(cb, b, cache.n_kv_heads, hq, max_ctx, k)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    cs = cache.struct()
    _check(load_library().tq_logits_topk(cb.handle, ctypes.byref(cs), _ptr(q), _dtype_code(q), b, hq,
                                          _ptr(ctx_len), max_ctx, k, _ptr(scores), _ptr(idx),
                                          _ptr(workspace), workspace.numel(), _stream(stream)))
    return scores, idx


class PolarCodec:
    """Handle of tq_polar: the recursive polar form of stage 1 for (d, bits, m)."""

    def __init__(self, d: int, bits: int, m: int, seed_pi: int, seed_s: int):
        lib = load_library()
        self.d, self.bits, self.m = d, bits, m
        h = ctypes.c_void_p()
        _check(lib.tq_polar_build(d, bits, m, seed_pi, seed_s, ctypes.byref(h)))
        self.handle = h
        self.record_bytes = int(lib.tq_polar_record_bytes(h))

    def close(self) -> None:
        if getattr(self, "handle", None):
            load_library().tq_polar_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def polar_encode(pc: PolarCodec, x, records=None, error_word=None, stream=None):
    """tq_polar_encode: x [n, d] -> records uint8 [n, record_bytes]."""
    import torch
    assert x.is_cuda and x.is_contiguous() and x.dim() == 2
    n = x.shape[0]
    if records is None:
        records = torch.zeros(n, pc.record_bytes, dtype=torch.uint8, device=x.device)
    _check(load_library().tq_polar_encode(pc.handle, _ptr(x), _dtype_code(x), n, _ptr(records),
                                           _ptr(error_word), _stream(stream)))
    return records


def polar_logits(pc: PolarCodec, records, q, out=None, workspace=None, stream=None):
    """tq_polar_logits: records [n, record_bytes], q [nq, d] -> out fp32 [nq, n]."""
    import torch
    assert q.is_cuda and q.is_contiguous() and q.dim() == 2
    n, nq = records.shape[0], q.shape[0]
    if out is None:
        out = torch.empty(nq, n, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(int(load_library().tq_polar_logits_workspace_bytes(pc.handle, nq)), 16),
                                dtype=torch.uint8, device=q.device)
    _check(load_library().tq_polar_logits(pc.handle, _ptr(records), n, _ptr(q), _dtype_code(q), nq, _ptr(out),
                                           out.stride(0), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def values_workspace_bytes(cb: Codebook, batch: int, n_kv_heads: int, n_q_heads: int, max_ctx: int) -> int:
    return int(load_library().tq_values_workspace_bytes(cb.handle, batch, n_kv_heads, n_q_heads, max_ctx))


def dequant_values(cb: Codebook, cache: PagedCache, ctx_len, max_ctx: int, batch: int,
                   weights=None, n_q_heads: int | None = None, out=None, out_dtype=None,
                   workspace=None, stream=None):
    """tq_dequant_values.  Mode A (weights None): out [batch, n_kv_heads, max_ctx, d].
    Mode B: weights fp32 [batch, n_q_heads, >= max_ctx] -> out fp32 [batch, n_q_heads, d]."""
    import torch
    dev = cache.pages.device
    if weights is None:
        out_dtype = out_dtype or torch.float32
        if out is None:
            out = torch.zeros(batch, cache.n_kv_heads, max_ctx, cb.d, dtype=out_dtype, device=dev)
        hq, w_stride, o_stride, ws = cache.n_kv_heads, 0, out.shape[2], workspace
    else:
        assert weights.is_cuda and weights.dtype == torch.float32 and weights.stride(2) == 1
        hq = weights.shape[1]
        if out is None:
            out = torch.empty(batch, hq, cb.d, dtype=torch.float32, device=dev)
        w_stride, o_stride = weights.stride(1), 0
        ws = workspace
        if ws is None:
            n = values_workspace_bytes(cb, batch, cache.n_kv_heads, hq, max_ctx)
            ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    cs = cache.struct()
    _check(load_library().tq_dequant_values(
        cb.handle, ctypes.byref(cs), _ptr(weights), w_stride, batch, hq, _ptr(ctx_len), max_ctx,
        _ptr(out), _dtype_code(out), o_stride, _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)))
    return out


def logits_noalloc(cb: Codebook, cache: PagedCache, q, ctx_len, max_ctx: int, out=None, stream=None):
    """tq_logits_noalloc: tq_logits with its scratch taken from the library's
    static device array (for callers that cannot allocate device memory)."""
    import torch
    assert q.is_cuda and q.is_contiguous() and q.dim() == 3
    b, hq, d = q.shape
    if out is None:
        out = torch.empty(b, hq, max_ctx, dtype=torch.float32, device=q.device)
    cs = cache.struct()
    _check(load_library().tq_logits_noalloc(cb.handle, ctypes.byref(cs), _ptr(q), _dtype_code(q), b, hq,
                                             _ptr(ctx_len), max_ctx, _ptr(out), out.stride(1),
                                             _stream(stream)))
    return out


def selftest_wait_timeout(error_word, stream=None) -> None:
    """tq_selftest_wait_timeout: a bounded wait that runs out (about 1 s) and
    reports DEV_ERR_TIMEOUT into `error_word` (device int32 [1])."""
    _check(load_library().tq_selftest_wait_timeout(_ptr(error_word), _stream(stream)))


def polar_angle_codebook(level: int, bits: int):
    """tq_polar_angle_codebook: (centroids, boundaries, distortion) of the
    Lloyd-Max quantizer of the level-`level` angles of the polar form."""
    import numpy as np
    c = np.zeros(1 << bits, dtype=np.float64)
    t = np.zeros((1 << bits) - 1, dtype=np.float64)
    dist = ctypes.c_double(0.0)
    _check(load_library().tq_polar_angle_codebook(level, bits, c.ctypes.data, t.ctypes.data if t.size else None,
                                                   ctypes.addressof(dist)))
    return c, t, dist.value


def attend_workspace_bytes(key_cb: Codebook, value_cb: Codebook, batch: int, n_kv_heads: int, n_q_heads: int,
                           max_ctx: int) -> int:
    return int(load_library().tq_attend_workspace_bytes(key_cb.handle, value_cb.handle, batch, n_kv_heads,
                                                        n_q_heads, max_ctx))


def attend(key_cb: Codebook, key_cache: PagedCache, value_cb: Codebook, value_cache: PagedCache, q, ctx_len,
           max_ctx: int, scale: float | None = None, out=None, workspace=None, stream=None):
    """tq_attend: softmax(scale * logits) @ v_hat from the two caches;
    q [batch, n_q_heads, d] -> out fp32 [batch, n_q_heads, d] (scale 1/sqrt(d) by default)."""
    import torch
    assert q.is_cuda and q.is_contiguous() and q.dim() == 3
    b, hq, d = q.shape
    if scale is None:
        scale = 1.0 / d ** 0.5
    if out is None:
        out = torch.empty(b, hq, d, dtype=torch.float32, device=q.device)
    if workspace is None:
        n = attend_workspace_bytes(key_cb, value_cb, b, key_cache.n_kv_heads, hq, max_ctx)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    ks, vs = key_cache.struct(), value_cache.struct()
    _check(load_library().tq_attend(key_cb.handle, ctypes.byref(ks), value_cb.handle, ctypes.byref(vs), _ptr(q),
                                    _dtype_code(q), b, hq, _ptr(ctx_len), max_ctx, float(scale), _ptr(out),
                                    _ptr(workspace), workspace.numel(), _stream(stream)))
    return out
