"""Seeded synthetic inputs for the codec's workloads (numpy only).

This module holds no codec arithmetic: it only draws keys, values, queries,
weights and block tables with the shapes and value laws of the workloads, so
that the CUDA library and the CPU oracle can be fed the same numbers.

bf16 tensors are returned as (bits uint16, exact float64 values) pairs; the
float64 array is exactly what the bf16 bits represent.
"""

from __future__ import annotations

import numpy as np

SEED_PI = 0x5EED0001
SEED_S = 0x5EED0002


def to_bf16(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 values to bfloat16 (nearest-even): (uint16 bits, float64 values)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    vals = (r.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return r, vals


def tiny_keys(seed: int = 1001, n: int = 4096, d: int = 128, n_queries: int = 16,
              n_outlier: int = 4, outlier_scale: float = 20.0):
    """fp32 keys ~ N(0, 1) with a few outlier channels scaled up, fp32 queries ~ N(0, 1).

    The outlier channels are the first `n_outlier` entries of a seeded
    permutation of the channels."""
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((n, d)).astype(np.float32)
    chans = rng.permutation(d)[:n_outlier]
    K[:, chans] *= outlier_scale
    Q = rng.standard_normal((n_queries, d)).astype(np.float32)
    return K, Q, chans


def decode_step(seed: int, batch: int, n_kv_heads: int, n_q_heads: int, ctx: int, d: int = 128):
    """bf16 K, V [batch, n_kv_heads, ctx, d] ~ N(0, 1) * scale[h, c] with one
    log-uniform [0.1, 10] scale per (KV head, channel), drawn separately for K
    and V; bf16 queries [batch, n_q_heads, d] ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    out = {}
    for name in ("k", "v"):
        scale = np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=(n_kv_heads, d))).astype(np.float32)
        x = rng.standard_normal((batch, n_kv_heads, ctx, d), dtype=np.float32)
        x *= scale[None, :, None, :]
        out[name] = to_bf16(x)
    out["q"] = to_bf16(rng.standard_normal((batch, n_q_heads, d), dtype=np.float32))
    return out


def append_batch(seed: int, batch: int, n_kv_heads: int, n_new: int, d: int = 128,
                 outlier_frac: float = 0.01, outlier_scale: float = 30.0):
    """bf16 [batch, n_kv_heads, n_new, d] ~ N(0, 1) with a seeded Bernoulli
    fraction of entries scaled up as outliers."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, n_kv_heads, n_new, d), dtype=np.float32)
    mask = rng.random(x.shape, dtype=np.float32) < outlier_frac
    x[mask] *= outlier_scale
    return to_bf16(x)


def block_table(seed: int, batch: int, pages_per_seq: int, n_pages: int | None = None) -> np.ndarray:
    """int32 [batch, pages_per_seq]: a seeded permutation of page ids, so the
    pages of one sequence are not contiguous."""
    rng = np.random.default_rng(seed)
    total = batch * pages_per_seq
    n_pages = n_pages or total
    return rng.permutation(n_pages)[:total].reshape(batch, pages_per_seq).astype(np.int32)


def softmax_like_weights(seed: int, batch: int, n_q_heads: int, ctx: int) -> np.ndarray:
    """fp32 [batch, n_q_heads, ctx] positive weights summing to 1 per row."""
    rng = np.random.default_rng(seed)
    w = rng.exponential(1.0, size=(batch, n_q_heads, ctx)).astype(np.float64)
    w /= w.sum(axis=-1, keepdims=True)
    return w.astype(np.float32)


def anisotropic_unit(seed: int, n: int, d: int = 200, chunk: int = 65536) -> np.ndarray:
    """float32 [n, d] rows ~ N(0, diag(1/i)), i = 1..d, scaled to unit norm."""
    rng = np.random.default_rng(seed)
    sd = (1.0 / np.sqrt(np.arange(1, d + 1))).astype(np.float32)
    out = np.empty((n, d), dtype=np.float32)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = rng.standard_normal((e - s, d), dtype=np.float32) * sd[None, :]
        out[s:e] = x / np.linalg.norm(x, axis=1, keepdims=True)
    return out


def decode_keys_device(seed: int, batch: int, n_kv_heads: int, n_q_heads: int, ctx: int, d: int = 128,
                       device="cuda"):
    """The decode-step laws of decode_step, drawn on the device with torch's
    seeded generator (for contexts too large to draw on the host): bf16 K
    [batch, n_kv_heads, ctx, d] ~ N(0, 1) * scale[h, c] (log-uniform [0.1, 10]
    per (KV head, channel)) and bf16 queries [batch, n_q_heads, d] ~ N(0, 1)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    lo, hi = float(np.log(0.1)), float(np.log(10.0))
    scale = torch.exp(torch.rand((n_kv_heads, d), generator=g, device=device) * (hi - lo) + lo)
    k = torch.randn((batch, n_kv_heads, ctx, d), generator=g, device=device)
    k.mul_(scale[None, :, None, :])
    q = torch.randn((batch, n_q_heads, d), generator=g, device=device)
    return k.to(torch.bfloat16), q.to(torch.bfloat16)
