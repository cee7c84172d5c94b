"""Seeded synthetic inputs for the KV-cache workloads.

This module is the one thing the CUDA path and the CPU oracle share: it draws
random numbers and lays them out, and it holds none of the method's
arithmetic (no rotation, no quantization, no attention).

Recipe (every array is reproducible from its seed on any machine):
  * Gaussian draws: the array is filled in chunks of 2**22 values; chunk c
    comes from numpy's SFC64 generator seeded with SeedSequence([seed, c]),
    ``standard_normal`` in float32.  Chunks are independent, so the fill can
    run on threads and the values do not depend on the thread count.
  * Outlier channels: fixed channel indices of the head dimension are
    multiplied by a factor (x20 on 4 fixed channels for the tiny case; x16 on
    round(1% of D) seeded channels per KV head for the throughput cases).
  * bf16 inputs are the fp32 draws rounded to nearest-even bf16 (raw uint16
    bit patterns are returned so both sides see identical bits).
  * Sequence lengths: uniform integers in [lo, hi] from a seeded generator.
  * Page tables: a seeded random permutation of the physical pages.
  * Octave sign pattern: sign_i = -1 where bit 0 of splitmix64(seed + i) is set.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_CHUNK = 1 << 22


def gaussian(seed: int, shape) -> np.ndarray:
    """float32 N(0,1) array of the given shape (chunked, thread-parallel fill)."""
    n = int(np.prod(shape))
    out = np.empty(n, np.float32)

    def fill(c):
        g = np.random.Generator(np.random.SFC64(np.random.SeedSequence([seed, c])))
        g.standard_normal(out=out[c * _CHUNK:(c + 1) * _CHUNK], dtype=np.float32)

    nchunks = (n + _CHUNK - 1) // _CHUNK
    if nchunks <= 1:
        for c in range(nchunks):
            fill(c)
    else:
        with ThreadPoolExecutor(min(nchunks, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


def _chunked(n: int, fn) -> None:
    """fn(lo, hi) over [0, n) in _CHUNK pieces, on threads for large n."""
    spans = [(lo, min(n, lo + _CHUNK)) for lo in range(0, n, _CHUNK)]
    if len(spans) <= 1:
        for lo, hi in spans:
            fn(lo, hi)
        return
    with ThreadPoolExecutor(min(len(spans), os.cpu_count() or 1)) as ex:
        list(ex.map(lambda sp: fn(*sp), spans))


def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest-even bf16; return the uint16 bits."""
    x = np.ascontiguousarray(x32, dtype=np.float32)
    u = x.view(np.uint32).reshape(-1)
    out = np.empty(u.size, np.uint16)

    def conv(lo, hi):
        t = u[lo:hi] >> np.uint32(16)
        t &= np.uint32(1)
        t += np.uint32(0x7FFF)
        t += u[lo:hi]
        t >>= np.uint32(16)
        out[lo:hi] = t

    _chunked(u.size, conv)
    return out.reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def outlier_channels(seed: int, n_heads: int, dim: int, frac: float = 0.01) -> np.ndarray:
    """(n_heads, k) seeded channel indices, k = round(frac * dim) (3 of 256 for 1%)."""
    k = max(1, int(round(frac * dim)))
    g = np.random.Generator(np.random.SFC64(np.random.SeedSequence([seed, 0xC4A])))
    return np.stack([g.choice(dim, size=k, replace=False) for _ in range(n_heads)])


def apply_outliers(x: np.ndarray, channels: np.ndarray, factor: float) -> np.ndarray:
    """Scale the given channels of the last dim; x is (..., H, D), channels (H, k)
    or (k,) for the same channels on every head."""
    if channels.ndim == 1:
        scale = np.ones(x.shape[-1], np.float32)
        scale[channels] = np.float32(factor)
    else:
        scale = np.ones(x.shape[-2:], np.float32)
        for h in range(channels.shape[0]):
            scale[h, channels[h]] = np.float32(factor)
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(x)
    rows = scale.size
    xf, of = x.reshape(-1, rows), out.reshape(-1, rows)
    step = max(1, _CHUNK // rows)
    for r0 in range(0, xf.shape[0], step):
        np.multiply(xf[r0:r0 + step], scale.reshape(-1), out=of[r0:r0 + step])
    return out


def seq_lens(seed: int, batch: int, lo: int, hi: int) -> np.ndarray:
    g = np.random.Generator(np.random.SFC64(np.random.SeedSequence([seed, 0x5E9])))
    return g.integers(lo, hi + 1, size=batch).astype(np.int32)


def page_table(seed: int, batch: int, pages_per_seq: np.ndarray, max_pages: int,
               extra_pages: int = 0):
    """Shuffled physical pages: returns (block_table[batch, max_pages], n_pages).
    Unused table entries are -1."""
    total = int(np.sum(pages_per_seq)) + extra_pages
    g = np.random.Generator(np.random.SFC64(np.random.SeedSequence([seed, 0x9A6E])))
    perm = g.permutation(total).astype(np.int32)
    bt = np.full((batch, max_pages), -1, np.int32)
    o = 0
    for b in range(batch):
        n = int(pages_per_seq[b])
        bt[b, :n] = perm[o:o + n]
        o += n
    return bt, total


def _splitmix64(z: int) -> int:
    m = (1 << 64) - 1
    z = (z + 0x9E3779B97F4A7C15) & m
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
    return z ^ (z >> 31)


def sign_pattern(n: int, seed: int = 0x0C7A7E) -> np.ndarray:
    """Fixed +-1 float32 pattern: -1 where bit 0 of splitmix64(seed + i) is set."""
    return np.array([-1.0 if _splitmix64(seed + i) & 1 else 1.0 for i in range(n)], np.float32)


# --------------------------------------------------------------------------
# The five workloads (shapes and seeds).  Values are drawn lazily by the
# helpers below so the bench and the tests build identical inputs.
# --------------------------------------------------------------------------
WORKLOADS = {
    "tiny": dict(batch=1, n_kv_heads=1, n_q_heads=4, dim=256, ctx=512, dtype="f32",
                 outlier_channels=(7, 64, 129, 250), outlier_factor=20.0, seed=1),
    "quantize": dict(batch=8, n_kv_heads=8, dim=256, prefill=4096, appends=256,
                     capacity=4352, dtype="bf16", outlier_frac=0.01, outlier_factor=16.0,
                     seed=2),
    "long_decode": dict(batch=1, n_q_heads=32, n_kv_heads=4, dim=256, ctx=131072,
                        dtype="bf16", outlier_frac=0.01, outlier_factor=16.0, seed=3),
    "paged_decode": dict(batch=32, n_q_heads=16, n_kv_heads=2, dim=256, ctx_lo=8192,
                         ctx_hi=32768, page_size=256, dtype="bf16", outlier_frac=0.01,
                         outlier_factor=16.0, seed=4),
    "octave": dict(batch=16, n_q_heads=32, n_kv_heads=8, head_size=128, rope_dim=64,
                   v_bits=4, ctx=16384, block_size=256, dtype="bf16", outlier_frac=0.01,
                   outlier_factor=16.0, seed=5),
}


def kv_tokens(seed: int, batch: int, n_tok: int, n_kv_heads: int, dim: int,
              outlier_frac: float, outlier_factor: float, stream: int = 0):
    """K and V, each (batch, n_tok, n_kv_heads, dim) float32 with outlier channels."""
    ch = outlier_channels(seed, n_kv_heads, dim, outlier_frac)
    k = gaussian(seed * 1000 + 10 + stream, (batch, n_tok, n_kv_heads, dim))
    v = gaussian(seed * 1000 + 20 + stream, (batch, n_tok, n_kv_heads, dim))
    return apply_outliers(k, ch, outlier_factor), apply_outliers(v, ch, outlier_factor)


def queries(seed: int, batch: int, n_q_heads: int, dim: int, stream: int = 0):
    return gaussian(seed * 1000 + 30 + stream, (batch, n_q_heads, dim))
