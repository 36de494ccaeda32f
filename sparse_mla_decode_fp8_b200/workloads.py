"""Seeded synthetic workloads for the sparse MLA decode step.

This module writes inputs only: a paged FP8 latent cache, a block table, topk
index lists, sequence lengths and bf16 queries.  It holds none of the decode
arithmetic (no dequantisation, no attention).  Its one piece of numerics is the
cache *writer* -- quantising an fp32 latent to 448 e4m3 bytes with one UE8M0
scale per 64 dims plus 64 bf16 rope values -- done with torch's own float8 and
bfloat16 casts (round to nearest even).

Byte layout written (source page "The Validation Gate: Writing a Standalone
Correctness Test for a Custom MMA Sparse-Decode Kernel", section "The Test
Design"): the cache is uint8 [num_pages, 256*584]; a page holds the 256 token
rows of 576 bytes (448 e4m3 nope bytes, then 64 little-endian bf16 rope
values) followed by the 256 scale rows of 8 bytes (7 UE8M0 bytes for nope dims
[64g, 64g+64), one zero pad byte).

The five workloads restate the benchmark configurations of the sparse MLA decode
north-star (H=64, sm_scale = 512^-0.5, q ~ N(0,1) in bf16, latents ~ N(0,1)):

  1. B=1,   4 pages, block_table [0,1,2,3], seq_len 1024, topk 64.
  2. B=1,   32 pages, block_table a seeded permutation, seq_len 8192, topk 512.
  3. B=16,  seq_len ~ U[256, 32768], disjoint random pages of one shared pool,
            topk 512 with -1 padding when seq_len < 512.
  4. B=64,  seq_len 65536 (256 pages each, 16384-page pool), topk 512,
            1% of token rows scaled by 20 before quantisation.
  5. B=256, seq_len ~ U[1024, 8192], pool of 8192 pages (2M tokens), topk 512.

Config k draws from ``numpy.random.default_rng(k)`` (PCG64) unless a seed is
given.  Only token rows that some topk slot references receive a latent
(``fill="referenced"``, the default); every other row stays zero bytes.  This
keeps generation of the 2.45 GB pool of config 4 to seconds and changes nothing
the decode step reads.  ``fill="all"`` writes every row inside each request's
sequence (used for dense brute-force checks on tiny caches).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

PAGE_TOKENS = 256
ROW_BYTES = 576
SCALE_ROW_BYTES = 8
PAGE_BYTES = PAGE_TOKENS * (ROW_BYTES + SCALE_ROW_BYTES)  # 149504
SCALE_BLOCK_OFFSET = PAGE_TOKENS * ROW_BYTES  # 147456
NOPE = 448
ROPE = 64
DIM = 512
GROUP = 64
HEADS = 64
E4M3_MAX = 448.0


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even) bit patterns as uint16."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def quantize_rows(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Cache writer: fp32 latents [n,512] -> (token rows [n,576], scale rows [n,8]).

    Per 64-dim nope group: e = ceil(log2(amax / 448)) clamped to [-127, 127]
    (e = -127 for an all-zero group), scale byte = e + 127, nope byte =
    e4m3(x / 2^e) with round-to-nearest-even.  Rope: bf16 round-to-nearest-even.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    n = x.shape[0]
    nope = x[:, :NOPE].reshape(n, NOPE // GROUP, GROUP).astype(np.float64)
    amax = np.abs(nope).max(axis=2)
    ratio = amax / E4M3_MAX
    mant, expo = np.frexp(ratio)  # ratio = mant * 2^expo, mant in [0.5, 1)
    e = np.where(mant == 0.5, expo - 1, expo)  # exact ceil(log2(ratio))
    e = np.where(amax == 0.0, -127, e)
    e = np.clip(e, -127, 127).astype(np.int64)
    scaled = np.ldexp(nope, -e[:, :, None])  # exact: division by a power of two
    scaled = np.clip(scaled, -E4M3_MAX, E4M3_MAX).astype(np.float32)
    fp8 = torch.from_numpy(scaled.reshape(n, NOPE)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    rope = to_bf16_bits(x[:, NOPE:]).view(np.uint8).reshape(n, 2 * ROPE)  # little-endian
    rows = np.concatenate([fp8, rope], axis=1)
    scales = np.zeros((n, SCALE_ROW_BYTES), np.uint8)
    scales[:, : NOPE // GROUP] = (e + 127).astype(np.uint8)
    return rows, scales


def row_views(cache: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Writable strided views [pages,256,576] and [pages,256,8] into a cache.

    A plain slice-and-reshape of the cache would copy (the row stride is the
    whole page), so the views are built with explicit strides.
    """
    assert cache.dtype == np.uint8 and cache.ndim == 2 and cache.shape[1] == PAGE_BYTES
    assert cache.flags["C_CONTIGUOUS"]
    P = cache.shape[0]
    st = np.lib.stride_tricks.as_strided
    rows = st(cache, shape=(P, PAGE_TOKENS, ROW_BYTES), strides=(PAGE_BYTES, ROW_BYTES, 1), writeable=True)
    scales = st(cache[:, SCALE_BLOCK_OFFSET:], shape=(P, PAGE_TOKENS, SCALE_ROW_BYTES),
                strides=(PAGE_BYTES, SCALE_ROW_BYTES, 1), writeable=True)
    return rows, scales


def write_tokens(cache: np.ndarray, pages: np.ndarray, slots: np.ndarray, latents: np.ndarray) -> None:
    """Quantise ``latents`` [n,512] and store them at (page, slot) pairs."""
    rows, scales = row_views(cache)
    r, s = quantize_rows(latents)
    rows[pages, slots] = r
    scales[pages, slots] = s


@dataclass
class Workload:
    """One decode batch (or ``R`` replicas of it sharing the cache)."""

    name: str
    q: np.ndarray  # uint16 bf16 bits [R,B,H,512]
    cache: np.ndarray  # uint8 [num_pages, 149504]
    block_table: np.ndarray  # int32 [B, max_blocks]
    topk_idx: np.ndarray  # int32 [R,B,topk]
    seq_lens: np.ndarray  # int32 [B]
    sm_scale: float
    outlier_codes: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))

    @property
    def R(self) -> int:
        return self.q.shape[0]

    @property
    def B(self) -> int:
        return self.q.shape[1]

    @property
    def H(self) -> int:
        return self.q.shape[2]

    @property
    def topk(self) -> int:
        return self.topk_idx.shape[2]

    @property
    def num_pages(self) -> int:
        return self.cache.shape[0]

    @property
    def max_blocks(self) -> int:
        return self.block_table.shape[1]

    def replica(self, r: int) -> "Workload":
        return Workload(self.name, self.q[r : r + 1], self.cache, self.block_table, self.topk_idx[r : r + 1],
                        self.seq_lens, self.sm_scale, self.outlier_codes)

    def valid_counts(self) -> np.ndarray:
        """Valid topk slots per (replica, request): 0 <= idx < seq_len and a mapped page."""
        idx = self.topk_idx.astype(np.int64)
        sl = self.seq_lens.astype(np.int64)[None, :, None]
        blk = np.where(idx >= 0, idx // PAGE_TOKENS, 0)
        inb = (idx >= 0) & (idx < sl) & (blk < self.max_blocks)
        blk = np.minimum(blk, self.max_blocks - 1)
        page = self.block_table[np.arange(self.B)[None, :, None], blk]
        ok = inb & (page >= 0) & (page < self.num_pages)
        return ok.sum(axis=2)


def _distinct(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    return rng.choice(n, size=k, replace=False).astype(np.int32)


def _layout(config: int, rng: np.random.Generator):
    """Sequence lengths, page pool size and disjoint block tables of a config."""
    if config == 1:
        seq = np.array([1024], np.int32)
        num_pages = 4
        tables = [np.arange(4, dtype=np.int32)]
    elif config == 2:
        seq = np.array([8192], np.int32)
        num_pages = 32
        tables = [rng.permutation(32).astype(np.int32)]
    elif config == 3:
        seq = rng.integers(256, 32768, size=16, endpoint=True).astype(np.int32)
        need = (seq.astype(np.int64) + PAGE_TOKENS - 1) // PAGE_TOKENS
        num_pages = int(need.sum())
        perm = rng.permutation(num_pages).astype(np.int32)
        cuts = np.concatenate([[0], np.cumsum(need)])
        tables = [perm[cuts[i] : cuts[i + 1]] for i in range(16)]
    elif config == 4:
        seq = np.full(64, 65536, np.int32)
        num_pages = 64 * 256
        perm = rng.permutation(num_pages).astype(np.int32)
        tables = [perm[256 * i : 256 * (i + 1)] for i in range(64)]
    elif config == 5:
        seq = rng.integers(1024, 8192, size=256, endpoint=True).astype(np.int32)
        need = (seq.astype(np.int64) + PAGE_TOKENS - 1) // PAGE_TOKENS
        num_pages = 8192
        perm = rng.permutation(num_pages).astype(np.int32)
        cuts = np.concatenate([[0], np.cumsum(need)])
        tables = [perm[cuts[i] : cuts[i + 1]] for i in range(256)]
    else:
        raise ValueError(f"unknown config {config}")
    max_blocks = max(len(t) for t in tables)
    bt = np.full((len(tables), max_blocks), -1, np.int32)
    for i, t in enumerate(tables):
        bt[i, : len(t)] = t
    return seq, num_pages, bt


CONFIG_TOPK = {1: 64, 2: 512, 3: 512, 4: 512, 5: 512}
CONFIG_OUTLIER_FRACTION = {4: 0.01}
OUTLIER_FACTOR = 20.0


def make_config(config: int, replicas: int = 1, seed: int | None = None, fill: str = "referenced") -> Workload:
    """Build workload ``config`` (1..5) with ``replicas`` independent (q, topk) draws."""
    rng = np.random.default_rng(config if seed is None else seed)
    seq, num_pages, bt = _layout(config, rng)
    B = len(seq)
    topk = CONFIG_TOPK[config]
    idx = np.full((replicas, B, topk), -1, np.int32)
    for r in range(replicas):
        for b in range(B):
            n = min(topk, int(seq[b]))
            idx[r, b, :n] = _distinct(rng, int(seq[b]), n)
    q = to_bf16_bits(rng.standard_normal((replicas, B, HEADS, DIM), dtype=np.float32))
    cache = np.zeros((num_pages, PAGE_BYTES), np.uint8)
    # tokens that receive a latent
    if fill == "all":
        codes = np.concatenate([bt[b, np.arange(int(seq[b])) // PAGE_TOKENS].astype(np.int64) * PAGE_TOKENS
                                + np.arange(int(seq[b])) % PAGE_TOKENS for b in range(B)])
    elif fill == "referenced":
        parts = []
        for b in range(B):
            v = idx[:, b, :].reshape(-1)
            v = v[(v >= 0) & (v < seq[b])].astype(np.int64)
            parts.append(bt[b, v // PAGE_TOKENS].astype(np.int64) * PAGE_TOKENS + v % PAGE_TOKENS)
        codes = np.concatenate(parts) if parts else np.zeros(0, np.int64)
    else:
        raise ValueError(fill)
    codes = np.unique(codes)
    frac = CONFIG_OUTLIER_FRACTION.get(config, 0.0)
    outliers = np.zeros(0, np.int64)
    chunk = 1 << 16
    for start in range(0, len(codes), chunk):
        c = codes[start : start + chunk]
        lat = rng.standard_normal((len(c), DIM), dtype=np.float32)
        if frac > 0:
            hit = rng.random(len(c)) < frac
            lat[hit] *= OUTLIER_FACTOR
            outliers = np.concatenate([outliers, c[hit]])
        write_tokens(cache, (c // PAGE_TOKENS).astype(np.int64), (c % PAGE_TOKENS).astype(np.int64), lat)
    return Workload(f"config{config}", q, cache, bt, idx, seq, DIM ** -0.5, outliers)


def make_custom(B: int, topk: int, seq_lens, num_pages: int | None = None, seed: int = 0, fill: str = "all",
                pad_fraction: float = 0.0, replicas: int = 1, outlier_fraction: float = 0.0,
                duplicates: bool = False) -> Workload:
    """A small free-form workload: ragged lengths, -1 padding, duplicates, outliers.

    ``pad_fraction`` of the slots of every request become -1 (scattered, not only
    at the end); ``duplicates`` draws indices with replacement.
    """
    rng = np.random.default_rng(seed)
    seq = np.asarray(seq_lens, np.int32).reshape(B)
    need = (seq.astype(np.int64) + PAGE_TOKENS - 1) // PAGE_TOKENS
    need = np.maximum(need, 1)
    total = int(need.sum())
    if num_pages is None:
        num_pages = total
    assert num_pages >= total
    perm = rng.permutation(num_pages).astype(np.int32)
    max_blocks = int(need.max())
    bt = np.full((B, max_blocks), -1, np.int32)
    cuts = np.concatenate([[0], np.cumsum(need)])
    for b in range(B):
        bt[b, : need[b]] = perm[cuts[b] : cuts[b + 1]]
    idx = np.full((replicas, B, topk), -1, np.int32)
    for r in range(replicas):
        for b in range(B):
            if seq[b] <= 0:
                continue
            if duplicates or seq[b] < topk:
                n = topk if duplicates else int(seq[b])
                v = rng.integers(0, seq[b], size=n) if duplicates else _distinct(rng, int(seq[b]), n)
            else:
                v = _distinct(rng, int(seq[b]), topk)
            row = np.full(topk, -1, np.int32)
            row[: len(v)] = v
            if pad_fraction > 0:
                row[rng.random(topk) < pad_fraction] = -1
            rng.shuffle(row)
            idx[r, b] = row
    q = to_bf16_bits(rng.standard_normal((replicas, B, HEADS, DIM), dtype=np.float32))
    cache = np.zeros((num_pages, PAGE_BYTES), np.uint8)
    if fill == "all":
        parts = [bt[b, np.arange(int(seq[b])) // PAGE_TOKENS].astype(np.int64) * PAGE_TOKENS
                 + np.arange(int(seq[b])) % PAGE_TOKENS for b in range(B) if seq[b] > 0]
    else:
        parts = []
        for b in range(B):
            v = idx[:, b, :].reshape(-1)
            v = v[(v >= 0) & (v < seq[b])].astype(np.int64)
            parts.append(bt[b, v // PAGE_TOKENS].astype(np.int64) * PAGE_TOKENS + v % PAGE_TOKENS)
    codes = np.unique(np.concatenate(parts)) if parts else np.zeros(0, np.int64)
    if len(codes):
        lat = rng.standard_normal((len(codes), DIM), dtype=np.float32)
        if outlier_fraction > 0:
            lat[rng.random(len(codes)) < outlier_fraction] *= OUTLIER_FACTOR
        write_tokens(cache, codes // PAGE_TOKENS, codes % PAGE_TOKENS, lat)
    return Workload(f"custom_B{B}_k{topk}", q, cache, bt, idx, seq, DIM ** -0.5)


def roofline_units(w: Workload) -> dict:
    """Algorithmic work of one decode call: valid (query, token) pairs and queries.

    Per valid (query, token): 584 bytes of KV (576-byte row + 8-byte scale row)
    and 2*2*64*512 = 131072 MMA FLOP (QK^T and PV over 64 heads); per query
    65536 bytes of bf16 Q.
    """
    pairs = int(w.valid_counts().sum())
    queries = w.R * w.B
    return {
        "valid_pairs": pairs,
        "queries": queries,
        "bytes": pairs * (ROW_BYTES + SCALE_ROW_BYTES) + queries * w.H * DIM * 2,
        "flops": pairs * 2 * 2 * w.H * DIM,
    }
