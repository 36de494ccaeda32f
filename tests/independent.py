"""A second, independent reading of the cache bytes and of the attention step.

Used only to pin the oracle.  Nothing here shares code with ``oracle/`` or the
CUDA path: e4m3, UE8M0 and bf16 decoding go through torch's own float8_e4m3fn,
float8_e8m0fnu and bfloat16 dtypes, byte offsets are written out again from the
page layout ("The Validation Gate", section "The Test Design"), and attention
is a dense masked softmax over *every* token of a request with each token
weighted by how many topk slots select it.
"""
from __future__ import annotations

import numpy as np
import torch

_PAGE = 256 * 584
_SCALES_AT = 256 * 576


def token_latents(cache: np.ndarray, pages, slots) -> np.ndarray:
    """fp64 [n,512] latents of tokens (page, slot), decoded with torch dtypes."""
    pages = np.asarray(pages, np.int64).reshape(-1)
    slots = np.asarray(slots, np.int64).reshape(-1)
    flat = cache.reshape(-1)
    row0 = pages * _PAGE + slots * 576
    sc0 = pages * _PAGE + _SCALES_AT + slots * 8
    rows = flat[row0[:, None] + np.arange(576)[None, :]]
    scl = flat[sc0[:, None] + np.arange(7)[None, :]]
    nope = torch.from_numpy(np.ascontiguousarray(rows[:, :448])).view(torch.float8_e4m3fn).double()
    scale = torch.from_numpy(np.ascontiguousarray(scl)).view(torch.float8_e8m0fnu).double()
    nope = nope * scale.repeat_interleave(64, dim=1)
    rope = torch.from_numpy(np.ascontiguousarray(rows[:, 448:576])).view(torch.bfloat16).double()
    return torch.cat([nope, rope], dim=1).numpy()


def q_values(q_bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(q_bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def dense_attention(q_bits, cache, block_table, topk_idx, seq_lens, sm_scale, num_pages=None):
    """Dense masked attention: every token t < seq_len of request b, weight
    count(t in topk_idx[b]) * exp(s_t - M).  Returns fp64 (out [B,H,512], lse [B,H])."""
    q = q_values(q_bits)
    B, H, D = q.shape
    num_pages = cache.shape[0] if num_pages is None else num_pages
    max_blocks = block_table.shape[1]
    out = np.zeros((B, H, D))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        n = int(seq_lens[b])
        if n <= 0:
            continue
        t = np.arange(n)
        blk = t // 256
        okb = blk < max_blocks
        page = np.where(okb, block_table[b, np.minimum(blk, max_blocks - 1)], -1)
        ok = okb & (page >= 0) & (page < num_pages)
        counts = np.zeros(n)
        for i in topk_idx[b]:
            if 0 <= i < n:
                counts[i] += 1
        counts[~ok] = 0
        sel = counts > 0
        if not sel.any():
            continue
        K = np.zeros((n, D))
        K[ok] = token_latents(cache, page[ok], (t % 256)[ok])
        for h in range(H):
            s = sm_scale * (K @ q[b, h])
            M = s[sel].max()
            w = np.where(sel, counts * np.exp(np.where(sel, s - M, 0.0)), 0.0)
            out[b, h] = (w[:, None] * K).sum(axis=0) / w.sum()
            lse[b, h] = M + np.log(w.sum())
    return out, lse
