"""The seeded input generator (CPU only)."""
import numpy as np
import pytest

from sparse_mla_decode_fp8_b200 import workloads as W
from tests import independent as ind


@pytest.mark.parametrize("k", [1, 2, 3])
def test_config_shapes_and_indices(k):
    w = W.make_config(k)
    assert w.H == 64 and w.topk == W.CONFIG_TOPK[k]
    assert w.cache.shape == (w.num_pages, 149504)
    used = w.block_table[w.block_table >= 0]
    assert len(np.unique(used)) == len(used), "block tables must be disjoint"
    assert used.max() < w.num_pages
    for b in range(w.B):
        row = w.topk_idx[0, b]
        v = row[row >= 0]
        assert len(np.unique(v)) == len(v), "indices must be distinct"
        assert v.max() < w.seq_lens[b]
        assert len(v) == min(w.topk, int(w.seq_lens[b]))
        assert np.all(row[len(v):] == -1), "padding goes at the end"
        need = -(-int(w.seq_lens[b]) // 256)
        assert np.all(w.block_table[b, :need] >= 0) and np.all(w.block_table[b, need:] == -1)
    assert abs(w.sm_scale - 512 ** -0.5) < 1e-15


def test_fixed_layouts():
    w1 = W.make_config(1)
    assert w1.block_table.tolist() == [[0, 1, 2, 3]] and w1.seq_lens.tolist() == [1024]
    w2 = W.make_config(2)
    assert sorted(w2.block_table[0].tolist()) == list(range(32)) and w2.seq_lens.tolist() == [8192]
    w3 = W.make_config(3)
    assert np.all((w3.seq_lens >= 256) & (w3.seq_lens <= 32768))


def test_deterministic():
    a = W.make_config(2)
    b = W.make_config(2)
    assert np.array_equal(a.cache, b.cache) and np.array_equal(a.q, b.q) and np.array_equal(a.topk_idx, b.topk_idx)
    c = W.make_config(2, seed=99)
    assert not np.array_equal(a.topk_idx, c.topk_idx)


def test_quantiser_error_bound():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((300, 512)).astype(np.float32)
    x[::7] *= 20
    x[5, :64] = 0.0
    rows, scales = W.quantize_rows(x)
    cache = np.zeros((2, W.PAGE_BYTES), np.uint8)
    pages = np.arange(300) // 256
    slots = np.arange(300) % 256
    W.write_tokens(cache, pages, slots, x)
    deq = ind.token_latents(cache, pages, slots)
    nope = x[:, :448].astype(np.float64).reshape(300, 7, 64)
    e = scales[:, :7].astype(np.int64) - 127
    amax = np.abs(nope).max(axis=2)
    nz = amax > 0
    assert np.all(2.0 ** e[nz] >= amax[nz] / 448) and np.all(2.0 ** (e[nz] - 1) < amax[nz] / 448)
    err = np.abs(deq[:, :448].reshape(300, 7, 64) - nope)
    # round-to-nearest e4m3: relative 2^-4 for normals, absolute 2^-10 * 2^e for subnormals
    bound = np.maximum(np.abs(nope) * 2.0 ** -4, 2.0 ** -10 * 2.0 ** e[:, :, None])
    assert np.all(err <= bound * (1 + 1e-12))
    assert np.all(deq[5, :64] == 0.0)
    rope_err = np.abs(deq[:, 448:] - x[:, 448:])
    assert np.all(rope_err <= np.abs(x[:, 448:]) * 2.0 ** -8)
    assert np.all(scales[:, 7] == 0)


def test_referenced_fill_and_outliers():
    w = W.make_config(4, replicas=1)
    assert w.B == 64 and w.num_pages == 16384 and np.all(w.seq_lens == 65536)
    n_ref = int(w.valid_counts().sum())
    assert n_ref == 64 * 512
    frac = len(w.outlier_codes) / n_ref
    assert 0.005 < frac < 0.015
    p, s = w.outlier_codes // 256, w.outlier_codes % 256
    lat = ind.token_latents(w.cache, p[:50], s[:50])
    assert np.abs(lat).max() > 30


def test_replicas_share_cache():
    w = W.make_config(2, replicas=3)
    assert w.q.shape[0] == 3 and w.topk_idx.shape[0] == 3
    assert not np.array_equal(w.topk_idx[0], w.topk_idx[1])
    r = w.replica(1)
    assert r.q.shape[0] == 1 and r.cache is w.cache


def test_roofline_units():
    w = W.make_config(2)
    u = W.roofline_units(w)
    assert u["valid_pairs"] == 512 and u["bytes"] == 512 * 584 + 65536 and u["flops"] == 512 * 131072
