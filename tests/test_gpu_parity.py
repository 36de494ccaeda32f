"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mla_decode_fp8_b200 as smla
from sparse_mla_decode_fp8_b200 import build
from sparse_mla_decode_fp8_b200 import workloads as W
from tests.gpu_util import device_inputs, parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    smla.library()


def _run(w, r=0, nsplit=0, ws=None):
    d = device_inputs(w, r)
    out, lse = smla.decode(d["q"], d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"], d["sm_scale"],
                           nsplit=nsplit, workspace=ws)
    torch.cuda.synchronize()
    return out, lse, d


def _oracle(w, r=0):
    return oracle.decode(w.q[r], w.cache, w.block_table, w.topk_idx[r], w.seq_lens, w.sm_scale)


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5])
def test_config_parity(k):
    w = W.make_config(k)
    out, lse, d = _run(w)
    ws = smla.binding.new_workspace(w.B, w.topk)
    smla.decode(d["q"], d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"], d["sm_scale"], workspace=ws)
    assert smla.read_error(ws) == 0
    ro, rl = _oracle(w)
    figs = parity(out, lse, ro, rl)
    print(f"config{k}: nsplit={smla.num_splits(w.B, w.topk)} {figs}")


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5])
def test_gather_bit_exact(k):
    # Index -> (page, slot) translation and dequantisation, bit for bit.  The decode kernel
    # translates every tile with the same two device helpers as this debug gather
    # (slot_in_range, then slot_code on the block-table entry), and its UE8M0 dequant is the
    # same dequant16: configs 4 and 5 cover the large page pools (65 536 and ~8 192 slots).
    w = W.make_config(k)
    d = device_inputs(w)
    lat, ps = smla.debug_gather(d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"])
    rlat, rps = oracle.gather(w.cache, w.block_table, w.topk_idx[0], w.seq_lens)
    assert np.array_equal(ps.cpu().numpy(), rps)
    assert np.array_equal(lat.cpu().numpy().astype(np.float64), rlat)


def test_gather_scale_extremes_bit_exact():
    # every e4m3 code except NaN, under scale bytes across the exact range (10..254) and 0xFF -> NaN
    cache = np.zeros((2, W.PAGE_BYTES), np.uint8)
    rows, scales = W.row_views(cache)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    svals = [10, 60, 100, 120, 127, 134, 142, 143, 180, 254, 255]
    for t in range(256):
        rows[0, t, :448] = np.resize(np.roll(codes, t), 448)
        rows[0, t, 448:] = np.random.default_rng(t).integers(0, 256, 128, dtype=np.uint8)
        rows[0, t, 448 + 1 :: 2] &= 0xBF  # top exponent bit of each rope bf16 cleared: finite values
        scales[0, t, :7] = [svals[(t + g) % len(svals)] for g in range(7)]
    bt = np.array([[0]], np.int32)
    idx = np.arange(256, dtype=np.int32)[None, :]
    sl = np.array([256], np.int32)
    lat, ps = smla.debug_gather(torch.from_numpy(cache).cuda(), torch.from_numpy(bt).cuda(),
                                torch.from_numpy(idx).cuda(), torch.from_numpy(sl).cuda())
    rlat, rps = oracle.gather(cache, bt, idx, sl)
    g = lat.cpu().numpy().astype(np.float64)
    assert np.array_equal(ps.cpu().numpy(), rps)
    # values beyond the bf16 range (scale byte 254 with |e4m3| >= 2) overflow to +-inf on the tensor-core path
    bf16_max = float(torch.finfo(torch.bfloat16).max)
    expect = np.where(np.abs(rlat) > bf16_max, np.sign(rlat) * np.inf, rlat)
    assert np.array_equal(np.isnan(g), np.isnan(expect))
    ok = ~np.isnan(expect)
    assert np.array_equal(g[ok], expect[ok])


# The validation runs of "The Moment of Validation: A Custom MMA Sparse-Decode Kernel Passes
# Correctness" (the table of its third attempt): B in {1, 4, 16, 32} x topk in {128, 512}, H = 64,
# each with len=0 and len=1.  Read here as: len=0 uniform lengths (every request has at least
# topk tokens, distinct indices, no -1), len=1 ragged lengths (some requests shorter than topk,
# their tails -1) with scattered -1 slots.  The default split count is used.
@pytest.mark.parametrize("B", [1, 4, 16, 32])
@pytest.mark.parametrize("topk", [128, 512])
@pytest.mark.parametrize("ragged", [0, 1])
def test_validation_matrix(B, topk, ragged):
    rng = np.random.default_rng(7000 + 100 * B + topk + ragged)
    if ragged:
        seq = rng.integers(1, 3 * topk, size=B)
        seq[0] = max(1, topk // 3)  # at least one request below topk
        w = W.make_custom(B, topk, seq, seed=int(rng.integers(1 << 30)), fill="referenced", pad_fraction=0.1)
    else:
        seq = rng.integers(topk, 8 * topk, size=B)
        w = W.make_custom(B, topk, seq, seed=int(rng.integers(1 << 30)), fill="referenced")
        assert np.all(w.topk_idx[0] >= 0)
    out, lse, _ = _run(w)
    ro, rl = _oracle(w)
    figs = parity(out, lse, ro, rl)
    print(f"B={B} topk={topk} len={ragged}: nsplit={smla.num_splits(B, topk)} {figs}")


# bf16 output (smla_options.out_bf16): the fp32 result rounded to nearest even, so the
# bound is the fp32 one plus the rounding, 2^-9 |O| (2^-8 here for margin); LSE stays fp32.
@pytest.mark.parametrize("k,ns", [(1, 0), (2, 0), (3, 0), (4, 0), (5, 0), (4, 1), (2, 2)])
def test_bf16_output(k, ns):
    w = W.make_config(k)
    d = device_inputs(w)
    args = (d["q"], d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"], d["sm_scale"])
    out, lse = smla.decode(*args, nsplit=ns, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert out.dtype == torch.bfloat16 and lse.dtype == torch.float32
    ro, rl = _oracle(w)
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.all(np.isfinite(o))
    assert np.all(np.abs(o - ro) <= 2e-3 + 2.0 ** -8 * np.abs(ro))
    assert np.linalg.norm(o - ro) <= 5e-3 * np.linalg.norm(ro)
    fin = np.isfinite(rl)
    assert np.array_equal(np.isneginf(l), np.isneginf(rl))
    assert np.abs(l[fin] - rl[fin]).max() <= 1e-3
    if (ns or smla.num_splits(w.B, w.topk)) == 1:
        # one split: exactly the fp32 output rounded to nearest even, the same LSE
        o32, l32 = smla.decode(*args, nsplit=ns)
        assert torch.equal(out, o32.to(torch.bfloat16)) and torch.equal(lse, l32)


@pytest.mark.parametrize("nsplit", [1, 2, 3, 4])
def test_split_counts_agree(nsplit):
    w = W.make_config(2)
    out, lse, _ = _run(w, nsplit=nsplit)
    ro, rl = _oracle(w)
    parity(out, lse, ro, rl)


@pytest.mark.parametrize("case", ["ragged_tail", "padding", "duplicates", "outliers", "empty_request",
                                  "topk1", "long_topk", "short_seq"])
def test_edge_cases(case):
    if case == "ragged_tail":
        w = W.make_custom(3, 333, [5000, 700, 333], seed=1, fill="referenced")
    elif case == "padding":
        w = W.make_custom(4, 256, [3000, 3000, 200, 50], seed=2, fill="referenced", pad_fraction=0.5)
    elif case == "duplicates":
        w = W.make_custom(2, 200, [300, 9], seed=3, fill="referenced", duplicates=True)
    elif case == "outliers":
        w = W.make_custom(8, 512, [20000] * 8, seed=4, fill="referenced", outlier_fraction=0.02)
    elif case == "empty_request":
        w = W.make_custom(3, 128, [1000, 0, 1000], seed=5, fill="referenced")
    elif case == "topk1":
        w = W.make_custom(5, 1, [10, 300, 1, 4000, 77], seed=6, fill="referenced")
    elif case == "long_topk":
        w = W.make_custom(2, 2048, [100000, 3000], seed=7, fill="referenced")
    else:
        w = W.make_custom(6, 512, [1, 2, 130, 129, 255, 257], seed=8, fill="referenced")
    for ns in (0, 1, 2):
        if ns > (w.topk + 127) // 128:
            continue
        out, lse, _ = _run(w, nsplit=ns)
        ro, rl = _oracle(w)
        parity(out, lse, ro, rl)


def test_bad_page_masked_and_flagged():
    w = W.make_custom(2, 128, [2000, 2000], seed=9, fill="referenced")
    bt = w.block_table.copy()
    bt[0, 1] = w.num_pages + 5  # out of the pool
    bt[1, 2] = -3
    w2 = W.Workload(w.name, w.q, w.cache, bt, w.topk_idx, w.seq_lens, w.sm_scale)
    d = device_inputs(w2)
    ws = smla.binding.new_workspace(w2.B, w2.topk)
    out, lse = smla.decode(d["q"], d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"], d["sm_scale"],
                           workspace=ws)
    flags = smla.read_error(ws)
    ro, rl = oracle.decode(w2.q[0], w2.cache, bt, w2.topk_idx[0], w2.seq_lens, w2.sm_scale)
    parity(out, lse, ro, rl)
    idx = w.topk_idx[0]
    hits = np.any((idx[0] >= 0) & (idx[0] < w.seq_lens[0]) & (idx[0] // 256 == 1)) or \
        np.any((idx[1] >= 0) & (idx[1] < w.seq_lens[1]) & (idx[1] // 256 == 2))
    assert bool(flags & smla.SMLA_FLAG_BAD_PAGE) == bool(hits)
    assert smla.read_error(ws) == 0


def test_combine_matches_oracle():
    rng = np.random.default_rng(3)
    B, H, ns = 3, 64, 5
    po = rng.standard_normal((B, H, ns, 512))
    pl = rng.standard_normal((B, H, ns)) * 5
    pl[0, :, 1] = -np.inf
    pl[1, 3, :] = -np.inf
    out, lse = smla.combine(torch.from_numpy(po).float().cuda(), torch.from_numpy(pl).float().cuda())
    ro, rl = oracle.combine(po.astype(np.float32).astype(np.float64), pl.astype(np.float32).astype(np.float64))
    parity(out, lse, ro, rl)


def test_cuda_graph_replay_matches_eager():
    w = W.make_config(3)
    d = device_inputs(w)
    ws = smla.binding.new_workspace(w.B, w.topk)
    out = torch.empty((w.B, 64, 512), device="cuda")
    lse = torch.empty((w.B, 64), device="cuda")
    args = (d["q"], d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"], d["sm_scale"])
    smla.decode(*args, out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    eager_o, eager_l = out.clone(), lse.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    out.zero_()
    with torch.cuda.graph(g, stream=s):
        smla.decode(*args, out=out, lse=lse, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager_o) and torch.equal(lse, eager_l)
