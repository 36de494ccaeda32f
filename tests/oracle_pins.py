"""Pins of the fp64 oracle to things other than itself.

Each ``check_*`` takes an oracle build (``lib=None`` is the real one) and raises
AssertionError on a mismatch.  ``test_oracle_pins.py`` runs them on the oracle;
``test_oracle_mutants.py`` runs them on deliberately broken copies of the
oracle source and requires every mutant to fail at least one of them.

What pins what:
  * e4m3 / UE8M0 / bf16 decoders -- torch's float8_e4m3fn, float8_e8m0fnu and
    bfloat16 conversions over all byte patterns, plus spot values of the OCP
    formats (0x7E = 448, 0x01 = 2^-9, 0x38 = 1, 0x7F = NaN ...).
  * page translation -- a hand-worked fixture (tests/golden/translate_small.json).
  * byte layout -- marker bytes planted at hand-computed offsets.
  * attention -- closed forms (two tokens: tanh / log-cosh; one token; Q = 0
    gives the mean; all slots equal), invariances (permutation, -1 slots,
    multiplicity), a dense masked brute force decoded through torch dtypes, and
    the LSE-merge identity for the combine.
  * cache writer -- the e4m3 / bf16 encoders against torch's float8_e4m3fn and
    bfloat16 casts (round to nearest even) and at every midpoint between codes;
    the scale exponent at exact powers 448 * 2^k and just above them; whole
    tokens against the numpy/torch writer of the synthetic workloads; the
    scatter against hand-computed (page, slot) offsets.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle
from sparse_mla_decode_fp8_b200 import workloads as W
from tests import independent as ind

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _close(a, b, atol=1e-12, rtol=1e-12):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    same_inf = (np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b)))
    fin = ~same_inf
    assert np.all(np.isfinite(a[fin])) and np.all(np.isfinite(b[fin])), "non-finite mismatch"
    err = np.abs(a[fin] - b[fin])
    lim = atol + rtol * np.abs(b[fin])
    assert np.all(err <= lim), f"max err {err.max() if err.size else 0} (worst at {np.argmax(err - lim)})"


# ---------------------------------------------------------------- decoders
def check_e4m3(lib=None):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3(b, lib) for b in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got)), "NaN codes differ"
    assert np.array_equal(ref[~nan], got[~nan]), "e4m3 values differ from torch.float8_e4m3fn"
    spots = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
             0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for b, v in spots.items():
        assert oracle.e4m3(b, lib) == v, (hex(b), oracle.e4m3(b, lib), v)
    assert math.isnan(oracle.e4m3(0x7F, lib)) and math.isnan(oracle.e4m3(0xFF, lib))


def check_ue8m0(lib=None):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    got = np.array([oracle.ue8m0(b, lib) for b in range(256)])
    assert np.isnan(got[255]) and np.isnan(ref[255])
    assert np.array_equal(ref[:255], got[:255]), "UE8M0 differs from torch.float8_e8m0fnu"
    assert oracle.ue8m0(127, lib) == 1.0 and oracle.ue8m0(128, lib) == 2.0 and oracle.ue8m0(120, lib) == 2.0 ** -7


def check_bf16(lib=None):
    rng = np.random.default_rng(7)
    bits = np.concatenate([np.array([0x0000, 0x8000, 0x3F80, 0x4000, 0xC040, 0x0001, 0x7F7F]),
                           rng.integers(0, 0x7F80, 500), rng.integers(0x8000, 0xFF80, 500)]).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16(int(b), lib) for b in bits])
    assert np.array_equal(ref, got)


# ---------------------------------------------------------------- layout
def check_translation_fixture(lib=None):
    g = json.load(open(os.path.join(GOLDEN, "translate_small.json")))
    bt = np.array(g["block_table"], np.int32)
    sl = np.array(g["seq_lens"], np.int32)
    idx = np.array(g["topk_idx"], np.int32)
    cache = np.zeros((g["num_pages"], W.PAGE_BYTES), np.uint8)
    _, ps = oracle.gather(cache, bt, idx, sl, lib=lib)
    assert np.array_equal(ps, np.array(g["expected_page_slot"], np.int32)), ps.tolist()


def _marker_cache():
    """3 pages; a few tokens carry marker bytes at hand-computed offsets."""
    cache = np.zeros((3, W.PAGE_BYTES), np.uint8)
    flat = cache.reshape(-1)
    marks = []  # (page, slot, nope_code, scale_bytes[7], rope_bits)
    for page, slot, code in [(2, 0, 0x38), (2, 255, 0x40), (0, 43, 0xB8), (1, 99, 0x30)]:
        row = page * 149504 + slot * 576
        scl = page * 149504 + 147456 + slot * 8
        flat[row : row + 448] = code
        sbytes = [127 + ((page + slot + g) % 5) - 2 for g in range(7)]
        flat[scl : scl + 7] = sbytes
        flat[scl + 7] = 0xAB  # padding byte: must be ignored
        rope = np.array([0x3F80, 0x4000, 0xC040, 0x0000] * 16, np.uint16)  # 1, 2, -3, 0
        flat[row + 448 : row + 576] = rope.view(np.uint8)
        marks.append((page, slot, code, sbytes))
    return cache, marks


def check_byte_layout(lib=None):
    cache, marks = _marker_cache()
    value = {0x38: 1.0, 0x40: 2.0, 0xB8: -1.0, 0x30: 0.5}
    for page, slot, code, sbytes in marks:
        bt = np.array([[page]], np.int32)
        lat, ps = oracle.gather(cache, bt, np.array([[slot]], np.int32), np.array([256], np.int32), lib=lib)
        assert ps[0, 0].tolist() == [page, slot]
        exp = np.empty(512)
        for d in range(448):
            exp[d] = value[code] * 2.0 ** (sbytes[d // 64] - 127)
        exp[448:] = [1.0, 2.0, -3.0, 0.0] * 16
        assert np.array_equal(lat[0, 0], exp), (page, slot)


# ---------------------------------------------------------------- attention
def _tiny(seed=0, B=3, topk=24, seq=(300, 40, 513), **kw):
    return W.make_custom(B, topk, seq, seed=seed, fill="all", **kw)


def _dec(w, lib=None, idx=None, q=None):
    return oracle.decode(w.q[0] if q is None else q, w.cache, w.block_table,
                         w.topk_idx[0] if idx is None else idx, w.seq_lens, w.sm_scale, lib=lib)


def check_two_token_closed_form(lib=None):
    # q = 2 e_0, k1 nope[0] = 1, k2 nope[0] = -1, everything else 0, sm_scale 1/2:
    # s = (+1, -1), O[0] = tanh(1), LSE = ln(e + 1/e) = ln(2 cosh 1).
    cache = np.zeros((1, W.PAGE_BYTES), np.uint8)
    flat = cache.reshape(-1)
    flat[0 * 576] = 0x38  # token 0, dim 0: +1.0
    flat[1 * 576] = 0xB8  # token 1, dim 0: -1.0
    flat[147456 : 147456 + 7] = 127
    flat[147456 + 8 : 147456 + 15] = 127
    q = np.zeros((1, 1, 512), np.uint16)
    q[0, 0, 0] = 0x4000  # 2.0
    o, l = oracle.decode(q, cache, np.array([[0]], np.int32), np.array([[1, 0]], np.int32),
                         np.array([2], np.int32), 0.5, lib=lib)
    exp = np.zeros(512)
    exp[0] = math.tanh(1.0)
    _close(o[0, 0], exp, atol=1e-15)
    _close(l[0, 0], math.log(2.0 * math.cosh(1.0)), atol=1e-15)
    # shifting both scores by a large constant leaves O unchanged and moves LSE by it
    q2 = q.copy()
    q2[0, 0, 448] = 0x4000  # q rope[0] = 2
    flat[448:450] = np.array([0x4480], np.uint16).view(np.uint8)  # k1 rope[0] = 1024
    flat[576 + 448 : 576 + 450] = np.array([0x4480], np.uint16).view(np.uint8)  # k2 rope[0] = 1024
    o2, l2 = oracle.decode(q2, cache, np.array([[0]], np.int32), np.array([[1, 0]], np.int32),
                           np.array([2], np.int32), 0.5, lib=lib)
    exp2 = exp.copy()
    exp2[448] = 1024.0
    _close(o2[0, 0], exp2, atol=1e-12)
    _close(l2[0, 0], 1024.0 + math.log(2.0 * math.cosh(1.0)), atol=1e-12)


def check_single_and_equal_slots(lib=None):
    w = _tiny(1)
    idx = w.topk_idx[0].copy()
    b, j = 0, 17
    page, slot = w.block_table[b, j // 256], j % 256
    kj = ind.token_latents(w.cache, [page], [slot])[0]
    qv = ind.q_values(w.q[0])
    s = w.sm_scale * qv[b] @ kj  # [H]
    # topk = 1 -> O = k_j, LSE = s_j
    o, l = _dec(w, lib, idx=np.full((w.B, 1), j, np.int32))
    _close(o[b], np.broadcast_to(kj, o[b].shape), atol=1e-12)
    _close(l[b], s, atol=1e-12)
    # all slots equal -> O = k_j, LSE = s_j + ln(topk)
    idx[:] = j
    o, l = _dec(w, lib, idx=idx)
    _close(o[b], np.broadcast_to(kj, o[b].shape), atol=1e-12)
    _close(l[b], s + math.log(w.topk), atol=1e-12)


def check_zero_q_mean(lib=None):
    w = _tiny(2, pad_fraction=0.3)
    o, l = _dec(w, lib, q=np.zeros_like(w.q[0]))
    for b in range(w.B):
        v = [i for i in w.topk_idx[0, b] if 0 <= i < w.seq_lens[b]]
        K = ind.token_latents(w.cache, w.block_table[b, np.array(v) // 256], np.array(v) % 256)
        _close(o[b], np.broadcast_to(K.mean(axis=0), o[b].shape), atol=1e-12)
        _close(l[b], np.full(w.H, math.log(len(v))), atol=1e-12)


def check_permutation_and_padding(lib=None):
    w = _tiny(3, pad_fraction=0.25)
    o, l = _dec(w, lib)
    rng = np.random.default_rng(11)
    perm = np.stack([rng.permutation(w.topk) for _ in range(w.B)])
    idx_p = np.take_along_axis(w.topk_idx[0], perm, axis=1)
    o2, l2 = _dec(w, lib, idx=idx_p)
    _close(o2, o, atol=1e-12)
    _close(l2, l, atol=1e-12)
    # -1 slots contribute nothing: the compacted list gives the same answer
    for b in range(w.B):
        v = np.array([i for i in w.topk_idx[0, b] if i >= 0], np.int32)
        o3, l3 = oracle.decode(w.q[0][b : b + 1], w.cache, w.block_table[b : b + 1], v[None, :],
                               w.seq_lens[b : b + 1], w.sm_scale, lib=lib)
        _close(o3[0], o[b], atol=1e-12)
        _close(l3[0], l[b], atol=1e-12)


def check_dense_brute_force(lib=None):
    for seed, kw in [(4, {}), (5, dict(pad_fraction=0.3, duplicates=True)), (6, dict(outlier_fraction=0.1))]:
        w = _tiny(seed, **kw)
        o, l = _dec(w, lib)
        od, ld = ind.dense_attention(w.q[0], w.cache, w.block_table, w.topk_idx[0], w.seq_lens, w.sm_scale)
        _close(o, od, atol=1e-10, rtol=1e-10)
        _close(l, ld, atol=1e-10, rtol=1e-12)
    # a request with no valid slot: O = 0, LSE = -inf
    w = _tiny(7, seq=(300, 0, 40))
    o, l = _dec(w, lib)
    assert np.all(o[1] == 0.0) and np.all(l[1] == -np.inf)


def check_combine_identity(lib=None):
    w = _tiny(8, B=2, topk=40, seq=(600, 300))
    idx = w.topk_idx[0]
    full_o, full_l = _dec(w, lib)
    parts = [idx.copy() for _ in range(3)]
    parts[0][:, 14:] = -1
    parts[1][:, :14] = -1
    parts[1][:, 30:] = -1
    parts[2][:, :30] = -1
    parts.append(np.full_like(idx, -1))  # an empty split: weight 0
    po, pl = zip(*[_dec(w, lib, idx=p) for p in parts])
    co, cl = oracle.combine(np.stack(po, axis=2), np.stack(pl, axis=2), lib=lib)
    _close(co, full_o, atol=1e-12, rtol=1e-12)
    _close(cl, full_l, atol=1e-12, rtol=1e-12)
    # all splits empty -> O = 0, LSE = -inf
    e = np.full((1, 2, 3), -np.inf)
    co, cl = oracle.combine(np.ones((1, 2, 3, 512)), e, lib=lib)
    assert np.all(co == 0.0) and np.all(cl == -np.inf)
    # two splits with hand values: weights e^1 : e^0 -> L = ln(e + 1), O = (e a + b) / (e + 1)
    a = np.full(512, 3.0)
    bvec = np.full(512, -1.0)
    co, cl = oracle.combine(np.stack([a, bvec])[None, None], np.array([[[1.0, 0.0]]]), lib=lib)
    _close(cl[0, 0], math.log(math.e + 1.0), atol=1e-15)
    _close(co[0, 0], (math.e * a + bvec) / (math.e + 1.0), atol=1e-14)


# ---------------------------------------------------------------- cache writer
def check_e4m3_encode(lib=None):
    # every finite code round-trips, both signs (0x80 is -0)
    for c in list(range(0x7F)) + list(range(0x80, 0xFF)):
        assert oracle.e4m3_encode(oracle.e4m3(c, lib), lib) == c, hex(c)
    # the midpoint between two neighbouring codes goes to the even one; a hair either side to the nearer
    for c in range(0x7E):
        lo, hi = oracle.e4m3(c, lib), oracle.e4m3(c + 1, lib)
        mid = 0.5 * (lo + hi)
        assert oracle.e4m3_encode(mid, lib) == (c if c % 2 == 0 else c + 1), hex(c)
        assert oracle.e4m3_encode(mid - (hi - lo) * 1e-6, lib) == c
        assert oracle.e4m3_encode(mid + (hi - lo) * 1e-6, lib) == c + 1
        assert oracle.e4m3_encode(-mid, lib) == 0x80 | (c if c % 2 == 0 else c + 1)
    # saturation and special values
    for x, code in ((448.0, 0x7E), (460.0, 0x7E), (1e6, 0x7E), (np.inf, 0x7E), (-np.inf, 0xFE), (-500.0, 0xFE),
                    (np.nan, 0x7F), (0.0, 0x00), (-0.0, 0x80), (2.0 ** -11, 0x00), (3 * 2.0 ** -11, 0x01)):
        assert oracle.e4m3_encode(x, lib) == code, (x, hex(oracle.e4m3_encode(x, lib)), hex(code))
    # against torch's cast (round to nearest even) on float32 values inside the finite range
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(4000) * np.exp2(rng.uniform(-14, 9, 4000))).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v), lib) for v in x], np.uint8)
    assert np.array_equal(got, ref), np.flatnonzero(got != ref)[:5]


def check_bf16_encode(lib=None):
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 1 << 32, 20000, dtype=np.uint64).astype(np.uint32)
    bits = bits[((bits >> 23) & 0xFF) != 0xFF]  # finite binary32 values (subnormals included)
    ties = (rng.integers(0, 1 << 16, 200, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000  # exact midpoints
    ties = ties[((ties >> 23) & 0xFF) != 0xFF]
    x = np.concatenate([bits, ties]).view(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_encode(float(v), lib) for v in x], np.uint16)
    assert np.array_equal(got, ref), np.flatnonzero(got != ref)[:5]
    assert oracle.bf16_encode(float("nan"), lib) == 0x7FC0
    assert oracle.bf16_encode(float("inf"), lib) == 0x7F80 and oracle.bf16_encode(float("-inf"), lib) == 0xFF80
    assert oracle.bf16_encode(3.4e38, lib) == 0x7F80  # past the largest finite bf16 by more than half an ulp


def check_scale_exponent(lib=None):
    g = np.zeros(64, np.float32)
    assert oracle.scale_exponent(g, lib) == -127  # all zero
    for k in (-120, -30, -8, -1, 0, 1, 5, 20, 100, 119):  # 448 * 2^119 is the largest in binary32
        a = np.float32(448.0 * 2.0 ** k)
        g[:] = 0.0
        g[17] = -a
        assert oracle.scale_exponent(g, lib) == k, k  # amax exactly 448 * 2^k: x / 2^k fits
        g[17] = np.nextafter(a, np.float32(np.inf))
        assert oracle.scale_exponent(g, lib) == k + 1, k  # just above: one more
    g[:] = 1.0
    assert oracle.scale_exponent(g, lib) == -8  # 1 <= 448 * 2^-8 = 1.75 but > 0.875
    g[:] = np.float32(1e-44)
    assert oracle.scale_exponent(g, lib) == -127  # below 448 * 2^-127: clamped
    g[3] = np.inf
    assert oracle.scale_exponent(g, lib) == 127
    g[3] = np.nan
    assert oracle.scale_exponent(g, lib) == 127


def check_quantize_vs_generator(lib=None):
    rng = np.random.default_rng(13)
    x = rng.standard_normal((24, 512)).astype(np.float32)
    x[3] *= 20.0  # an outlier row
    x[5, :64] *= 1e-3  # groups of very different magnitudes
    x[6, 64:128] = 0.0  # an all-zero group
    x[7, 128:192] *= 1e4
    rows, scales = W.quantize_rows(x)
    for i in range(x.shape[0]):
        r, sc = oracle.quantize_token(x[i], lib)
        assert np.array_equal(r, rows[i]), i
        assert np.array_equal(sc, scales[i]), i
    # decoding a written token gives every nope value within half an e4m3 step of x / 2^e (times 2^e)
    cache = np.zeros((1, W.PAGE_BYTES), np.uint8)
    written = oracle.write_kv(x[:2], [0, 0], [5, 200], np.array([[0]], np.int32), cache, lib)
    assert written == 0
    lat, _ = oracle.gather(cache, np.array([[0]], np.int32), np.array([[5, 200]], np.int32),
                           np.array([256], np.int32), lib)
    for j in range(2):
        for g in range(7):
            e = oracle.scale_exponent(x[j, 64 * g:64 * g + 64], lib)
            step = np.exp2(np.floor(np.log2(np.maximum(np.abs(x[j, 64 * g:64 * g + 64]) / 2.0 ** e, 2.0 ** -6))) - 3)
            assert np.all(np.abs(lat[0, j, 64 * g:64 * g + 64] - x[j, 64 * g:64 * g + 64]) <= 0.5 * step * 2.0 ** e)


def check_write_scatter(lib=None):
    rng = np.random.default_rng(14)
    x = rng.standard_normal((6, 512)).astype(np.float32)
    bt = np.array([[2, 0], [1, -1]], np.int32)  # request 0: pages 2, 0; request 1: page 1, then none
    cache = np.full((3, W.PAGE_BYTES), 0xA5, np.uint8)
    req = np.array([0, 0, 1, 1, 2, 0], np.int32)
    pos = np.array([3, 300, 255, 256, 0, -1], np.int32)  # (0,3) (0,300) (1,255) ok; the rest skipped
    skipped = oracle.write_kv(x, req, pos, bt, cache, lib)
    assert skipped == 3
    expect = np.full((3, W.PAGE_BYTES), 0xA5, np.uint8)
    for i, (page, slot) in enumerate([(2, 3), (0, 44), (1, 255)]):
        r, sc = oracle.quantize_token(x[i], lib)
        expect[page, slot * 576:(slot + 1) * 576] = r
        expect[page, 147456 + slot * 8:147456 + slot * 8 + 8] = sc
    assert np.array_equal(cache, expect)


ALL_CHECKS = [check_e4m3, check_ue8m0, check_bf16, check_translation_fixture, check_byte_layout,
              check_two_token_closed_form, check_single_and_equal_slots, check_zero_q_mean,
              check_permutation_and_padding, check_dense_brute_force, check_combine_identity,
              check_e4m3_encode, check_bf16_encode, check_scale_exponent, check_quantize_vs_generator,
              check_write_scatter]
