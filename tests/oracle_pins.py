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


ALL_CHECKS = [check_e4m3, check_ue8m0, check_bf16, check_translation_fixture, check_byte_layout,
              check_two_token_closed_form, check_single_and_equal_slots, check_zero_q_mean,
              check_permutation_and_padding, check_dense_brute_force, check_combine_identity]
