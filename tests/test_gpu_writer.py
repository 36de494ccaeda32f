"""The CUDA cache writer (smla_write_kv) against the oracle's writer, byte for byte (needs a B200).

Both sides quantise the same latents with the rule of the synthetic caches (per 64-dim
UE8M0 scale, e4m3 and bf16 round to nearest even) and scatter them through the block
table; every byte of the cache must agree, including the untouched ones and the special
cases (all-zero, tiny and huge groups, exact powers 448 * 2^k, ties, infinities, NaN).
"""
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
    assert torch.cuda.is_available()
    build.build()
    smla.library()


def _latents(n, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 512)).astype(np.float32)
    x[::7] *= 20.0  # outlier rows
    x[1, 0:64] = 0.0  # an all-zero group (scale byte 0)
    x[2, 64:128] *= np.float32(1e-39)  # subnormal binary32 values: the scale clamps at 2^-127
    x[3, 128:192] *= np.float32(1e30)  # a huge group
    x[4, 192:256] = np.float32(448.0 * 2.0 ** -3)  # amax exactly 448 * 2^k: e = k, x / 2^e = 448
    x[4, 200] = np.nextafter(np.float32(56.0), np.float32(np.inf))  # ... one ulp above: e = k + 1
    # e4m3 ties after scaling (amax 448 -> e = 0): midpoints between neighbouring codes
    mids = np.array([1.0625, 1.1875, 3.0 * 2.0 ** -10, 0.5 * 2.0 ** -9, 2.0 ** -10, 13.0, 15.0, 240.0], np.float32)
    x[5, 256:320] = np.resize(np.concatenate([mids, -mids]), 64)
    x[5, 256] = 448.0
    x[6, 320:384] = np.float32(2.0 ** -12) * rng.standard_normal(64).astype(np.float32)  # e4m3 subnormal range
    x[6, 320] = 1.0
    x[8, 384:448] *= 3.0
    x[8, 400] = np.inf  # a non-finite group: e = 127, inf -> 448
    x[9, 10] = np.nan  # NaN -> 0x7F
    x[10, 450] = np.nan  # NaN rope value -> 0x7FC0
    x[11, 460] = -np.inf
    ties = (rng.integers(0, 1 << 16, 64, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    ties[(ties >> 23 & 0xFF) == 0xFF] &= 0x807FFFFF
    x[12, 448:] = ties.view(np.float32)  # bf16 ties
    return x


def _destinations(n, seed, B, max_blocks):
    rng = np.random.default_rng(seed)
    flat = rng.choice(B * max_blocks * 256, size=n, replace=False)  # distinct (request, position)
    req = (flat // (max_blocks * 256)).astype(np.int32)
    pos = (flat % (max_blocks * 256)).astype(np.int32)
    req[3], pos[5], pos[7], req[9] = -1, -4, max_blocks * 256 + 3, B  # out of range: skipped
    return req, pos


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_writer_bytes_match_oracle(dtype):
    n, B, max_blocks, P = 300, 3, 4, 10
    x = _latents(n, 40 if dtype == "fp32" else 41)
    req, pos = _destinations(n, 42, B, max_blocks)
    bt = np.array([[7, 0, 3, -1], [2, 9, 11, 5], [4, 1, 6, 8]], np.int32)  # -1 and 11 are out of [0, 10)
    cache0 = np.full((P, W.PAGE_BYTES), 0x5A, np.uint8)
    xt = torch.from_numpy(x).cuda()
    if dtype == "bf16":
        xt = xt.to(torch.bfloat16)
        x = xt.float().cpu().numpy()  # the oracle gets the same (bf16-valued) inputs
    dcache = torch.from_numpy(cache0.copy()).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    smla.write_kv(xt, torch.from_numpy(req).cuda(), torch.from_numpy(pos).cuda(), torch.from_numpy(bt).cuda(),
                  dcache, err=err)
    torch.cuda.synchronize()
    ref = cache0.copy()
    skipped = oracle.write_kv(x, req, pos, bt, ref)
    assert skipped >= 4
    got = dcache.cpu().numpy()
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, (bad[:8], got.reshape(-1)[bad[:8]], ref.reshape(-1)[bad[:8]])
    assert int(err.item()) == smla.SMLA_FLAG_BAD_PAGE


def test_writer_then_decode_matches_oracle():
    # a cache written by the writer decodes like the oracle's reading of the same latents
    B, seq, topk = 2, 700, 256
    rng = np.random.default_rng(43)
    pages = (seq + 255) // 256
    bt = rng.permutation(B * pages).astype(np.int32).reshape(B, pages)
    lat = rng.standard_normal((B * seq, 512)).astype(np.float32)
    lat[::50] *= 20.0
    req = np.repeat(np.arange(B, dtype=np.int32), seq)
    pos = np.tile(np.arange(seq, dtype=np.int32), B)
    dcache = torch.zeros((B * pages, W.PAGE_BYTES), dtype=torch.uint8, device="cuda")
    smla.write_kv(torch.from_numpy(lat).cuda(), torch.from_numpy(req).cuda(), torch.from_numpy(pos).cuda(),
                  torch.from_numpy(bt).cuda(), dcache)
    ref = np.zeros((B * pages, W.PAGE_BYTES), np.uint8)
    assert oracle.write_kv(lat, req, pos, bt, ref) == 0
    assert np.array_equal(dcache.cpu().numpy(), ref)
    idx = np.stack([rng.choice(seq, topk, replace=False) for _ in range(B)]).astype(np.int32)
    q = W.to_bf16_bits(rng.standard_normal((B, 64, 512)).astype(np.float32))
    sl = np.full(B, seq, np.int32)
    w = W.Workload("written", q[None], ref, bt, idx[None], sl, 512 ** -0.5)
    d = device_inputs(w)
    out, lse = smla.decode(d["q"], dcache, d["block_table"], d["topk_idx"], d["seq_lens"], d["sm_scale"])
    ro, rl = oracle.decode(q, ref, bt, idx, sl, 512 ** -0.5)
    parity(out, lse, ro, rl)
