"""Argument checks and the bounded-wait error path (needs a B200)."""
import ctypes

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


def test_invalid_arguments_rejected_without_launch():
    lib = smla.library()
    w = W.make_config(1)
    d = device_inputs(w)
    ws = smla.binding.new_workspace(1, 64)
    out = torch.empty((1, 64, 512), device="cuda")
    lse = torch.empty((1, 64), device="cuda")
    base = [d["q"].data_ptr(), d["kv_cache"].data_ptr(), d["block_table"].data_ptr(), d["topk_idx"].data_ptr(),
            d["seq_lens"].data_ptr(), ctypes.c_float(w.sm_scale), out.data_ptr(), lse.data_ptr(), 1, 64, 64, 4, 4,
            ws.data_ptr(), ws.numel(), None]
    assert lib.smla_decode(*base) == 0
    bad = {9: 32, 10: 0, 11: 0, 12: 1 << 23, 14: 100}  # H, topk, max_blocks, num_pages, workspace too small
    for pos, val in bad.items():
        args = list(base)
        args[pos] = val
        assert lib.smla_decode(*args) == -1, pos
    args = list(base)
    args[1] = d["kv_cache"].data_ptr() + 8  # misaligned cache
    assert lib.smla_decode(*args) == -1
    args = list(base)
    args[0] = None
    assert lib.smla_decode(*args) == -1
    args = list(base)
    args[5] = ctypes.c_float(float("nan"))
    assert lib.smla_decode(*args) == -1
    torch.cuda.synchronize()
    assert smla.read_error(ws) == 0


@pytest.mark.parametrize("nsplit", [1, 2, 3, 16])
def test_wait_timeout_reports_poisons_and_context_survives(nsplit):
    # The debug hook sends tile 0's S^T commit elsewhere, so every CTA's workers run out of
    # their 2 ms wait.  Such a call must flag the timeout AND leave its out/lse rows NaN
    # through every merge path: direct (1 split), the pair's atomic adds (2), the cluster
    # exchange (3) and the partials + combine kernel (16).  The next call is normal.
    if nsplit == 16:
        w = W.make_custom(1, 2048, [100000], seed=11, fill="referenced")
    else:
        w = W.make_config(2)
    d = device_inputs(w)
    ws = smla.binding.new_workspace(w.B, w.topk, nsplit=nsplit)
    args = (d["q"], d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"], d["sm_scale"])
    out = torch.zeros((w.B, 64, 512), device="cuda")
    lse = torch.zeros((w.B, 64), device="cuda")
    smla.decode(*args, out=out, lse=lse, workspace=ws, nsplit=nsplit, wait_timeout_ns=2_000_000,
                debug_flags=smla.SMLA_DEBUG_SKIP_FIRST_COMMIT)
    torch.cuda.synchronize()
    flags = smla.read_error(ws)
    assert flags & smla.SMLA_FLAG_TIMEOUT
    assert torch.isnan(out).all() and torch.isnan(lse).all()
    out, lse = smla.decode(*args, workspace=ws, nsplit=nsplit)
    assert smla.read_error(ws) == 0
    ro, rl = oracle.decode(w.q[0], w.cache, w.block_table, w.topk_idx[0], w.seq_lens, w.sm_scale)
    parity(out, lse, ro, rl)
