"""smla_decode_noalloc, the entry point for callers that cannot allocate (needs a B200).

Some callers cannot give the library a workspace: a serving engine that froze
its device memory pool after capturing its decode step into CUDA graphs, or a
plugin host that owns every device allocation.  smla_decode_noalloc serves them
from a scratch array inside the library's device image.  This file checks, through
the C ABI, that two calls in a row give the same results as smla_decode with a
caller workspace, within the parity tolerances used by every GPU test.  It is
named to run last, so a run that stops at the first failure has run the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_mla_decode_fp8_b200 as smla
from sparse_mla_decode_fp8_b200 import build
from sparse_mla_decode_fp8_b200 import workloads as W
from tests.gpu_util import LSE_MAX_ABS, O_MAX_ABS, O_REL_L2, device_inputs

pytestmark = pytest.mark.gpu


def _close(o, l, ro, rl):
    o, l, ro, rl = (t.double().cpu().numpy() for t in (o, l, ro, rl))
    assert np.array_equal(np.isneginf(l), np.isneginf(rl))
    fin = ~np.isneginf(rl)
    assert np.abs(o - ro).max() <= O_MAX_ABS
    assert np.linalg.norm(o - ro) <= O_REL_L2 * np.linalg.norm(ro)
    assert np.abs(l[fin] - rl[fin]).max() <= LSE_MAX_ABS


def _noalloc_fn():
    lib = ctypes.CDLL(build.build())
    P, I = ctypes.c_void_p, ctypes.c_int
    fn = lib.smla_decode_noalloc
    fn.argtypes = [P, P, P, P, P, ctypes.c_float, P, P, I, I, I, I, I, P]
    fn.restype = I
    return fn


def _call(fn, w, d, out, lse, H=64):
    return fn(d["q"].data_ptr(), d["kv_cache"].data_ptr(), d["block_table"].data_ptr(), d["topk_idx"].data_ptr(),
              d["seq_lens"].data_ptr(), ctypes.c_float(w.sm_scale), out.data_ptr(), lse.data_ptr(), w.B, H,
              w.topk, w.max_blocks, w.num_pages, torch.cuda.current_stream().cuda_stream)


def _workloads():
    # split-K partials in the one scratch array, through every merge path:
    #   B=64 topk=512 -> 2 splits (pair merge), B=1 topk=512 -> 4 splits (cluster merge),
    #   B=1 topk=2048 -> 16 splits (global partials + merge kernel),
    #   B=29 topk=640 -> 5 splits on 145 CTAs: 19.0 MB of partials, near the 19.4 MB worst case
    yield W.make_config(4)
    yield W.make_config(2)
    yield W.make_custom(1, 2048, [100000], seed=21, fill="referenced")
    yield W.make_custom(29, 640, [4000 + 97 * b for b in range(29)], seed=22, fill="referenced")


def test_noalloc_matches_workspace_entry_point_in_sequence():
    assert torch.cuda.is_available()
    fn = _noalloc_fn()
    seen = set()
    for w in _workloads():
        seen.add(smla.num_splits(w.B, w.topk))
        d = device_inputs(w)
        ref_o, ref_l = smla.decode(d["q"], d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"],
                                   d["sm_scale"])
        out = torch.full((w.B, 64, 512), float("nan"), device="cuda")
        lse = torch.full((w.B, 64), float("nan"), device="cuda")
        assert _call(fn, w, d, out, lse) == 0
        torch.cuda.synchronize()
        _close(out, lse, ref_o, ref_l)
    assert seen == {2, 4, 16, 5}
    # bad sizes are rejected before any launch
    assert _call(fn, w, d, out, lse, H=32) == -1


def test_noalloc_allocates_nothing():
    fn = _noalloc_fn()
    w = W.make_custom(29, 640, [4000 + 97 * b for b in range(29)], seed=22, fill="referenced")
    d = device_inputs(w)
    out = torch.empty((w.B, 64, 512), device="cuda")
    lse = torch.empty((w.B, 64), device="cuda")
    assert _call(fn, w, d, out, lse) == 0  # warm-up: module load, attributes
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _call(fn, w, d, out, lse) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
