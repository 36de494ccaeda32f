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


def test_noalloc_matches_workspace_entry_point_twice():
    assert torch.cuda.is_available()
    lib = ctypes.CDLL(build.build())
    P, I = ctypes.c_void_p, ctypes.c_int
    fn = lib.smla_decode_noalloc
    fn.argtypes = [P, P, P, P, P, ctypes.c_float, P, P, I, I, I, I, I, P]
    fn.restype = I
    stream = torch.cuda.current_stream()
    # two calls in a row: split-K partials (B=64 -> 2 splits, B=1 -> 4 splits) live in the shared scratch
    for k in (4, 2):
        w = W.make_config(k)
        d = device_inputs(w)
        ref_o, ref_l = smla.decode(d["q"], d["kv_cache"], d["block_table"], d["topk_idx"], d["seq_lens"],
                                   d["sm_scale"])
        out = torch.full((w.B, 64, 512), float("nan"), device="cuda")
        lse = torch.full((w.B, 64), float("nan"), device="cuda")
        rc = fn(d["q"].data_ptr(), d["kv_cache"].data_ptr(), d["block_table"].data_ptr(), d["topk_idx"].data_ptr(),
                d["seq_lens"].data_ptr(), ctypes.c_float(w.sm_scale), out.data_ptr(), lse.data_ptr(), w.B, 64,
                w.topk, w.max_blocks, w.num_pages, stream.cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        _close(out, lse, ref_o, ref_l)
    # bad sizes are rejected before any launch
    assert fn(d["q"].data_ptr(), d["kv_cache"].data_ptr(), d["block_table"].data_ptr(), d["topk_idx"].data_ptr(),
              d["seq_lens"].data_ptr(), ctypes.c_float(w.sm_scale), out.data_ptr(), lse.data_ptr(), w.B, 32,
              w.topk, w.max_blocks, w.num_pages, stream.cuda_stream) == -1
