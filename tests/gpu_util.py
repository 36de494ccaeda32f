"""Helpers for the GPU parity tests: device copies of a workload and the tolerance checks.

Tolerances (the sparse MLA decode target): max|dO| <= 2e-3, relative L2 of O
<= 5e-3, |dLSE| <= 1e-3 on finite entries, and -inf LSE exactly where the
oracle has -inf (requests with no valid slot).
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 2e-3
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


def device_inputs(w, r: int = 0, device="cuda"):
    return dict(
        q=torch.from_numpy(np.ascontiguousarray(w.q[r]).view(np.int16)).view(torch.bfloat16).to(device),
        kv_cache=torch.from_numpy(w.cache).to(device),
        block_table=torch.from_numpy(np.ascontiguousarray(w.block_table)).to(device),
        topk_idx=torch.from_numpy(np.ascontiguousarray(w.topk_idx[r])).to(device),
        seq_lens=torch.from_numpy(np.ascontiguousarray(w.seq_lens)).to(device),
        sm_scale=w.sm_scale,
    )


def parity(out, lse, ref_out, ref_lse):
    """Returns the error figures; raises AssertionError if a bound is broken."""
    o = out.detach().double().cpu().numpy() if isinstance(out, torch.Tensor) else np.asarray(out, np.float64)
    l = lse.detach().double().cpu().numpy() if isinstance(lse, torch.Tensor) else np.asarray(lse, np.float64)
    ro = np.asarray(ref_out, np.float64)
    rl = np.asarray(ref_lse, np.float64)
    assert o.shape == ro.shape and l.shape == rl.shape
    assert np.all(np.isfinite(o)), "non-finite output"
    d = np.abs(o - ro)
    max_abs = float(d.max()) if d.size else 0.0
    nrm = float(np.linalg.norm(ro))
    rel = float(np.linalg.norm(o - ro) / nrm) if nrm > 0 else float(np.linalg.norm(o))
    ref_inf = np.isneginf(rl)
    assert np.array_equal(ref_inf, np.isneginf(l)), "-inf LSE pattern differs"
    fin = ~ref_inf
    lse_abs = float(np.abs(l[fin] - rl[fin]).max()) if fin.any() else 0.0
    figs = dict(max_abs=max_abs, rel_l2=rel, lse_abs=lse_abs)
    assert max_abs <= O_MAX_ABS, figs
    assert rel <= O_REL_L2, figs
    assert lse_abs <= LSE_MAX_ABS, figs
    return figs
