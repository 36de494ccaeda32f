"""ctypes binding of libsmla.so: argument marshalling only.

Names follow the C ABI (``include/smla.h``): ``decode`` -> ``smla_decode_ex``,
``combine`` -> ``smla_combine``, ``debug_gather`` -> ``smla_debug_gather``,
``workspace_bytes`` -> ``smla_workspace_bytes_ex``, ``read_error`` ->
``smla_read_error``.  Tensors must already be on the current CUDA device, dense
and of the documented dtype; nothing is copied or converted here.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

SMLA_FLAG_BAD_PAGE = 0x1
SMLA_FLAG_TIMEOUT = 0x2
SMLA_FLAG_SMEM = 0x4
SMLA_DEBUG_SKIP_FIRST_COMMIT = 0x1
HEADS = 64
DIM = 512
PAGE_BYTES = 149504

_ERRORS = {-1: "invalid argument", -2: "unsupported device (needs sm_100)", -3: "CUDA runtime error",
           -4: "kernel launch failed"}


class SmlaError(RuntimeError):
    pass


class _Options(ctypes.Structure):
    _fields_ = [("nsplit", ctypes.c_int), ("out_bf16", ctypes.c_int), ("wait_timeout_ns", ctypes.c_uint64),
                ("debug_flags", ctypes.c_uint32), ("reserved1", ctypes.c_uint32)]


_lock = threading.Lock()
_lib = None


def library():
    """Load libsmla.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_build.LIB):
                raise SmlaError(f"{_build.LIB} is missing: build it with sparse_mla_decode_fp8_b200.build.build()")
            lib = ctypes.CDLL(_build.LIB)
            P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            lib.smla_decode.argtypes = [P, P, P, P, P, ctypes.c_float, P, P, I, I, I, I, I, P, Z, P]
            lib.smla_decode.restype = I
            lib.smla_decode_ex.argtypes = [P, P, P, P, P, ctypes.c_float, P, P, I, I, I, I, I, P, Z,
                                           ctypes.POINTER(_Options), P]
            lib.smla_decode_ex.restype = I
            lib.smla_combine.argtypes = [P, P, I, P, P, I, I, P]
            lib.smla_combine.restype = I
            lib.smla_num_splits.argtypes = [I, I, I]
            lib.smla_num_splits.restype = I
            lib.smla_workspace_bytes.argtypes = [I, I, I]
            lib.smla_workspace_bytes.restype = Z
            lib.smla_workspace_bytes_ex.argtypes = [I, I, I, I]
            lib.smla_workspace_bytes_ex.restype = Z
            lib.smla_read_error.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
            lib.smla_read_error.restype = I
            lib.smla_debug_gather.argtypes = [P, P, P, P, I, I, I, I, P, P, P, Z, P]
            lib.smla_debug_gather.restype = I
            lib.smla_write_kv.argtypes = [P, I, I, P, P, P, I, I, I, P, P, P]
            lib.smla_write_kv.restype = I
            lib.smla_version.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise SmlaError(f"{what}: {_ERRORS.get(rc, rc)}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise SmlaError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise SmlaError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise SmlaError(f"{name} must be contiguous")
    return t.data_ptr()


def version() -> str:
    return library().smla_version().decode()


def num_splits(B: int, topk: int) -> int:
    n = library().smla_num_splits(B, HEADS, topk)
    _check(min(n, 0), "smla_num_splits")
    return n


def workspace_bytes(B: int, topk: int, nsplit: int = 0) -> int:
    lib = library()
    n = lib.smla_workspace_bytes_ex(B, HEADS, topk, nsplit) if nsplit else lib.smla_workspace_bytes(B, HEADS, topk)
    if n == 0:
        raise SmlaError("smla_workspace_bytes: invalid sizes")
    return int(n)


def new_workspace(B: int, topk: int, nsplit: int = 0, device=None) -> torch.Tensor:
    """A zeroed uint8 workspace of the required size (the first 4 bytes are the error word)."""
    n = workspace_bytes(B, topk, nsplit)
    return torch.zeros(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def decode(q, kv_cache, block_table, topk_idx, seq_lens, sm_scale, out=None, lse=None, workspace=None,
           nsplit: int = 0, wait_timeout_ns: int = 0, debug_flags: int = 0, stream=None, out_dtype=None):
    """smla_decode_ex: returns (out [B,64,512], lse fp32 [B,64]).  out is fp32, or bf16 when
    ``out_dtype`` is torch.bfloat16 or a bf16 ``out`` tensor is given."""
    B, H, D = q.shape
    topk = topk_idx.shape[1]
    if out_dtype is None:
        out_dtype = out.dtype if out is not None else torch.float32
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise SmlaError("out must be float32 or bfloat16")
    if out is None:
        out = torch.empty((B, H, D), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(B, topk, nsplit, q.device)
    opts = _Options(nsplit, 1 if out_dtype == torch.bfloat16 else 0, wait_timeout_ns, debug_flags, 0)
    rc = library().smla_decode_ex(
        _dev(q, torch.bfloat16, "q"), _dev(kv_cache, torch.uint8, "kv_cache"),
        _dev(block_table, torch.int32, "block_table"), _dev(topk_idx, torch.int32, "topk_idx"),
        _dev(seq_lens, torch.int32, "seq_lens"), float(sm_scale), _dev(out, out_dtype, "out"),
        _dev(lse, torch.float32, "lse"), B, H, topk, block_table.shape[1], kv_cache.shape[0],
        _dev(workspace, torch.uint8, "workspace"), workspace.numel(), ctypes.byref(opts), _stream(stream))
    _check(rc, "smla_decode")
    return out, lse


def combine(part_o, part_lse, out=None, lse=None, stream=None):
    """smla_combine: merge [B,H,nsplit,512] partials by their log-sum-exp."""
    B, H, ns, D = part_o.shape
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=part_o.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=part_o.device)
    rc = library().smla_combine(_dev(part_o, torch.float32, "part_o"), _dev(part_lse, torch.float32, "part_lse"), ns,
                                _dev(out, torch.float32, "out"), _dev(lse, torch.float32, "lse"), B, H,
                                _stream(stream))
    _check(rc, "smla_combine")
    return out, lse


def read_error(workspace, stream=None) -> int:
    """smla_read_error: synchronise, return and clear the device error word."""
    v = ctypes.c_uint32(0)
    _check(library().smla_read_error(_dev(workspace, torch.uint8, "workspace"), _stream(stream), ctypes.byref(v)),
           "smla_read_error")
    return int(v.value)


def debug_gather(kv_cache, block_table, topk_idx, seq_lens, workspace=None, stream=None):
    """smla_debug_gather: (latents fp32 [B,topk,512], page_slot int32 [B,topk,2])."""
    B, topk = topk_idx.shape
    lat = torch.empty((B, topk, DIM), dtype=torch.float32, device=kv_cache.device)
    ps = torch.empty((B, topk, 2), dtype=torch.int32, device=kv_cache.device)
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=kv_cache.device)
    rc = library().smla_debug_gather(
        _dev(kv_cache, torch.uint8, "kv_cache"), _dev(block_table, torch.int32, "block_table"),
        _dev(topk_idx, torch.int32, "topk_idx"), _dev(seq_lens, torch.int32, "seq_lens"), B, topk,
        block_table.shape[1], kv_cache.shape[0], _dev(lat, torch.float32, "latents"),
        _dev(ps, torch.int32, "page_slot"), _dev(workspace, torch.uint8, "workspace"), workspace.numel(),
        _stream(stream))
    _check(rc, "smla_debug_gather")
    return lat, ps


def write_kv(latents, req, pos, block_table, kv_cache, err=None, stream=None) -> None:
    """smla_write_kv: quantise latents [n,512] (fp32 or bf16) into ``kv_cache`` at position
    pos[i] of request req[i]; ``err`` (a uint32 CUDA tensor of one element, or None)
    receives SMLA_FLAG_BAD_PAGE when a token's destination is out of range."""
    if latents.dtype not in (torch.float32, torch.bfloat16):
        raise SmlaError("latents must be float32 or bfloat16")
    n = latents.shape[0] if latents.dim() == 2 else 0
    if latents.dim() != 2 or latents.shape[1] != DIM:
        raise SmlaError("latents must be [n, 512]")
    if req.shape != (n,) or pos.shape != (n,):
        raise SmlaError("req and pos must be [n]")
    ep = None
    if err is not None:
        if err.dtype not in (torch.int32, torch.uint32) or err.numel() < 1 or not err.is_cuda:
            raise SmlaError("err must be a CUDA int32/uint32 tensor")
        ep = err.data_ptr()
    rc = library().smla_write_kv(
        _dev(latents, latents.dtype, "latents"), 1 if latents.dtype == torch.bfloat16 else 0, n,
        _dev(req, torch.int32, "req"), _dev(pos, torch.int32, "pos"), _dev(block_table, torch.int32, "block_table"),
        block_table.shape[0], block_table.shape[1], kv_cache.shape[0], _dev(kv_cache, torch.uint8, "kv_cache"), ep,
        _stream(stream))
    _check(rc, "smla_write_kv")
