"""fp64 CPU oracle for the sparse MLA decode step (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never touches it.  The arithmetic lives in ``smla_oracle.c``
(plain C, double precision, OpenMP over requests); this module only builds that
file with gcc and marshals numpy arrays through ctypes.

Every function here states what it computes and which passage of the source
pages it follows; the pins that tie it to something other than itself are in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "smla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

DIM = 512
NOPE = 448
ROPE = 64
PAGE_TOKENS = 256
PAGE_BYTES = 256 * (576 + 8)


def build(force: bool = False) -> str:
    """Compile ``smla_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.orc_e4m3.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3.restype = ctypes.c_double
    lib.orc_ue8m0.argtypes = [ctypes.c_uint8]
    lib.orc_ue8m0.restype = ctypes.c_double
    lib.orc_bf16.argtypes = [ctypes.c_uint16]
    lib.orc_bf16.restype = ctypes.c_double
    lib.orc_num_threads.restype = ctypes.c_int
    lib.orc_gather.argtypes = [P, ctypes.c_int64, P, ctypes.c_int, P, P, ctypes.c_int, ctypes.c_int, P, P]
    lib.orc_gather.restype = ctypes.c_int
    lib.orc_decode.argtypes = [P, P, ctypes.c_int64, P, ctypes.c_int, P, P, ctypes.c_double,
                               ctypes.c_int, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, P]
    lib.orc_decode.restype = ctypes.c_int
    lib.orc_combine.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
    lib.orc_combine.restype = ctypes.c_int
    lib.orc_e4m3_encode.argtypes = [ctypes.c_double]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_bf16_encode.argtypes = [ctypes.c_float]
    lib.orc_bf16_encode.restype = ctypes.c_uint16
    lib.orc_scale_exponent.argtypes = [P]
    lib.orc_scale_exponent.restype = ctypes.c_int
    lib.orc_quantize_token.argtypes = [P, P, P]
    lib.orc_quantize_token.restype = None
    lib.orc_write_kv.argtypes = [P, ctypes.c_int, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int64, P]
    lib.orc_write_kv.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB_PATH)
    return _lib


def load_variant(path: str):
    """Bind another build of ``smla_oracle.c`` (used by the mutation tests)."""
    return _bind(path)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads(lib=None) -> int:
    """OpenMP threads the oracle uses (its ``cores`` figure)."""
    return int((lib or _load()).orc_num_threads())


def e4m3(byte: int, lib=None) -> float:
    """OCP e4m3fn value of one byte (bias 7, subnormals, 0x7F/0xFF NaN)."""
    return float((lib or _load()).orc_e4m3(int(byte) & 0xFF))


def ue8m0(byte: int, lib=None) -> float:
    """UE8M0 scale 2^(byte-127); 0xFF is NaN."""
    return float((lib or _load()).orc_ue8m0(int(byte) & 0xFF))


def bf16(bits: int, lib=None) -> float:
    """Value of a bf16 bit pattern."""
    return float((lib or _load()).orc_bf16(int(bits) & 0xFFFF))


def gather(cache, block_table, topk_idx, seq_lens, lib=None):
    """Index translation and dequantisation of every topk slot.

    Follows the cache layout of "The Validation Gate" ("The Test Design") and the
    page indexing of "The Validation Moment".  Returns ``(latents, page_slot)``:
    fp64 [B,topk,512] (zeros for invalid slots) and int32 [B,topk,2]
    (``-1,-1`` for invalid slots).
    """
    cache = _c(cache, np.uint8)
    bt = _c(block_table, np.int32)
    idx = _c(topk_idx, np.int32)
    sl = _c(seq_lens, np.int32)
    B, topk = idx.shape
    lat = np.empty((B, topk, DIM), np.float64)
    ps = np.empty((B, topk, 2), np.int32)
    rc = (lib or _load()).orc_gather(_ptr(cache), cache.shape[0], _ptr(bt), bt.shape[1], _ptr(idx), _ptr(sl),
                            B, topk, _ptr(lat), _ptr(ps))
    if rc != 0:
        raise ValueError("orc_gather rejected its arguments")
    return lat, ps


def decode(q_bits, cache, block_table, topk_idx, seq_lens, sm_scale, rows=None, lib=None):
    """The sparse MLA decode step in fp64.

    ``q_bits``: uint16 bf16 bits [B,H,512].  Follows "The Turning Point" (Step 1
    and Output Knowledge item 2: dequantize -> concat -> matmul -> softmax ->
    weighted sum over the gathered latents, one shared KV head for all heads).
    Returns ``(out, lse)``: fp64 [B,H,512] and [B,H], or, when ``rows`` (an
    int array of (b,h) pairs) is given, [len(rows),512] and [len(rows)].
    """
    q = _c(q_bits, np.uint16)
    cache = _c(cache, np.uint8)
    bt = _c(block_table, np.int32)
    idx = _c(topk_idx, np.int32)
    sl = _c(seq_lens, np.int32)
    B, H, D = q.shape
    assert D == DIM
    topk = idx.shape[1]
    if rows is None:
        out = np.empty((B, H, DIM), np.float64)
        lse = np.empty((B, H), np.float64)
        rws, nrows = None, 0
    else:
        rws = _c(rows, np.int32).reshape(-1, 2)
        nrows = rws.shape[0]
        out = np.empty((nrows, DIM), np.float64)
        lse = np.empty((nrows,), np.float64)
    rc = (lib or _load()).orc_decode(_ptr(q), _ptr(cache), cache.shape[0], _ptr(bt), bt.shape[1], _ptr(idx),
                            _ptr(sl), float(sm_scale), B, H, topk, _ptr(rws), nrows, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("orc_decode rejected its arguments")
    return out, lse


def combine(part_o, part_lse, lib=None):
    """Split-K LSE merge ("The Turning Point", Step 5).

    ``part_o``: [B,H,nsplit,512] normalised partial outputs; ``part_lse``:
    [B,H,nsplit].  Returns ``(out, lse)`` with L = ln sum exp(L_s) and
    O = sum exp(L_s - L) O_s; -inf splits weigh 0.
    """
    po = _c(part_o, np.float64)
    pl = _c(part_lse, np.float64)
    B, H, ns, D = po.shape
    assert D == DIM and pl.shape == (B, H, ns)
    out = np.empty((B, H, DIM), np.float64)
    lse = np.empty((B, H), np.float64)
    rc = (lib or _load()).orc_combine(_ptr(po), _ptr(pl), B, H, ns, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("orc_combine rejected its arguments")
    return out, lse


def e4m3_encode(x: float, lib=None) -> int:
    """e4m3 (fn) code nearest to x (ties to the even code); |x| >= 448 saturates; NaN -> 0x7F."""
    return int((lib or _load()).orc_e4m3_encode(float(x)))


def bf16_encode(x: float, lib=None) -> int:
    """bf16 bits of a binary32 value, round to nearest even; NaN -> 0x7FC0."""
    return int((lib or _load()).orc_bf16_encode(float(np.float32(x))))


def scale_exponent(group, lib=None) -> int:
    """Scale exponent e of one 64-value nope group: the smallest e with max|x| <= 448 * 2^e,
    clamped to [-127, 127] (-127 when all zero, 127 when a value is not finite)."""
    g = _c(group, np.float32)
    assert g.shape == (64,)
    return int((lib or _load()).orc_scale_exponent(_ptr(g)))


def quantize_token(latent, lib=None):
    """One 512-d fp32 latent -> (576-byte row, 8-byte scale row): the cache format of "The
    Validation Gate" ("The Test Design"), per 64-dim UE8M0 scale and e4m3 nope, bf16 rope."""
    x = _c(latent, np.float32)
    assert x.shape == (DIM,)
    row = np.zeros(576, np.uint8)
    sc = np.zeros(8, np.uint8)
    (lib or _load()).orc_quantize_token(_ptr(x), _ptr(row), _ptr(sc))
    return row, sc


def write_kv(latents, req, pos, block_table, cache, lib=None) -> int:
    """Quantise latents [n,512] and store each at position pos[i] of request req[i]
    (page = block_table[req][pos // 256], slot = pos % 256), in place in ``cache``
    [pages, PAGE_BYTES] uint8.  Out-of-range destinations are skipped; returns their count."""
    x = _c(latents, np.float32).reshape(-1, DIM)
    r = _c(req, np.int32)
    p = _c(pos, np.int32)
    bt = _c(block_table, np.int32)
    assert cache.dtype == np.uint8 and cache.flags["C_CONTIGUOUS"] and cache.shape[-1] == PAGE_BYTES
    n = x.shape[0]
    assert r.shape == (n,) and p.shape == (n,)
    return int((lib or _load()).orc_write_kv(_ptr(x), n, _ptr(r), _ptr(p), _ptr(bt), bt.shape[0], bt.shape[1],
                                             cache.shape[0], _ptr(cache)))
