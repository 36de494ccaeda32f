"""The C ABI library loads and exports every symbol include/smla.h declares (CPU only)."""
import ctypes
import os
import re

from sparse_mla_decode_fp8_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "smla.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(smla_\w+)\s*\(", text, re.M)))


def test_header_declares_entry_points():
    syms = declared_symbols()
    for s in ["smla_decode", "smla_decode_ex", "smla_combine", "smla_workspace_bytes", "smla_read_error",
              "smla_debug_gather", "smla_num_splits", "smla_version"]:
        assert s in syms, s


def test_library_builds_loads_and_exports_all():
    lib_path = build.build()
    lib = ctypes.CDLL(lib_path)
    for s in declared_symbols():
        assert hasattr(lib, s), f"{s} not exported"
    lib.smla_version.restype = ctypes.c_char_p
    assert b"sm_100a" in lib.smla_version()


def test_no_gpu_calls_fail_cleanly():
    # without a device the size queries report an error instead of crashing
    import torch

    if torch.cuda.is_available():
        return
    lib = ctypes.CDLL(build.build())
    lib.smla_num_splits.argtypes = [ctypes.c_int] * 3
    assert lib.smla_num_splits(64, 64, 512) < 0
    lib.smla_workspace_bytes.restype = ctypes.c_size_t
    lib.smla_workspace_bytes.argtypes = [ctypes.c_int] * 3
    assert lib.smla_workspace_bytes(64, 64, 512) == 0
