"""Sparse MLA decode over an FP8 paged latent cache, for B200 (sm_100a).

The compute lives in ``libsmla.so`` (CUDA, C ABI in ``include/smla.h``); this
package is its Python binding.  The binding only marshals arguments -- torch
tensors in device memory, the current CUDA stream -- into the C calls; every
step of the decode runs in the library's kernels.  Importing works without a
GPU; calling needs the built library and an sm_100 device, and fails loudly
otherwise (there is no fallback path).
"""
from .binding import (  # noqa: F401
    SMLA_FLAG_BAD_PAGE,
    SMLA_FLAG_SMEM,
    SMLA_FLAG_TIMEOUT,
    SMLA_DEBUG_SKIP_FIRST_COMMIT,
    SmlaError,
    combine,
    debug_gather,
    decode,
    library,
    num_splits,
    read_error,
    version,
    workspace_bytes,
    write_kv,
)
