"""B200 (sm_100a) WAITS prefill KV-eviction path: score -> select -> compact.

The work runs in ``libwaits.so`` (hand-written CUDA kernels behind a C ABI,
``include/waits.h``); :mod:`.api` marshals torch tensors into it.  Importing
this package does not load the library; the first call does, and raises if
it is missing (there is no fallback).
"""

from .api import (  # noqa: F401
    Compressor, HostCompressor, compact, compress, score, score_static, select,
    select_compact,
    workspace_bytes, make_shape)
from ._lib import WaitsError, WaitsLibraryError  # noqa: F401
