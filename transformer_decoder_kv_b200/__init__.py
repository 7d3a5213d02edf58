"""Batched single-token decoder step for B200 (sm_100a): C ABI library + thin binding.

The decode step runs entirely in libdec.so (hand-written CUDA kernels); this
package only builds it (build.py) and marshals arguments (binding.py).
"""
from .binding import (  # noqa: F401
    Decoder, DecError, attention, debug_fail_alloc, attention_noalloc, attention_workspace_size, i8_dot, lib,
    load_library, EXPORTS, LIB_PATH,
)
