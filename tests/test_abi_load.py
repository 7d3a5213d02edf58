"""The C-ABI library loads and exports every symbol include/dec.h declares (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dec.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dec_[a-z0-9_]+)\s*\(", src)))


def test_header_declarations_match_binding_list():
    import transformer_decoder_kv_b200 as pkg
    assert _declared() == sorted(pkg.EXPORTS)


def test_library_exports_every_declared_symbol():
    from transformer_decoder_kv_b200 import binding
    if not os.path.exists(binding.LIB_PATH):
        from transformer_decoder_kv_b200 import build
        build.build()
    lib = ctypes.CDLL(binding.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_sets_signatures_without_gpu():
    from transformer_decoder_kv_b200 import binding
    lib = binding.load_library()
    assert lib.dec_last_error(None) == b""
    # a create call with a bad config is rejected on the host before touching the GPU
    cfg = binding.DecConfig(7, 1, 128, 2, 64, 256, 10, 10, 0, 0, 1e-5, 0.0, 1, 8, 0, 0, 0, 0)
    w = binding.DecWeights()
    h = ctypes.c_void_p()
    st = lib.dec_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h))
    assert st == binding.DEC_EINVAL
    assert b"family" in lib.dec_last_error(None)
    assert not h.value
