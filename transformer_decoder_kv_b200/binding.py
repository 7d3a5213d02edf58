"""ctypes binding of the C ABI in include/dec.h (argument marshalling only).

Every step of the decoder runs in the CUDA library libdec.so built from csrc/.
There is no CPU path: if the library is missing this module raises on import.
Device buffers are passed as raw pointers (e.g. torch.Tensor.data_ptr()), streams
as cudaStream_t handles (e.g. torch.cuda.current_stream().cuda_stream).
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdec.so")

DEC_OK, DEC_EINVAL, DEC_ERANGE, DEC_EOVERFLOW, DEC_ESTATE, DEC_ENOMEM, DEC_ECUDA, DEC_ETIMEOUT = range(8)
STATUS_NAMES = ["DEC_OK", "DEC_EINVAL", "DEC_ERANGE", "DEC_EOVERFLOW", "DEC_ESTATE", "DEC_ENOMEM",
                "DEC_ECUDA", "DEC_ETIMEOUT"]
FAMILY = {"whisper": 0, "qwen2": 1}
HEAD = {"exact": 0, "int8": 1}
PROJ = {"f32": 0, "w8a8": 1, "w8a32": 2}

# Every symbol include/dec.h declares.
EXPORTS = ["dec_create", "dec_destroy", "dec_last_error", "dec_prefill", "dec_kv_append", "dec_step",
           "dec_step_host", "dec_slot_len", "dec_kv_read", "dec_hidden", "dec_set_layer_trace", "dec_sync",
           "dec_reset", "dec_set_wait_limit", "dec_debug_inject", "dec_debug_fail_alloc", "dec_step_kernels",
           "dec_next_tokens", "dec_get_config", "dec_generate", "dec_set_prefill_chunk",
           "dec_set_phase_timing", "dec_phase_times", "dec_release_slot", "dec_kv_pages_free",
           "dec_attention_workspace_size", "dec_attention", "dec_attention_plan", "dec_attention_noalloc",
           "dec_i8_dot"]
I8_PATH = {"dp4a": 0, "tcgen05": 1}
DEC_INJECT_DROP_ATTN_COPY = 1
PHASE_NAMES = {1: "embed", 2: "qkv", 3: "self_attn", 4: "o", 5: "cross_q", 6: "cross_attn", 7: "cross_o",
               8: "ffn_up", 9: "ffn_down", 10: "head"}


class DecError(RuntimeError):
    def __init__(self, status: int, msg: str):
        self.status = status
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{name}: {msg}")


class DecConfig(C.Structure):
    _fields_ = [("family", C.c_int32), ("n_layers", C.c_int32), ("d_model", C.c_int32),
                ("n_heads", C.c_int32), ("head_dim", C.c_int32), ("d_ff", C.c_int32),
                ("vocab", C.c_int32), ("max_pos", C.c_int32), ("enc_len", C.c_int32),
                ("proj_fmt", C.c_int32), ("norm_eps", C.c_float), ("rope_theta", C.c_float),
                ("max_slots", C.c_int32), ("max_cache_len", C.c_int32), ("head_fmt", C.c_int32),
                ("n_kv_heads", C.c_int32), ("kv_page_rows", C.c_int32), ("kv_pages", C.c_int32)]


class DecProj(C.Structure):
    _fields_ = [("w", C.c_void_p), ("scale", C.c_void_p), ("bias", C.c_void_p)]


class DecLayerWeights(C.Structure):
    _fields_ = [("norm1_w", C.c_void_p), ("norm1_b", C.c_void_p),
                ("q", DecProj), ("k", DecProj), ("v", DecProj), ("o", DecProj),
                ("norm2_w", C.c_void_p), ("norm2_b", C.c_void_p),
                ("xq", DecProj), ("xk", DecProj), ("xv", DecProj), ("xo", DecProj),
                ("norm3_w", C.c_void_p), ("norm3_b", C.c_void_p),
                ("fc1", DecProj), ("fc2", DecProj),
                ("gate", DecProj), ("up", DecProj), ("down", DecProj)]


class DecRequest(C.Structure):
    _fields_ = [("prompt", C.POINTER(C.c_int32)), ("n_prompt", C.c_int32), ("max_new", C.c_int32),
                ("eos", C.c_int32), ("enc_hidden", C.c_void_p)]


class DecWeights(C.Structure):
    _fields_ = [("tok_emb", C.c_void_p), ("pos_emb", C.c_void_p), ("final_w", C.c_void_p),
                ("final_b", C.c_void_p), ("layers", C.POINTER(DecLayerWeights))]


def load_library(path: str = LIB_PATH) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"CUDA decoder library not built: {path} is missing "
                          "(run transformer_decoder_kv_b200.build.build())")
    lib = C.CDLL(path)
    vp, i32, pi32 = C.c_void_p, C.c_int32, C.POINTER(C.c_int32)
    sig = {
        "dec_create": (C.c_int, [C.POINTER(DecConfig), C.POINTER(DecWeights), C.POINTER(vp)]),
        "dec_destroy": (C.c_int, [vp]),
        "dec_last_error": (C.c_char_p, [vp]),
        "dec_prefill": (C.c_int, [vp, i32, pi32, i32, vp, vp, vp]),
        "dec_kv_append": (C.c_int, [vp, i32, i32, i32, vp, vp, vp]),
        "dec_step": (C.c_int, [vp, i32, pi32, pi32, pi32, pi32, vp, vp, vp]),
        "dec_step_host": (C.c_int, [vp, i32, pi32, pi32, pi32, pi32, vp, vp, vp]),
        "dec_slot_len": (C.c_int, [vp, i32, pi32]),
        "dec_kv_read": (C.c_int, [vp, i32, i32, i32, i32, vp, vp, vp]),
        "dec_hidden": (C.c_int, [vp, vp, i32, vp]),
        "dec_set_layer_trace": (C.c_int, [vp, vp]),
        "dec_sync": (C.c_int, [vp, vp]),
        "dec_reset": (C.c_int, [vp]),
        "dec_release_slot": (C.c_int, [vp, i32]),
        "dec_kv_pages_free": (C.c_int, [vp, pi32]),
        "dec_set_prefill_chunk": (C.c_int, [vp, i32]),
        "dec_set_phase_timing": (C.c_int, [vp, i32]),
        "dec_phase_times": (C.c_int, [vp, i32, C.POINTER(C.c_float), pi32, pi32, pi32]),
        "dec_next_tokens": (C.c_int, [vp, i32, pi32, pi32, vp]),
        "dec_get_config": (C.c_int, [vp, C.POINTER(DecConfig)]),
        "dec_generate": (C.c_int, [vp, C.POINTER(DecRequest), i32, i32, pi32, i32, pi32, vp]),
        "dec_set_wait_limit": (C.c_int, [vp, C.c_uint64]),
        "dec_debug_inject": (C.c_int, [vp, i32, i32]),
        "dec_debug_fail_alloc": (None, [i32]),
        "dec_step_kernels": (C.c_int, [vp, pi32]),
        "dec_attention_workspace_size": (C.c_size_t, [i32, i32, i32]),
        "dec_attention": (C.c_int, [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, C.c_size_t, vp]),
        "dec_attention_plan": (C.c_int, [vp, i32, pi32]),
        "dec_attention_noalloc": (C.c_int, [vp, vp, vp, vp, i32, i32, i32, vp, vp]),
        "dec_i8_dot": (C.c_int, [vp, vp, i32, i32, i32, i32, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib: Optional[C.CDLL] = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _i32arr(values) -> Optional[C.Array]:
    if values is None:
        return None
    a = np.ascontiguousarray(np.asarray(values, dtype=np.int32))
    return (C.c_int32 * len(a))(*a.tolist())


def _ptr(a) -> Optional[int]:
    """Pointer of a numpy array (host) or a tensor-like with data_ptr() (device); None stays None."""
    if a is None:
        return None
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    return a.ctypes.data


class Decoder:
    """One handle of the CUDA decoder (dec_create ... dec_destroy)."""

    def __init__(self, cfg, weights: dict, max_slots: int, max_cache_len: int, head: str = "exact",
                 kv_page_rows: int = 0, kv_pages: int = 0):
        self._lib = lib()
        c = DecConfig(FAMILY[cfg.family], cfg.n_layers, cfg.d_model, cfg.n_heads, cfg.head_dim,
                      cfg.d_ff, cfg.vocab, cfg.max_pos, cfg.enc_len, PROJ[cfg.proj_fmt],
                      float(cfg.norm_eps), float(cfg.rope_theta), max_slots, max_cache_len, HEAD[head],
                      int(getattr(cfg, "n_kv_heads", 0)), kv_page_rows, kv_pages)
        self.cfg = cfg
        self.max_slots = max_slots
        self.max_cache_len = max_cache_len
        keep = []

        def arr(x, dtype):
            if x is None:
                return None
            a = np.ascontiguousarray(x, dtype=dtype)
            keep.append(a)
            return a.ctypes.data

        wdt = np.float32 if cfg.proj_fmt == "f32" else np.int8

        def proj(p):
            if p is None:
                return DecProj(None, None, None)
            return DecProj(arr(p["w"], wdt), arr(p["s"], np.float32), arr(p["b"], np.float32))

        layers = (DecLayerWeights * cfg.n_layers)()
        for i, L in enumerate(weights["layers"]):
            lw = layers[i]
            lw.norm1_w = arr(L.get("norm1_w"), np.float32)
            lw.norm1_b = arr(L.get("norm1_b"), np.float32)
            lw.norm2_w = arr(L.get("norm2_w"), np.float32)
            lw.norm2_b = arr(L.get("norm2_b"), np.float32)
            lw.norm3_w = arr(L.get("norm3_w"), np.float32)
            lw.norm3_b = arr(L.get("norm3_b"), np.float32)
            for name in ("q", "k", "v", "o", "xq", "xk", "xv", "xo", "fc1", "fc2", "gate", "up", "down"):
                setattr(lw, name, proj(L.get(name)))
        w = DecWeights(arr(weights["tok_emb"], np.float32), arr(weights.get("pos_emb"), np.float32),
                       arr(weights["final_w"], np.float32), arr(weights.get("final_b"), np.float32),
                       layers)
        h = C.c_void_p()
        st = self._lib.dec_create(C.byref(c), C.byref(w), C.byref(h))
        del keep
        if st != DEC_OK:
            raise DecError(st, self._lib.dec_last_error(None).decode())
        self._h = h

    # -- helpers --
    def _check(self, st: int):
        if st != DEC_OK:
            raise DecError(st, self._lib.dec_last_error(self._h).decode())

    def close(self):
        if getattr(self, "_h", None):
            self._lib.dec_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- the C ABI --
    def prefill(self, slot: int, tokens: Sequence[int], enc_hidden=None, last_logits=None, stream: int = 0):
        toks = _i32arr(tokens) if len(tokens) else None
        self._check(self._lib.dec_prefill(self._h, slot, toks, len(tokens), _ptr(enc_hidden),
                                          _ptr(last_logits), stream))

    def kv_append(self, slot: int, start: int, n_rows: int, k, v, stream: int = 0):
        self._check(self._lib.dec_kv_append(self._h, slot, start, n_rows, _ptr(k), _ptr(v), stream))

    def step(self, batch: int, slots, tokens, positions, cache_lens, logits=None, argmax=None,
             stream: int = 0):
        self._check(self._lib.dec_step(self._h, batch, _i32arr(slots), _i32arr(tokens),
                                       _i32arr(positions), _i32arr(cache_lens), _ptr(logits),
                                       _ptr(argmax), stream))

    def step_host(self, batch: int, slots, tokens, positions, cache_lens, logits_host=None,
                  argmax_host=None, stream: int = 0):
        self._check(self._lib.dec_step_host(self._h, batch, _i32arr(slots), _i32arr(tokens),
                                            _i32arr(positions), _i32arr(cache_lens),
                                            _ptr(logits_host), _ptr(argmax_host), stream))

    def slot_len(self, slot: int) -> int:
        n = C.c_int32()
        self._check(self._lib.dec_slot_len(self._h, slot, C.byref(n)))
        return n.value

    def kv_read(self, slot: int, layer: int, start: int, n: int, k_out, v_out, stream: int = 0):
        self._check(self._lib.dec_kv_read(self._h, slot, layer, start, n, _ptr(k_out), _ptr(v_out), stream))

    def hidden(self, out, batch: int, stream: int = 0):
        self._check(self._lib.dec_hidden(self._h, _ptr(out), batch, stream))

    def set_layer_trace(self, buf):
        """Device buffer f32 [n_layers, batch, d_model] for the residual leaving each layer
        of every later step (None turns tracing off)."""
        self._check(self._lib.dec_set_layer_trace(self._h, _ptr(buf)))

    def sync(self, stream: int = 0):
        self._check(self._lib.dec_sync(self._h, stream))

    def attention_plan(self, cross: bool = False) -> int:
        """Tiles per split of the step's self- (or cross-) attention launches."""
        n = C.c_int32(0)
        self._check(self._lib.dec_attention_plan(self._h, 1 if cross else 0, C.byref(n)))
        return int(n.value)

    def next_tokens(self, slots, stream: int = 0):
        """Each slot's greedy continuation token (host list)."""
        out = (C.c_int32 * len(slots))()
        self._check(self._lib.dec_next_tokens(self._h, len(slots), _i32arr(slots), out, stream))
        return list(out)

    def generate(self, requests, max_active: int, stream: int = 0):
        """Greedy generation with continuous batching. requests: list of dicts with
        'prompt' (token ids), 'max_new', optional 'eos' (-1) and 'enc_hidden' (device
        tensor, whisper). Returns one list of token ids per request."""
        n = len(requests)
        keep = []
        arr = (DecRequest * max(1, n))()
        stride = max([int(r["max_new"]) for r in requests] + [1])
        for i, r in enumerate(requests):
            p = _i32arr(r["prompt"])
            keep.append(p)
            arr[i] = DecRequest(C.cast(p, C.POINTER(C.c_int32)), len(r["prompt"]), int(r["max_new"]),
                                int(r.get("eos", -1)), _ptr(r.get("enc_hidden")))
        toks = (C.c_int32 * (max(1, n) * stride))()
        lens = (C.c_int32 * max(1, n))()
        self._check(self._lib.dec_generate(self._h, arr, n, max_active, toks, stride, lens, stream))
        return [list(toks[i * stride: i * stride + lens[i]]) for i in range(n)]

    def set_phase_timing(self, enabled: bool):
        self._check(self._lib.dec_set_phase_timing(self._h, 1 if enabled else 0))

    def phase_times(self):
        """[(layer, phase name, ms)] of the most recent phase-timed step."""
        cap = 4096
        ms = (C.c_float * cap)()
        layer = (C.c_int32 * cap)()
        kind = (C.c_int32 * cap)()
        n = C.c_int32(0)
        self._check(self._lib.dec_phase_times(self._h, cap, ms, layer, kind, C.byref(n)))
        return [(int(layer[i]), PHASE_NAMES.get(int(kind[i]), str(kind[i])), float(ms[i]))
                for i in range(min(n.value, cap))]

    def set_prefill_chunk(self, rows: int):
        self._check(self._lib.dec_set_prefill_chunk(self._h, rows))

    def release_slot(self, slot: int):
        self._check(self._lib.dec_release_slot(self._h, slot))

    def kv_pages_free(self) -> int:
        n = C.c_int32(0)
        self._check(self._lib.dec_kv_pages_free(self._h, C.byref(n)))
        return int(n.value)

    def reset(self):
        self._check(self._lib.dec_reset(self._h))

    def set_wait_limit(self, ns: int):
        self._check(self._lib.dec_set_wait_limit(self._h, int(ns)))

    def debug_inject(self, what: int, value: int):
        self._check(self._lib.dec_debug_inject(self._h, what, value))

    def step_kernels(self) -> int:
        """Kernels launched by one step of the most recent step call (-1: not captured)."""
        n = C.c_int32(0)
        self._check(self._lib.dec_step_kernels(self._h, C.byref(n)))
        return int(n.value)


def debug_fail_alloc(nth: int):
    """The nth allocation of the next Decoder created on this thread fails (0: off)."""
    lib().dec_debug_fail_alloc(int(nth))


def _raise_thread_error(st: int):
    if st != DEC_OK:
        raise DecError(st, lib().dec_last_error(None).decode())


def attention(q, k, v, lens, batch: int, n_heads: int, ld: int, out, workspace, workspace_bytes: int,
              stream: int = 0, tiles_per_split: int = 0):
    _raise_thread_error(lib().dec_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(lens), batch, n_heads, ld,
                                            tiles_per_split, _ptr(out), _ptr(workspace), workspace_bytes,
                                            stream))


def attention_noalloc(q, k, v, lens, batch: int, n_heads: int, ld: int, out, stream: int = 0):
    """dec_attention without a caller workspace: the library's fixed scratch array is used."""
    _raise_thread_error(lib().dec_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(lens), batch, n_heads, ld,
                                                    _ptr(out), stream))


def attention_workspace_size(batch: int, n_heads: int, ld: int) -> int:
    return int(lib().dec_attention_workspace_size(batch, n_heads, ld))


def i8_dot(xq, wq, m: int, n: int, kdim: int, acc, stream: int = 0, path: str = "dp4a"):
    _raise_thread_error(lib().dec_i8_dot(_ptr(xq), _ptr(wq), m, n, kdim, I8_PATH[path], _ptr(acc), stream))
