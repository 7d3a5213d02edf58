"""Seeded synthetic inputs for the batched single-token decoder step.

This module is shared by the CPU oracle tests, the GPU parity tests and the
benchmark. It only DRAWS inputs: model shapes, random weights with the
distributions below, encoder hidden states, token ids, cache lengths and
seeded K/V rows. It holds none of the decode step's arithmetic.

The one transformation it applies is the offline per-row symmetric int8
quantisation of projection weights for the int8 model formats. That step
stands in for the pre-quantised checkpoint records the decoders load
(franken_ocr native_engine/decoder_qwen2.rs, `GotLayerW` / `quant_oc_loaded`:
"int8 GEMMs read verbatim from the .focrq QInt8PerChan records"; lattice-
inference forward/cpu_q8.rs module doc: "per-row symmetric INT8 quantized").
It happens before any decode step and is not part of the step.

Distributions (all seeded, every tensor from its own child generator so any
tensor can be regenerated alone):
  * projection weights, token embedding, learned position table: N(0, 0.02)
  * LayerNorm gamma and RMSNorm weight: 1 + N(0, 0.02); LayerNorm beta: N(0, 0.01)
  * biases: N(0, 0.01)
  * encoder hidden states: N(0, 1), one [enc_len, d] block per stream
  * token ids: uniform over [0, vocab)
  * seeded K/V cache rows: N(0, 1)
Normals are drawn with numpy's Generator.standard_normal in float32.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "ModelConfig", "Workload", "MODELS", "WORKLOADS", "make_weights",
    "quantize_weight_rows_offline", "encoder_hidden", "token_ids", "cache_lens",
    "seed_kv", "workload",
]

# Tags that separate the random streams of different kinds of input.
_TAG_WEIGHT = 11
_TAG_ENC = 23
_TAG_TOK = 37
_TAG_LENS = 41
_TAG_KV = 53

PROJ_F32 = "f32"
PROJ_W8A8 = "w8a8"     # int8 weights, int8 activations quantised per row, int32 accumulate
PROJ_W8A32 = "w8a32"   # int8 weights dequantised per row, f32 activations


@dataclass(frozen=True)
class ModelConfig:
    """Shape of one pre-norm decoder.

    family "whisper": LayerNorm (with bias), learned positions, self-attention,
    cross-attention over encoder K/V, GELU(tanh) FFN, every projection biased.
    family "qwen2": RMSNorm, NEOX RoPE, SwiGLU MLP, q/k/v bias only.
    Both tie the LM head to the token embedding.
    """
    name: str
    family: str
    n_layers: int
    d_model: int
    n_heads: int
    head_dim: int
    d_ff: int
    vocab: int
    max_pos: int          # learned position rows (whisper) / RoPE position bound (qwen2)
    enc_len: int          # encoder rows for cross-attention (whisper), 0 otherwise
    proj_fmt: str         # PROJ_F32 | PROJ_W8A8 | PROJ_W8A32
    norm_eps: float
    rope_theta: float = 0.0
    n_kv_heads: int = 0   # grouped-query attention: K/V heads (0: one per query head)

    @property
    def is_whisper(self) -> bool:
        return self.family == "whisper"

    @property
    def kv_heads(self) -> int:
        return self.n_kv_heads or self.n_heads

    @property
    def kv_dim(self) -> int:
        return self.kv_heads * self.head_dim

    @property
    def qkv_bias(self) -> bool:
        return True

    @property
    def o_bias(self) -> bool:
        return self.is_whisper

    @property
    def mlp_bias(self) -> bool:
        return self.is_whisper


@dataclass(frozen=True)
class Workload:
    """One decode workload: a model, a batch of streams and how their caches start.

    cache_init "prefill": each stream's cache is built by prefilling `lens[b]`
    seeded tokens at positions 0..lens[b]-1 (then decoding continues from there).
    cache_init "kv_seed": each stream's cache is filled with `lens[b]` rows of
    N(0,1) K and V per layer, and positions equal cache lengths.
    """
    name: str
    model: ModelConfig
    batch: int
    max_cache_len: int
    cache_init: str
    lens_lo: int
    lens_hi: int          # inclusive
    steps: int
    retire_at: Optional[int] = None   # a stream stops once its length reaches this


def _m(**kw) -> ModelConfig:
    return ModelConfig(**kw)


MODELS: Dict[str, ModelConfig] = {
    # Whisper-tiny-shaped single decoder block (one layer + final LN + tied head).
    "whisper_tiny_block": _m(name="whisper_tiny_block", family="whisper", n_layers=1, d_model=384,
                             n_heads=6, head_dim=64, d_ff=1536, vocab=51865, max_pos=448,
                             enc_len=1500, proj_fmt=PROJ_F32, norm_eps=1e-5),
    "whisper_base": _m(name="whisper_base", family="whisper", n_layers=6, d_model=512, n_heads=8,
                       head_dim=64, d_ff=2048, vocab=51865, max_pos=448, enc_len=1500,
                       proj_fmt=PROJ_F32, norm_eps=1e-5),
    "qwen2_0_5b_int8": _m(name="qwen2_0_5b_int8", family="qwen2", n_layers=24, d_model=1024,
                          n_heads=16, head_dim=64, d_ff=2816, vocab=151936, max_pos=32768,
                          enc_len=0, proj_fmt=PROJ_W8A8, norm_eps=1e-6, rope_theta=1e6),
    "whisper_large_v3_w8a32": _m(name="whisper_large_v3_w8a32", family="whisper", n_layers=32,
                                 d_model=1280, n_heads=20, head_dim=64, d_ff=5120, vocab=51866,
                                 max_pos=448, enc_len=1500, proj_fmt=PROJ_W8A32, norm_eps=1e-5),
    # Small models for oracle pins and fast parity tests. Sizes still span several
    # kernel tiles and leave ragged tails (odd vocab, d_ff not a power of two).
    "tiny_whisper": _m(name="tiny_whisper", family="whisper", n_layers=2, d_model=128, n_heads=2,
                       head_dim=64, d_ff=384, vocab=1031, max_pos=64, enc_len=40,
                       proj_fmt=PROJ_F32, norm_eps=1e-5),
    "tiny_whisper_w8a32": _m(name="tiny_whisper_w8a32", family="whisper", n_layers=2, d_model=192,
                             n_heads=3, head_dim=64, d_ff=320, vocab=997, max_pos=64, enc_len=37,
                             proj_fmt=PROJ_W8A32, norm_eps=1e-5),
    "tiny_qwen2": _m(name="tiny_qwen2", family="qwen2", n_layers=2, d_model=128, n_heads=2,
                     head_dim=64, d_ff=352, vocab=1009, max_pos=32768, enc_len=0,
                     proj_fmt=PROJ_W8A8, norm_eps=1e-6, rope_theta=1e6),
    "small_qwen2": _m(name="small_qwen2", family="qwen2", n_layers=3, d_model=256, n_heads=4,
                      head_dim=64, d_ff=704, vocab=4099, max_pos=32768, enc_len=0,
                      proj_fmt=PROJ_W8A8, norm_eps=1e-6, rope_theta=1e6),
    # Mid-size models whose matrices are large enough that batches of 8+ take the
    # tensor-core projection kernels (q|k|v, gate/up, down for W8A8; fc2 for f32).
    "mid_whisper": _m(name="mid_whisper", family="whisper", n_layers=2, d_model=256, n_heads=4,
                      head_dim=64, d_ff=2048, vocab=1031, max_pos=64, enc_len=40,
                      proj_fmt=PROJ_F32, norm_eps=1e-5),
    "mid_qwen2": _m(name="mid_qwen2", family="qwen2", n_layers=2, d_model=896, n_heads=14,
                    head_dim=64, d_ff=2432, vocab=1009, max_pos=32768, enc_len=0,
                    proj_fmt=PROJ_W8A8, norm_eps=1e-6, rope_theta=1e6),
    # Grouped-query attention (two query heads per K/V head, and seven as in Qwen2-0.5B's
    # 14 query / 2 K/V heads at d 896).
    "tiny_qwen2_gqa": _m(name="tiny_qwen2_gqa", family="qwen2", n_layers=2, d_model=256, n_heads=4,
                         head_dim=64, d_ff=352, vocab=1009, max_pos=32768, enc_len=0,
                         proj_fmt=PROJ_W8A8, norm_eps=1e-6, rope_theta=1e6, n_kv_heads=2),
    "mid_qwen2_gqa": _m(name="mid_qwen2_gqa", family="qwen2", n_layers=2, d_model=896, n_heads=14,
                        head_dim=64, d_ff=2432, vocab=1009, max_pos=32768, enc_len=0,
                        proj_fmt=PROJ_W8A8, norm_eps=1e-6, rope_theta=1e6, n_kv_heads=2),
}

WORKLOADS: Dict[str, Workload] = {
    # Single decode step of the one-block Whisper-tiny decoder; 31 prefilled positions.
    "c1_whisper_tiny_block_b1": Workload("c1_whisper_tiny_block_b1", MODELS["whisper_tiny_block"],
                                         batch=1, max_cache_len=448, cache_init="prefill",
                                         lens_lo=31, lens_hi=31, steps=1),
    # Whisper-base, 16 streams with ragged prefilled lengths, 64 greedy steps; a stream
    # retires when its cache reaches the 448-row position table.
    "c2_whisper_base_b16": Workload("c2_whisper_base_b16", MODELS["whisper_base"], batch=16,
                                    max_cache_len=448, cache_init="prefill", lens_lo=1,
                                    lens_hi=447, steps=64, retire_at=448),
    # Qwen2-0.5B int8, batch 1, 1024 prefilled tokens then 128 greedy steps.
    "c3_qwen2_0_5b_int8_b1": Workload("c3_qwen2_0_5b_int8_b1", MODELS["qwen2_0_5b_int8"], batch=1,
                                      max_cache_len=1152, cache_init="prefill", lens_lo=1024,
                                      lens_hi=1024, steps=128),
    # Same model, 64 streams, caches seeded with N(0,1) K/V of ragged lengths, 32 steps.
    "c4_qwen2_0_5b_int8_b64": Workload("c4_qwen2_0_5b_int8_b64", MODELS["qwen2_0_5b_int8"],
                                       batch=64, max_cache_len=4128, cache_init="kv_seed",
                                       lens_lo=128, lens_hi=4096, steps=32),
    # Whisper-large-v3 with int8 per-row weights and f32 activations, 32 streams,
    # 4 prompt tokens then 200 greedy steps.
    "c5_whisper_large_v3_w8a32_b32": Workload("c5_whisper_large_v3_w8a32_b32",
                                              MODELS["whisper_large_v3_w8a32"], batch=32,
                                              max_cache_len=448, cache_init="prefill", lens_lo=4,
                                              lens_hi=4, steps=200),
    # Small workloads for tests.
    "tiny_whisper_b3": Workload("tiny_whisper_b3", MODELS["tiny_whisper"], batch=3,
                                max_cache_len=64, cache_init="prefill", lens_lo=1, lens_hi=20,
                                steps=6),
    "tiny_whisper_w8a32_b3": Workload("tiny_whisper_w8a32_b3", MODELS["tiny_whisper_w8a32"],
                                      batch=3, max_cache_len=64, cache_init="prefill", lens_lo=1,
                                      lens_hi=20, steps=6),
    # batch 9: the tensor-core projection path (batch tiles of 16)
    "tiny_whisper_b9": Workload("tiny_whisper_b9", MODELS["tiny_whisper"], batch=9,
                                max_cache_len=64, cache_init="prefill", lens_lo=1, lens_hi=20,
                                steps=4),
    "tiny_whisper_w8a32_b9": Workload("tiny_whisper_w8a32_b9", MODELS["tiny_whisper_w8a32"],
                                      batch=9, max_cache_len=64, cache_init="prefill", lens_lo=1,
                                      lens_hi=20, steps=4),
    "tiny_qwen2_b3": Workload("tiny_qwen2_b3", MODELS["tiny_qwen2"], batch=3, max_cache_len=96,
                              cache_init="prefill", lens_lo=1, lens_hi=40, steps=6),
    "tiny_qwen2_b9": Workload("tiny_qwen2_b9", MODELS["tiny_qwen2"], batch=9, max_cache_len=96,
                              cache_init="prefill", lens_lo=1, lens_hi=40, steps=4),
    "mid_whisper_b9": Workload("mid_whisper_b9", MODELS["mid_whisper"], batch=9, max_cache_len=64,
                               cache_init="prefill", lens_lo=1, lens_hi=10, steps=3),
    "mid_qwen2_b9": Workload("mid_qwen2_b9", MODELS["mid_qwen2"], batch=9, max_cache_len=64,
                             cache_init="prefill", lens_lo=1, lens_hi=10, steps=3),
    "tiny_qwen2_gqa_b3": Workload("tiny_qwen2_gqa_b3", MODELS["tiny_qwen2_gqa"], batch=3, max_cache_len=96,
                                  cache_init="prefill", lens_lo=1, lens_hi=40, steps=4),
    "mid_qwen2_gqa_b9": Workload("mid_qwen2_gqa_b9", MODELS["mid_qwen2_gqa"], batch=9, max_cache_len=200,
                                 cache_init="kv_seed", lens_lo=1, lens_hi=150, steps=3),
    "small_qwen2_kv_b5": Workload("small_qwen2_kv_b5", MODELS["small_qwen2"], batch=5,
                                  max_cache_len=700, cache_init="kv_seed", lens_lo=1,
                                  lens_hi=600, steps=4),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def _rng(seed: int, *path: int) -> np.random.Generator:
    return np.random.default_rng([int(seed)] + [int(p) for p in path])


def _normal(rng: np.random.Generator, shape, std: float, mean: float = 0.0) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if mean != 0.0:
        x += np.float32(mean)
    return x


def quantize_weight_rows_offline(w: np.ndarray):
    """Offline per-output-row symmetric int8 quantisation of a weight matrix.

    Stands in for the pre-quantised checkpoint records: per row n,
    s_n = max_k |W_nk| / 127 and q_nk = clamp(rint(W_nk / s_n), -127, 127),
    round half to even, all in float32; an all-zero row has s_n = 0 and q = 0.
    Returns (q int8 [N, K], s float32 [N]).
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    amax = np.max(np.abs(w), axis=1)
    s = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = np.rint(w / safe[:, None])
    q = np.clip(q, -127, 127)
    q[s == 0] = 0
    return q.astype(np.int8), s


# Per-layer tensor ids: fixed numbering so the draw of any tensor is reproducible alone.
_LAYER_TENSORS = {
    "whisper": ["norm1_w", "norm1_b", "q", "k", "v", "o", "norm2_w", "norm2_b",
                "xq", "xk", "xv", "xo", "norm3_w", "norm3_b", "fc1", "fc2"],
    "qwen2": ["norm1_w", "norm2_w", "q", "k", "v", "o", "gate", "up", "down"],
}


def _proj_shape(cfg: ModelConfig, name: str):
    d, f, kv = cfg.d_model, cfg.d_ff, cfg.kv_dim
    return {"q": (d, d), "k": (kv, d), "v": (kv, d), "o": (d, d),
            "xq": (d, d), "xk": (d, d), "xv": (d, d), "xo": (d, d),
            "fc1": (f, d), "fc2": (d, f),
            "gate": (f, d), "up": (f, d), "down": (d, f)}[name]


def _proj_has_bias(cfg: ModelConfig, name: str) -> bool:
    if cfg.is_whisper:
        return True
    return name in ("q", "k", "v")


def make_weights(cfg: ModelConfig, seed: int = 0) -> dict:
    """Draw all weights of `cfg`.

    Returns a dict:
      tok_emb [V, d] f32 (also the tied LM head), pos_emb [max_pos, d] f32 (whisper),
      final_w [d], final_b [d] (whisper LayerNorm) or None,
      layers: list of per-layer dicts. Norm params are f32 vectors under norm1_w /
      norm1_b / norm2_w / norm2_b / norm3_w / norm3_b (b None for RMSNorm). Each
      projection is a dict {"w": f32 [out,in] or int8 [out,in], "s": f32 [out] row
      scales or None, "b": f32 [out] or None}.
    """
    fam = cfg.family
    d = cfg.d_model
    W: dict = {"config": cfg}
    W["tok_emb"] = _normal(_rng(seed, _TAG_WEIGHT, 0, 0), (cfg.vocab, d), 0.02)
    if cfg.is_whisper:
        W["pos_emb"] = _normal(_rng(seed, _TAG_WEIGHT, 0, 1), (cfg.max_pos, d), 0.02)
        W["final_w"] = _normal(_rng(seed, _TAG_WEIGHT, 0, 2), (d,), 0.02, 1.0)
        W["final_b"] = _normal(_rng(seed, _TAG_WEIGHT, 0, 3), (d,), 0.01)
    else:
        W["pos_emb"] = None
        W["final_w"] = _normal(_rng(seed, _TAG_WEIGHT, 0, 2), (d,), 0.02, 1.0)
        W["final_b"] = None
    layers = []
    for l in range(cfg.n_layers):
        L: dict = {}
        for t, name in enumerate(_LAYER_TENSORS[fam]):
            g = _rng(seed, _TAG_WEIGHT, l + 1, t)
            if name.startswith("norm"):
                if name.endswith("_w"):
                    L[name] = _normal(g, (d,), 0.02, 1.0)
                else:
                    L[name] = _normal(g, (d,), 0.01)
                continue
            shape = _proj_shape(cfg, name)
            w = _normal(g, shape, 0.02)
            b = _normal(g, (shape[0],), 0.01) if _proj_has_bias(cfg, name) else None
            if cfg.proj_fmt == PROJ_F32:
                L[name] = {"w": w, "s": None, "b": b}
            else:
                q, s = quantize_weight_rows_offline(w)
                L[name] = {"w": q, "s": s, "b": b}
        if not cfg.is_whisper:
            L["norm1_b"] = None
            L["norm2_b"] = None
        layers.append(L)
    W["layers"] = layers
    return W


def encoder_hidden(cfg: ModelConfig, stream: int, seed: int = 0) -> np.ndarray:
    """N(0,1) encoder hidden states [enc_len, d] f32 for one stream (whisper only)."""
    return _normal(_rng(seed, _TAG_ENC, stream), (cfg.enc_len, cfg.d_model), 1.0)


def token_ids(cfg: ModelConfig, stream: int, n: int, seed: int = 0) -> np.ndarray:
    """n uniform token ids in [0, vocab) for one stream, int32."""
    return _rng(seed, _TAG_TOK, stream).integers(0, cfg.vocab, size=n, dtype=np.int64).astype(np.int32)


def cache_lens(wl: Workload, seed: int = 0) -> np.ndarray:
    """Initial cache length of each stream, uniform over [lens_lo, lens_hi], int32."""
    if wl.lens_lo == wl.lens_hi:
        return np.full(wl.batch, wl.lens_lo, dtype=np.int32)
    g = _rng(seed, _TAG_LENS, wl.batch, wl.lens_lo, wl.lens_hi)
    return g.integers(wl.lens_lo, wl.lens_hi + 1, size=wl.batch, dtype=np.int64).astype(np.int32)


def seed_kv(cfg: ModelConfig, stream: int, layer: int, n_rows: int, seed: int = 0):
    """N(0,1) K and V rows [n_rows, kv heads * head_dim] f32 for one stream and layer (token-major)."""
    g = _rng(seed, _TAG_KV, stream, layer)
    dm = cfg.kv_dim
    k = g.standard_normal((n_rows, dm), dtype=np.float32)
    v = g.standard_normal((n_rows, dm), dtype=np.float32)
    return k, v


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (for smaller test variants)."""
    return dataclasses.replace(wl, **changes)
