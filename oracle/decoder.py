"""Plain, slow, obviously-correct CPU decoder step (test infrastructure only).

Sources (docs.rs source pages), cited by crate, file and item:
  [wa-dec]  whisper-apr 0.3.3 src/model/decoder_generated.rs
  [wa-cuda] whisper-apr 0.3.0 src/cuda/impl_generated.rs
  [focr]    franken_ocr 0.8.0 src/native_engine/decoder_qwen2.rs
  [cera]    cera 0.5.4 src/model/whisper.rs
  [q8]      lattice-inference 0.4.0 src/forward/cpu_q8.rs

Every tensor the pages store is stored here as float32; every reduction is an
f64 library primitive (matmul, sum). The activation quantiser and the argmax
decide integers in float32, as the pages do.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np

F32 = np.float32
F64 = np.float64

# ---------------------------------------------------------------------------
# Leaf operations
# ---------------------------------------------------------------------------


def layer_norm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * g + b.

    Population variance (divide by d), eps added inside the square root
    ([wa-dec] final-norm trace in `forward_traced`: mean, variance over d,
    std = sqrt(var + 1e-5); [cera] `decode_step_into`, layer_norm_inplace with
    LAYER_NORM_EPS). Pinned: constant row gives b; torch layer_norm in f64.
    """
    x64 = np.asarray(x, dtype=F32).astype(F64)
    mu = x64.mean(axis=-1, keepdims=True)
    var = np.square(x64 - mu).mean(axis=-1, keepdims=True)
    y = (x64 - mu) / np.sqrt(var + float(F32(eps))) * g.astype(F64) + b.astype(F64)
    return y.astype(F32)


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * w.

    Qwen2 input and post-attention norms and the final norm ([focr] module doc:
    "RMSNorm eps=1e-6"; `qwen2_decode_step`, `family_norm`). The body of the
    pages' rms_norm is not shown; this is the standard Qwen2 form with a plain
    weight (not the 1+gamma form of another model on the [q8] page).
    Pinned: closed form on a hand vector; torch rms_norm in f64.
    """
    x64 = np.asarray(x, dtype=F32).astype(F64)
    ms = np.square(x64).mean(axis=-1, keepdims=True)
    y = x64 / np.sqrt(ms + float(F32(eps))) * w.astype(F64)
    return y.astype(F32)


def quantize_rows_i8_te(x: np.ndarray):
    """Per-row symmetric int8 activation quantisation, round half to even.

    [focr] `qwen2_decode_step` quantises each normed row once
    (`quantize_row_i8_te`) before the int8 GEMV; the module doc names the rule
    "ties-to-even". The body is not on the page; reading taken, all in float32:
      amax = max_i |x_i|; if amax == 0 then q = 0 and a = 0;
      else inv = 127 / amax (one f32 division), q_i = clamp(rint(x_i * inv), -127, 127),
      a = amax / 127.
    Symmetric: -128 never occurs. Returns (q int8 [M,K], a f32 [M]).
    Pinned: hand-computed codes incl. exact .5 ties; round trips; error <= a/2.
    """
    x = np.atleast_2d(np.asarray(x, dtype=F32))
    amax = np.max(np.abs(x), axis=1).astype(F32)
    nz = amax > 0
    inv = np.zeros_like(amax)
    inv[nz] = F32(127.0) / amax[nz]
    prod = (x * inv[:, None]).astype(F32)
    q = np.clip(np.rint(prod), -127, 127).astype(np.int8)
    a = (amax / F32(127.0)).astype(F32)
    return q, a


def dequantize_rows_i8(q: np.ndarray, a: np.ndarray) -> np.ndarray:
    """q * a per row, f32 (the value an int8 row stands for)."""
    return (q.astype(F64) * a.astype(F64)[:, None]).astype(F32)


def quantize_weight_rows(w: np.ndarray):
    """Per-output-row symmetric int8 weight quantisation (offline, checkpoint side).

    [q8] module doc: projection matrices are "per-row symmetric INT8 quantized"
    with f32 activations; [focr] `GotLayerW`: int8 records with per-output-
    channel scales. Reading taken (body not shown), in float32:
      s_n = max_k |W_nk| / 127; q_nk = clamp(rint(W_nk / s_n), -127, 127);
      an all-zero row has s_n = 0, q = 0.
    Pinned: hand values; round trip; error <= s/2; equals the synthetic
    checkpoint writer on the same weights.
    """
    w = np.asarray(w, dtype=F32)
    amax = np.max(np.abs(w), axis=1).astype(F32)
    s = (amax / F32(127.0)).astype(F32)
    q = np.zeros(w.shape, dtype=np.int8)
    nz = s > 0
    q[nz] = np.clip(np.rint((w[nz] / s[nz, None]).astype(F32)), -127, 127).astype(np.int8)
    return q, s


def _as64(w: np.ndarray, w64: Optional[np.ndarray]) -> np.ndarray:
    """The weights in f64: `w64` when the caller already holds that exact conversion
    (the decoder keeps one per matrix so that it converts each matrix once), else a new one."""
    return w.astype(F64) if w64 is None else w64


def int8_dot_acc(xq: np.ndarray, wq: np.ndarray, w64: Optional[np.ndarray] = None) -> np.ndarray:
    """Exact integer dot products acc[m, n] = sum_k xq[m,k] * wq[n,k] (int64).

    The int32 accumulation of the int8 GEMV ([focr] `gemv_i8_bias_prequant`,
    "int8, int32 accumulate"). f64 matmul is exact here: every product is at
    most 127^2 and every sum below 2^53. Pinned: brute-force Python int loop.
    """
    acc = np.atleast_2d(xq).astype(F64) @ _as64(np.atleast_2d(wq), w64).T
    return np.rint(acc).astype(np.int64)


def linear_f32(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray],
               w64: Optional[np.ndarray] = None) -> np.ndarray:
    """y = x W^T (+ b), f32 weights and activations ([cera] `linear_proj`).

    Pinned: zero weights give the bias (the page's own worked case:
    W = 0, b = 1 gives y = 1); brute-force loop on tiny shapes.
    """
    y = np.atleast_2d(x).astype(F64) @ _as64(w, w64).T
    if b is not None:
        y = y + b.astype(F64)
    return y.astype(F32)


def linear_w8a8(xq: np.ndarray, a: np.ndarray, wq: np.ndarray, s: np.ndarray,
                b: Optional[np.ndarray], w64: Optional[np.ndarray] = None) -> np.ndarray:
    """int8 x int8 projection: y_n = acc_n * (a * s_n) + b_n.

    [focr] `linear_auto` / `add_bias`: the int8 path dequantises the int32
    accumulator per row and adds the f32 bias after dequant. Reading of the
    dequant: acc times activation scale times row scale, then bias.
    Pinned: integer part by brute force; zero activation row gives the bias;
    per-row scales by a brute-force loop with non-uniform scales.
    """
    acc = int8_dot_acc(xq, wq, w64).astype(F64)
    y = acc * np.asarray(a, dtype=F32).astype(F64)[:, None] * s.astype(F64)[None, :]
    if b is not None:
        y = y + b.astype(F64)
    return y.astype(F32)


def linear_w8a32(x: np.ndarray, wq: np.ndarray, s: np.ndarray,
                 b: Optional[np.ndarray], w64: Optional[np.ndarray] = None) -> np.ndarray:
    """int8 weights with f32 activations: y_n = s_n * sum_k q_nk x_k + b_n.

    [q8] module doc: int8 per-row weights are dequantised to f32 and used
    against f32 activations (`matmul_bt_q8`). Same value as dequantise-then-
    matmul up to rounding. Pinned: equals linear_f32 on the dequantised matrix;
    per-row scales by a brute-force loop with non-uniform scales.
    """
    y = (np.atleast_2d(x).astype(F64) @ _as64(wq, w64).T) * s.astype(F64)[None, :]
    if b is not None:
        y = y + b.astype(F64)
    return y.astype(F32)


def rope_cos_sin(pos: int, theta: float, head_dim: int = 64):
    """NEOX RoPE table row for one position: cos and sin of pos * theta^(-2i/head_dim).

    [focr] module doc: "RoPE theta=1e6", NEOX rotate-half (HF Qwen2). The
    table builder is not on the page; angles and their cos/sin are taken in
    f64 and rounded to f32. Returns (cos f32 [half], sin f32 [half]).
    """
    half = head_dim // 2
    i = np.arange(half, dtype=F64)
    inv_freq = np.power(F64(theta), -2.0 * i / head_dim)
    ang = F64(pos) * inv_freq
    return np.cos(ang).astype(F32), np.sin(ang).astype(F32)


def apply_rope_neox(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE on each head of x [..., H, head_dim].

    Pairs are (i, i + half): x_i' = x_i c - x_{i+half} s, x_{i+half}' = x_i s + x_{i+half} c
    ([q8] full-attention step, "stride-half pairing (i, half+i)"; [focr]
    `qwen2_decode_step` applies it to q and k before the cache append).
    Pinned: norm preservation, identity at pos 0, complex-number form,
    interleaved-pairing mutation moves the result.
    """
    x64 = np.asarray(x, dtype=F32).astype(F64)
    half = x64.shape[-1] // 2
    c = cos.astype(F64)
    s = sin.astype(F64)
    x0 = x64[..., :half]
    x1 = x64[..., half:]
    out = np.empty_like(x64)
    out[..., :half] = x0 * c - x1 * s
    out[..., half:] = x0 * s + x1 * c
    return out.astype(F32)


def softmax_weights(scores: np.ndarray) -> np.ndarray:
    """Max-subtracted softmax along the last axis (f64), failing closed per row.

    [focr] `decode_attn_head`: subtract the row max, exponentiate, divide by
    the sum. [q8] full-attention step: a non-finite or non-positive sum gives
    all-zero weights instead of NaN. Pinned: sums to 1 within 1e-6; NaN row
    gives zeros; single entry gives 1.
    """
    s = np.asarray(scores, dtype=F64)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    den = e.sum(axis=-1, keepdims=True)
    ok = np.isfinite(den) & (den > 0)
    return np.where(ok, e / np.where(ok, den, 1.0), 0.0)


def _attend_heads(q64: np.ndarray, k64h: np.ndarray, v64h: np.ndarray) -> np.ndarray:
    """q64 [H, dh]; k64h, v64h [H, n, dh] (f64) -> [H, dh] f64 (see attention_decode)."""
    dh = q64.shape[-1]
    scale = 1.0 / math.sqrt(dh)
    sc = np.matmul(k64h, q64[:, :, None])[:, :, 0] * scale     # [H, n]
    p = softmax_weights(sc)
    return np.matmul(p[:, None, :], v64h)[:, 0, :]


def attention_decode(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """One query row attending all given cached rows, per head.

    q [H, dh] f32; k, v [n, H, dh] f32 (token-major cache rows 0..n-1, the new
    row included). For each head: s_j = (q . k_j) / sqrt(dh) (1/8 at dh = 64),
    p = softmax(s), out = sum_j p_j v_j ([focr] `qwen2_decode_attention` /
    `decode_attn_head`; [cera] `multi_head_attention`). No mask: every cached
    row is at or before the query. Returns [H, dh] f32.
    Pinned: torch scaled_dot_product_attention in f64; one key gives v;
    identical keys give the mean of v.
    """
    q64 = np.asarray(q, dtype=F32).astype(F64)
    k64h = np.asarray(k, dtype=F32).astype(F64).transpose(1, 0, 2)
    v64h = np.asarray(v, dtype=F32).astype(F64).transpose(1, 0, 2)
    return _attend_heads(q64, k64h, v64h).astype(F32)


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).

    [wa-cuda] `gelu`; the Whisper FFN activation. Pinned: torch gelu
    (approximate='tanh') in f64; gelu(0) = 0; odd-part identity.
    """
    x64 = np.asarray(x, dtype=F32).astype(F64)
    y = 0.5 * x64 * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x64 + 0.044715 * x64 ** 3)))
    return y.astype(F32)


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU: x / (1 + exp(-x)) ([focr] SwiGLU MLP gate). Pinned: torch silu in f64."""
    x64 = np.asarray(x, dtype=F32).astype(F64)
    return (x64 / (1.0 + np.exp(-x64))).astype(F32)


def argmax_first(logits: np.ndarray) -> int:
    """Greedy pick over one f32 logit row; the lowest index wins ties ([focr] `argmax`:
    fold keeping the earlier index unless a later value is strictly greater).

    NaN never wins (a NaN comparison is false). Pinned: hand rows with ties.
    """
    row = np.asarray(logits, dtype=F32)
    clean = np.where(np.isnan(row), F32(-np.inf), row)
    i = int(np.argmax(clean))   # numpy returns the first index of the maximum
    if not clean[i] > F32(-np.inf):
        return 0
    return i


# ---------------------------------------------------------------------------
# Decoder
# ---------------------------------------------------------------------------

# Distance, in code units of x * 127 / amax, from a rounding boundary within which another
# correct f32 implementation may put an activation on the other side, per quantisation site of
# a qwen2 layer: norm and SwiGLU outputs (sites 0, 2, 3) differ by a few ulps (a few 1e-5 code
# units); the attention context feeding the o projection (site 1) is an f32 online softmax over
# up to thousands of keys and differs by more.
NEAR_TIE_EPS = {0: 2e-4, 1: 5e-3, 2: 2e-4, 3: 2e-4}


class StreamState:
    """One stream's decode state: per-layer self K/V rows and static cross K/V.

    Self caches are token-major [max_len, kv heads * dh] f32 per layer, holding post-RoPE
    K (qwen2) and V ([focr] `Qwen2KvCache`; [cera] `WhisperDecoderKVCache`).
    Cross K/V [enc_len, d] f32 per layer are computed once from the encoder
    hidden states ([cera] `precompute_cross_attention`).
    """

    def __init__(self, n_layers: int, kv_dim: int, max_len: int):
        self.n = 0
        self.max_len = max_len
        self.k = [np.zeros((max_len, kv_dim), dtype=F32) for _ in range(n_layers)]
        self.v = [np.zeros((max_len, kv_dim), dtype=F32) for _ in range(n_layers)]
        self.xk: Optional[List[np.ndarray]] = None
        self.xv: Optional[List[np.ndarray]] = None


class OracleDecoder:
    """The pages' decoder forward, one or many new rows per call.

    `weights` is the dict produced by the synthetic generator (synth.make_weights):
    f32 token embedding (tied LM head), f32 learned positions (whisper), norm
    parameters, and per-layer projections {"w", "s", "b"} in the model's format.
    """

    def __init__(self, weights: dict, max_cache_len: int, quant_jitter: Optional[int] = None,
                 share_weights_with: Optional["OracleDecoder"] = None):
        """quant_jitter: None (the oracle proper) or a seed. With a seed, every activation
        whose value times 127 / amax lies within NEAR_TIE_EPS of a rounding boundary rounds
        to the other neighbouring integer with probability 1/2. That models another correct
        f32 implementation of the norm / attention / SwiGLU feeding the quantiser, whose value
        may differ in the last bits and so round the other way at a tie. Tests use a few such
        runs to measure how far correct implementations drift apart; it changes nothing when
        None."""
        self.W = weights
        self.cfg = weights["config"]
        self.max_len = max_cache_len
        self._c64: dict = share_weights_with._c64 if share_weights_with is not None else {}
        self._jitter = np.random.default_rng(quant_jitter) if quant_jitter is not None else None
        # Diagnostics only (no effect on results): per-row smallest distance, in code
        # units, between an activation's x * inv and a rounding boundary k + 1/2, over all
        # int8 quantisations of the last forward_rows call.
        self.last_margins: Optional[np.ndarray] = None
        self._margins: Optional[np.ndarray] = None
        # Tie bookkeeping of layer_forward (off unless a test asks): quantisation sites are
        # numbered in call order within one layer (qwen2: 0 the q|k|v input, 1 the o input,
        # 2 the gate/up input, 3 the down input). `tie_log`, when a list, receives
        # (site, row, col, distance) for every activation whose x * inv lies within
        # `tie_eps` code units (a number, or a dict site -> number) of a rounding
        # boundary; `flips` maps site -> [(row, col)] of
        # activations to round to the other neighbouring integer instead (a correct
        # implementation whose value sat on the other side of the tie).
        self.tie_log: Optional[list] = None
        self.tie_eps = 0.0
        self.flips: Optional[dict] = None
        self._site = 0

    # -- helpers ------------------------------------------------------------

    def _w64(self, key, arr: np.ndarray) -> np.ndarray:
        c = self._c64.get(key)
        if c is None:
            c = arr.astype(F64)
            self._c64[key] = c
        return c

    def _proj(self, x: np.ndarray, p: dict, key) -> np.ndarray:
        """Whisper projection in the model's format: f32 weights (linear_f32) or int8
        weights with per-row scales and f32 activations (linear_w8a32)."""
        w64 = self._w64(key, p["w"])
        if p["s"] is None:
            return linear_f32(x, p["w"], p["b"], w64=w64)
        return linear_w8a32(x, p["w"], p["s"], p["b"], w64=w64)

    def _proj_i8(self, x: np.ndarray, p: dict, key, quantised=None) -> np.ndarray:
        """Qwen2 W8A8 projection (linear_w8a8): each input row quantised, exact integer
        dot, dequantised, bias. `quantised` = (codes, scales) of x when the caller already
        quantised it (one quantisation shared by several projections of the same row)."""
        xq, a = self._quant(x) if quantised is None else quantised
        return linear_w8a8(xq, a, p["w"], p["s"], p["b"], w64=self._w64(key, p["w"]))

    def _quant(self, x):
        q, a = quantize_rows_i8_te(x)
        site = self._site
        self._site += 1
        if self._jitter is not None:
            # another correct implementation: every activation within NEAR_TIE_EPS of a
            # rounding boundary rounds to the other neighbouring integer with probability 1/2
            x32 = np.atleast_2d(np.asarray(x, F32))
            inv = np.where(a > 0, F32(127.0) / np.where(a > 0, np.max(np.abs(x32), axis=1), F32(1)), F32(0))
            prod = (x32 * inv.astype(F32)[:, None]).astype(np.float64)
            near = np.abs(prod - np.floor(prod) - 0.5) < NEAR_TIE_EPS.get(site, NEAR_TIE_EPS[0])
            flip = near & (self._jitter.random(prod.shape) < 0.5)
            if flip.any():
                q = q.copy()
                alt = q.astype(np.int64) + np.where(prod > q, 1, -1)
                q[flip] = np.clip(alt[flip], -127, 127).astype(np.int8)
        if self._margins is not None or self.tie_log is not None or self.flips:
            x32 = np.atleast_2d(np.asarray(x, F32))
            inv = np.where(a > 0, F32(127.0) / np.where(a > 0, np.max(np.abs(x32), axis=1), F32(1)), F32(0))
            prod = (x32 * inv.astype(F32)[:, None]).astype(np.float64)
            dist = np.abs(prod - np.floor(prod) - 0.5)
            if self._margins is not None:
                self._margins = np.minimum(self._margins, dist.min(axis=1))
            if self.tie_log is not None:
                eps = self.tie_eps.get(site, 0.0) if isinstance(self.tie_eps, dict) else self.tie_eps
                for r, c in zip(*np.nonzero(dist < eps)):
                    self.tie_log.append((site, int(r), int(c), float(dist[r, c])))
            if self.flips and site in self.flips:
                q = q.copy()
                for r, c in self.flips[site]:
                    alt = int(q[r, c]) + (1 if prod[r, c] > q[r, c] else -1)
                    q[r, c] = np.int8(min(127, max(-127, alt)))
        return q, a

    def _norm(self, x, w, b):
        if self.cfg.is_whisper:
            return layer_norm(x, w, b, self.cfg.norm_eps)
        return rms_norm(x, w, self.cfg.norm_eps)

    def new_state(self, enc_hidden: Optional[np.ndarray] = None) -> StreamState:
        cfg = self.cfg
        st = StreamState(cfg.n_layers, cfg.kv_dim, self.max_len)
        if cfg.is_whisper:
            if enc_hidden is None:
                raise ValueError("whisper stream needs encoder hidden states")
            enc = np.asarray(enc_hidden, dtype=F32)
            if enc.shape != (cfg.enc_len, cfg.d_model):
                raise ValueError(f"encoder hidden must be [{cfg.enc_len}, {cfg.d_model}]")
            st.xk, st.xv = [], []
            for l, L in enumerate(self.W["layers"]):
                st.xk.append(self._proj(enc, L["xk"], (l, "xk")))
                st.xv.append(self._proj(enc, L["xv"], (l, "xv")))
        return st

    # -- forward ------------------------------------------------------------

    def embed(self, tokens, positions) -> np.ndarray:
        """x = E[token] (+ P[position] for whisper), one row per token."""
        cfg = self.cfg
        E = self.W["tok_emb"]
        x = np.empty((len(tokens), cfg.d_model), dtype=F32)
        for r, (t, p) in enumerate(zip(tokens, positions)):
            if not (0 <= int(t) < cfg.vocab):
                raise ValueError(f"token {t} outside vocab {cfg.vocab}")
            if not (0 <= int(p) < cfg.max_pos):
                raise ValueError(f"position {p} outside [0, {cfg.max_pos})")
            x[r] = E[int(t)]
            if cfg.is_whisper:
                # learned position row added to the token row ([cera] decode_step_into step 1)
                x[r] = x[r] + self.W["pos_emb"][int(p)]
        return x

    def _self_attention(self, l, q, row_states, row_slots):
        """Per row: attend cache rows 0..row_slots[r] of its own stream (all heads). With
        grouped K/V heads, query head h attends K/V head h // (H / H_kv) ([focr] native
        kv-lane mapping of grouped-query attention)."""
        cfg = self.cfg
        H, dh, Hkv = cfg.n_heads, cfg.head_dim, cfg.kv_heads
        group = H // Hkv
        ctx = np.empty_like(q)
        views = {}
        for r in range(len(row_slots)):
            st = row_states[r]
            if id(st) not in views:
                top = max(sl for s2, sl in zip(row_states, row_slots) if s2 is st) + 1
                kh = st.k[l][:top].astype(F64).reshape(top, Hkv, dh).transpose(1, 0, 2)
                vh = st.v[l][:top].astype(F64).reshape(top, Hkv, dh).transpose(1, 0, 2)
                views[id(st)] = (np.ascontiguousarray(np.repeat(kh, group, axis=0)),
                                 np.ascontiguousarray(np.repeat(vh, group, axis=0)))
            kh, vh = views[id(st)]
            n = row_slots[r] + 1
            ctx[r] = _attend_heads(q[r].reshape(H, dh).astype(F64), kh[:, :n], vh[:, :n]).astype(F32).reshape(-1)
        return ctx

    def layer_forward(self, l: int, x: np.ndarray, row_states: Sequence[StreamState],
                      row_slots: Sequence[int], positions: Sequence[int]) -> np.ndarray:
        """Layer l of the decoder on rows x [R, d] (the residual stream entering the layer);
        writes each row's K/V at its cache row and returns the residual leaving the layer.
        Row r attends cache rows 0..row_slots[r] of its own stream."""
        cfg = self.cfg
        H, dh = cfg.n_heads, cfg.head_dim
        R = x.shape[0]
        L = self.W["layers"][l]
        self._site = 0
        # ---- self-attention block ----
        h = self._norm(x, L["norm1_w"], L["norm1_b"])
        if cfg.is_whisper:
            q = self._proj(h, L["q"], (l, "q"))
            k = self._proj(h, L["k"], (l, "k"))
            v = self._proj(h, L["v"], (l, "v"))
        else:
            # one quantisation of the normed row shared by q, k, v ([focr] fused q|k|v GEMV)
            hq = self._quant(h)
            q = self._proj_i8(h, L["q"], (l, "q"), hq)
            k = self._proj_i8(h, L["k"], (l, "k"), hq)
            v = self._proj_i8(h, L["v"], (l, "v"), hq)
            for r in range(R):
                c, s = rope_cos_sin(int(positions[r]), cfg.rope_theta, dh)
                q[r] = apply_rope_neox(q[r].reshape(H, dh), c, s).reshape(-1)
                k[r] = apply_rope_neox(k[r].reshape(cfg.kv_heads, dh), c, s).reshape(-1)
        for r in range(R):
            row_states[r].k[l][row_slots[r]] = k[r]
            row_states[r].v[l][row_slots[r]] = v[r]
        ctx = self._self_attention(l, q, row_states, row_slots)
        if cfg.is_whisper:
            x = x + self._proj(ctx, L["o"], (l, "o"))
        else:
            x = x + self._proj_i8(ctx, L["o"], (l, "o"))
        # ---- cross-attention block (whisper) ----
        if cfg.is_whisper:
            h = self._norm(x, L["norm2_w"], L["norm2_b"])
            qx = self._proj(h, L["xq"], (l, "xq"))
            cx = np.empty_like(qx)
            xviews = {}
            ne = cfg.enc_len
            for r in range(R):
                st = row_states[r]
                if id(st) not in xviews:
                    xviews[id(st)] = (
                        np.ascontiguousarray(st.xk[l].astype(F64).reshape(ne, H, dh).transpose(1, 0, 2)),
                        np.ascontiguousarray(st.xv[l].astype(F64).reshape(ne, H, dh).transpose(1, 0, 2)))
                kh, vh = xviews[id(st)]
                cx[r] = _attend_heads(qx[r].reshape(H, dh).astype(F64), kh, vh).astype(F32).reshape(-1)
            x = x + self._proj(cx, L["xo"], (l, "xo"))
        # ---- feed-forward block ----
        if cfg.is_whisper:
            h = self._norm(x, L["norm3_w"], L["norm3_b"])
            f = gelu_tanh(self._proj(h, L["fc1"], (l, "fc1")))
            x = x + self._proj(f, L["fc2"], (l, "fc2"))
        else:
            h = self._norm(x, L["norm2_w"], L["norm2_b"])
            hq = self._quant(h)  # shared by gate and up
            g = self._proj_i8(h, L["gate"], (l, "gate"), hq)
            u = self._proj_i8(h, L["up"], (l, "up"), hq)
            m = (silu(g) * u).astype(F32)
            x = x + self._proj_i8(m, L["down"], (l, "down"))
        return x

    def forward_rows(self, row_states: Sequence[StreamState], row_slots: Sequence[int],
                     tokens: Sequence[int], positions: Sequence[int],
                     logits_rows: Optional[Sequence[int]] = None):
        """Run rows through all layers.

        Row r belongs to stream row_states[r]; its K/V are written at cache row
        row_slots[r] and it attends cache rows 0..row_slots[r] of its own stream
        (causal: rows written by this call at later slots are not attended).
        Returns (final hidden before the final norm [R, d], logits [len(logits_rows), V]).
        """
        cfg = self.cfg
        R = len(tokens)
        for st, sl in zip(row_states, row_slots):
            if not (0 <= sl < st.max_len):
                raise ValueError(f"cache row {sl} outside [0, {st.max_len})")
        x = self.embed(tokens, positions)
        self._margins = np.full(R, np.inf)
        for l in range(cfg.n_layers):
            x = self.layer_forward(l, x, row_states, row_slots, positions)
        hidden = x
        self.last_margins, self._margins = self._margins, None
        if logits_rows is None:
            logits_rows = range(R)
        rows = list(logits_rows)
        logits = self.head(hidden[rows]) if rows else np.zeros((0, cfg.vocab), F32)
        return hidden, logits

    def head(self, x: np.ndarray) -> np.ndarray:
        """Final norm then the tied head: logits = E . norm(x) ([focr] `got_lm_head`,
        f32 arm; [cera] ln_post then proj_w gemv)."""
        h = self._norm(x, self.W["final_w"], self.W["final_b"])
        E64 = self._w64("tok_emb", self.W["tok_emb"])
        return (h.astype(F64) @ E64.T).astype(F32)

    # -- the calls the library exposes -----------------------------------------

    def step(self, states: Sequence[StreamState], tokens, positions):
        """One decode step over B streams: stream b's new row goes at its length."""
        slots = [st.n for st in states]
        for st in states:
            if st.n + 1 > st.max_len:
                raise OverflowError("cache overflow")
        hidden, logits = self.forward_rows(states, slots, tokens, positions)
        for st in states:
            st.n += 1
        return hidden, logits

    def prefill(self, st: StreamState, tokens, positions=None):
        """Run N tokens of one stream at cache rows st.n..st.n+N-1 (positions default
        to those rows) and return the last row's logits [V]."""
        n0 = st.n
        N = len(tokens)
        if positions is None:
            positions = list(range(n0, n0 + N))
        if n0 + N > st.max_len:
            raise OverflowError("cache overflow")
        _, logits = self.forward_rows([st] * N, list(range(n0, n0 + N)), tokens, positions,
                                      logits_rows=[N - 1])
        st.n = n0 + N
        return logits[0]

    def kv_append(self, st: StreamState, start: int, k: np.ndarray, v: np.ndarray):
        """Write rows [start, start+n) of every layer's K and V (k, v [L, n, d]) and
        set the stream length to start + n ([focr] `Qwen2KvCache::seed`)."""
        n = k.shape[1]
        if start + n > st.max_len:
            raise OverflowError("cache overflow")
        for l in range(self.cfg.n_layers):
            st.k[l][start:start + n] = k[l]
            st.v[l][start:start + n] = v[l]
        st.n = start + n

    def reprefill_logits(self, tokens, enc_hidden=None):
        """The O(n^2) path: a fresh stream prefilled with all tokens; last-row logits.

        [focr] module doc: `generate_greedy` (full re-prefill per token) is the
        correctness oracle the KV-cache decode must match argmax-exactly.
        """
        st = self.new_state(enc_hidden)
        return self.prefill(st, tokens)
