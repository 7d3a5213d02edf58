"""Pins for the oracle's whole decoder step on small models (CPU only).

  * KV-cache decode equals the O(n^2) re-prefill (argmax-exact, logits within 1e-5):
    franken_ocr decoder_qwen2.rs module doc, `generate_greedy` vs
    `generate_greedy_kvcache`.
  * Causal invariance: logits at position t do not depend on later tokens.
  * Batched step equals solo steps bit for bit (decoder_qwen2.rs,
    `qwen2_batched_decode_step`: per-stream logits byte-for-byte equal).
  * Cache round trip: seeding a fresh stream with another stream's K/V rows
    (`Qwen2KvCache::seed`) decodes identically.
  * Zero-weight decoders reduce to closed forms computed with torch routines.
  * Error conditions raise (token range, position range, cache overflow).
"""
import copy

import numpy as np
import pytest
import torch

import oracle
import synth

F32 = np.float32


def _model(name, seed=0):
    cfg = synth.MODELS[name]
    return cfg, synth.make_weights(cfg, seed)


def _new(dec, cfg, stream, seed=0):
    enc = synth.encoder_hidden(cfg, stream, seed) if cfg.is_whisper else None
    return dec.new_state(enc), enc


@pytest.mark.parametrize("name", ["tiny_whisper", "tiny_qwen2", "tiny_whisper_w8a32"])
def test_kv_decode_equals_reprefill(name):
    cfg, W = _model(name)
    dec = oracle.OracleDecoder(W, 64)
    st, enc = _new(dec, cfg, 0)
    toks = list(synth.token_ids(cfg, 0, 5))
    logits = dec.prefill(st, toks)
    for t in range(6):
        nxt = oracle.argmax_first(logits)
        ref = dec.reprefill_logits(toks, enc)
        assert oracle.argmax_first(ref) == nxt
        np.testing.assert_allclose(logits, ref, rtol=1e-5, atol=1e-6)
        toks.append(nxt)
        _, lg = dec.step([st], [nxt], [st.n])
        logits = lg[0]


@pytest.mark.parametrize("name", ["tiny_whisper", "tiny_qwen2"])
def test_causal_invariance(name):
    cfg, W = _model(name)
    dec = oracle.OracleDecoder(W, 64)
    a = list(synth.token_ids(cfg, 1, 12))
    b = a[:7] + list(synth.token_ids(cfg, 2, 5))
    assert a[7:] != b[7:]
    outs = []
    for toks in (a, b):
        st, _ = _new(dec, cfg, 0)
        _, lg = dec.forward_rows([st] * 12, list(range(12)), toks, list(range(12)))
        outs.append(lg)
    np.testing.assert_array_equal(outs[0][:7], outs[1][:7])
    assert np.abs(outs[0][7:] - outs[1][7:]).max() > 1e-3


@pytest.mark.parametrize("name", ["tiny_whisper", "tiny_qwen2"])
def test_batched_step_equals_solo_bitwise(name):
    cfg, W = _model(name)
    dec = oracle.OracleDecoder(W, 64)
    lens = [3, 9, 1]
    states, solo_states = [], []
    for s, n in enumerate(lens):
        st, _ = _new(dec, cfg, s)
        dec.prefill(st, list(synth.token_ids(cfg, s, n)))
        states.append(st)
        solo_states.append(copy.deepcopy(st))
    toks = [5, 17, 2]
    pos = [st.n for st in states]
    _, batched = dec.step(states, toks, pos)
    for s in range(3):
        _, solo = dec.step([solo_states[s]], [toks[s]], [pos[s]])
        np.testing.assert_array_equal(batched[s], solo[0])


@pytest.mark.parametrize("name", ["tiny_whisper", "tiny_qwen2"])
def test_cache_seed_round_trip(name):
    cfg, W = _model(name)
    dec = oracle.OracleDecoder(W, 64)
    st, enc = _new(dec, cfg, 0)
    dec.prefill(st, list(synth.token_ids(cfg, 0, 10)))
    fresh = dec.new_state(enc)
    n = st.n
    k = np.stack([st.k[l][:n] for l in range(cfg.n_layers)])
    v = np.stack([st.v[l][:n] for l in range(cfg.n_layers)])
    dec.kv_append(fresh, 0, k, v)
    _, a = dec.step([st], [7], [n])
    _, b = dec.step([fresh], [7], [n])
    np.testing.assert_array_equal(a, b)


def _zero_projections(W):
    for L in W["layers"]:
        for key, p in L.items():
            if isinstance(p, dict):
                p["w"] = np.zeros_like(p["w"])
                if p["s"] is not None:
                    p["s"] = np.zeros_like(p["s"])
    return W


def test_zero_weight_whisper_closed_form():
    cfg, W = _model("tiny_whisper")
    W = _zero_projections(W)
    L0 = W["layers"]
    # keep fc2 non-zero so the GELU -> fc2 -> residual chain is exercised
    rng = np.random.default_rng(0)
    for L in L0:
        L["fc2"]["w"] = (rng.standard_normal(L["fc2"]["w"].shape) * 0.02).astype(F32)
    dec = oracle.OracleDecoder(W, 64)
    st, _ = _new(dec, cfg, 0)
    dec.prefill(st, [3, 4, 5])
    tok, pos = 11, 3
    hidden, logits = dec.step([st], [tok], [pos])
    x = torch.from_numpy(W["tok_emb"][tok]).double() + torch.from_numpy(W["pos_emb"][pos]).double()
    for L in L0:
        # self-attention over rows that all equal b_v gives b_v; W_o = 0 leaves b_o
        x = x + torch.from_numpy(L["o"]["b"]).double()
        x = x + torch.from_numpy(L["xo"]["b"]).double()
        g = torch.nn.functional.gelu(torch.from_numpy(L["fc1"]["b"]).double(), approximate="tanh")
        x = x + torch.from_numpy(L["fc2"]["w"]).double() @ g + torch.from_numpy(L["fc2"]["b"]).double()
    np.testing.assert_allclose(hidden[0], x.numpy(), rtol=1e-5, atol=1e-6)
    h = torch.nn.functional.layer_norm(x, (cfg.d_model,), torch.from_numpy(W["final_w"]).double(),
                                       torch.from_numpy(W["final_b"]).double(), eps=1e-5)
    ref = torch.from_numpy(W["tok_emb"]).double() @ h
    np.testing.assert_allclose(logits[0], ref.numpy(), rtol=1e-4, atol=1e-5)


def test_zero_weight_qwen2_closed_form_with_identity_o():
    cfg, W = _model("tiny_qwen2")
    W = _zero_projections(W)
    d = cfg.d_model
    for L in W["layers"]:
        # o = identity: q = 127 on the diagonal with scale 1/127, so y = dequant(quant(ctx))
        L["o"]["w"] = (np.eye(d) * 127).astype(np.int8)
        L["o"]["s"] = np.full(d, F32(1.0) / F32(127.0), F32)
    dec = oracle.OracleDecoder(W, 64)
    st, _ = _new(dec, cfg, 0)
    dec.prefill(st, [1, 2, 3, 4])
    tok = 9
    hidden, logits = dec.step([st], [tok], [4])
    x = W["tok_emb"][tok].astype(np.float64)
    for L in W["layers"]:
        # every V row is b_v, so each head's context is b_v whatever the softmax weights
        bv = L["v"]["b"][None, :]
        q, a = oracle.quantize_rows_i8_te(bv)
        # acc_n = 127 q_n, then acc * a * (1/127) + no bias
        y = (q[0].astype(np.float64) * 127.0 * float(a[0]) * float(F32(1) / F32(127))).astype(F32)
        x = (x.astype(F32) + y).astype(np.float64)
    np.testing.assert_allclose(hidden[0], x, rtol=1e-5, atol=1e-6)
    h = torch.nn.functional.rms_norm(torch.from_numpy(x), (d,), torch.from_numpy(W["final_w"]).double(),
                                     eps=float(F32(1e-6)))
    ref = torch.from_numpy(W["tok_emb"]).double() @ h
    np.testing.assert_allclose(logits[0], ref.numpy(), rtol=1e-4, atol=1e-5)


def test_errors_raise():
    cfg, W = _model("tiny_whisper")
    dec = oracle.OracleDecoder(W, 8)
    st, _ = _new(dec, cfg, 0)
    with pytest.raises(ValueError):
        dec.step([st], [cfg.vocab], [0])
    with pytest.raises(ValueError):
        dec.step([st], [0], [cfg.max_pos])
    dec.prefill(st, list(range(8)))
    with pytest.raises(OverflowError):
        dec.step([st], [0], [8])


def test_identity_structured_whisper_layer_closed_form():
    """One Whisper layer with identity-like projections at position 0.

    q, k, xq, xk are zero; v, o, xv, xo are identities; fc1 = [I; 0], fc2 = [I, 0].
    Then, with x0 = E[t] + P[0] and the encoder mean m_enc:
      x1 = x0 + LN1(x0) + b_v + b_o                  (one cached row: weight 1)
      x2 = x1 + m_enc + b_xv + b_xo                   (equal keys: uniform weights)
      x3 = x2 + gelu(LN3(x2) + b_fc1)[:d] + b_fc2
    and logits = E . LN_f(x3). Built from torch routines only.
    """
    cfg = synth.dataclasses.replace(synth.MODELS["tiny_whisper"], n_layers=1)
    W = synth.make_weights(cfg, 3)
    W = _zero_projections(W)
    d, f = cfg.d_model, cfg.d_ff
    L = W["layers"][0]
    eye = np.eye(d, dtype=F32)
    for k in ("v", "o", "xv", "xo"):
        L[k]["w"] = eye.copy()
    L["fc1"]["w"] = np.concatenate([eye, np.zeros((f - d, d), F32)], axis=0)
    L["fc2"]["w"] = np.concatenate([eye, np.zeros((d, f - d), F32)], axis=1)
    dec = oracle.OracleDecoder(W, 16)
    enc = synth.encoder_hidden(cfg, 0, 3)
    st = dec.new_state(enc)
    tok = 77
    hidden, logits = dec.step([st], [tok], [0])
    T = lambda a: torch.from_numpy(np.asarray(a)).double()
    ln = lambda x, g, b: torch.nn.functional.layer_norm(x, (d,), T(g), T(b), eps=float(F32(1e-5)))
    x0 = T(W["tok_emb"][tok]) + T(W["pos_emb"][0])
    x1 = x0 + ln(x0, L["norm1_w"], L["norm1_b"]) + T(L["v"]["b"]) + T(L["o"]["b"])
    x2 = x1 + T(enc).mean(0) + T(L["xv"]["b"]) + T(L["xo"]["b"])
    g = torch.nn.functional.gelu(ln(x2, L["norm3_w"], L["norm3_b"]) + T(L["fc1"]["b"][:d]),
                                 approximate="tanh")
    x3 = x2 + g + T(L["fc2"]["b"])
    np.testing.assert_allclose(hidden[0], x3.numpy(), rtol=1e-5, atol=2e-6)
    ref = T(W["tok_emb"]) @ ln(x3, W["final_w"], W["final_b"])
    np.testing.assert_allclose(logits[0], ref.numpy(), rtol=1e-4, atol=1e-5)


def test_identity_structured_qwen2_mlp_closed_form():
    """One Qwen2 layer at position 0: attention zeroed (o = 0), gate = up = [I; 0]
    (int8 127 with scale 1/127), down = [I, 0]. Then with h = RMS2(x0):
      g = u = dequant(quant(h)) on the first d rows, m = silu(g) * u,
      x1 = x0 + dequant(quant(m))[:d].
    """
    cfg = synth.dataclasses.replace(synth.MODELS["tiny_qwen2"], n_layers=1)
    W = synth.make_weights(cfg, 4)
    W = _zero_projections(W)
    d, f = cfg.d_model, cfg.d_ff
    L = W["layers"][0]
    eye = (np.eye(d) * 127).astype(np.int8)
    inv = F32(1.0) / F32(127.0)
    L["gate"]["w"] = np.concatenate([eye, np.zeros((f - d, d), np.int8)], axis=0)
    L["up"]["w"] = L["gate"]["w"].copy()
    L["gate"]["s"] = np.full(f, inv, F32)
    L["up"]["s"] = np.full(f, inv, F32)
    L["down"]["w"] = np.concatenate([eye, np.zeros((d, f - d), np.int8)], axis=1)
    L["down"]["s"] = np.full(d, inv, F32)
    dec = oracle.OracleDecoder(W, 16)
    st = dec.new_state(None)
    tok = 5
    hidden, _ = dec.step([st], [tok], [0])
    x0 = W["tok_emb"][tok]
    h = torch.nn.functional.rms_norm(torch.from_numpy(x0).double(), (d,),
                                     torch.from_numpy(L["norm2_w"]).double(),
                                     eps=float(F32(1e-6))).numpy().astype(F32)
    q, a = oracle.quantize_rows_i8_te(h[None, :])
    gu = (q[0].astype(np.float64) * 127 * float(a[0]) * float(inv)).astype(F32)
    sil = torch.nn.functional.silu(torch.from_numpy(gu).double()).numpy().astype(F32)
    m = (sil * gu).astype(F32)
    mq, am = oracle.quantize_rows_i8_te(np.concatenate([m, np.zeros(f - d, F32)])[None, :])
    y = (mq[0, :d].astype(np.float64) * 127 * float(am[0]) * float(inv)).astype(F32)
    np.testing.assert_allclose(hidden[0], (x0 + y).astype(F32), rtol=1e-6, atol=1e-7)


def test_quantisation_margin_diagnostic():
    """The oracle's near-tie diagnostic reports 0 for an exact .5 tie and the true
    distance otherwise, and changes no result."""
    cfg, W = _model("tiny_qwen2")
    dec = oracle.OracleDecoder(W, 8)
    dec._margins = np.full(2, np.inf)
    x = np.array([[127.0, 2.5, 1.0], [127.0, 2.25, 1.0]], F32)
    q, a = dec._quant(x)
    assert np.array_equal(q, oracle.quantize_rows_i8_te(x)[0])
    assert dec._margins[0] == 0.0 and dec._margins[1] == 0.25


def test_quant_jitter_flips_only_near_ties_and_is_off_by_default():
    """The ensemble runs of the W8A8 parity check round only activations within NEAR_TIE_EPS
    of a rounding boundary the other way (about half of them), by one code, and only when
    asked; the oracle proper is unchanged."""
    cfg, W = _model("tiny_qwen2")
    a = oracle.OracleDecoder(W, 32)
    b = oracle.OracleDecoder(W, 32, quant_jitter=None, share_weights_with=a)
    c = oracle.OracleDecoder(W, 32, quant_jitter=7, share_weights_with=a)
    x = (np.random.default_rng(0).standard_normal((64, 256)) * 2).astype(F32)
    x[:, 0] = 127.0   # amax 127: x * 127 / amax is x itself
    x[:, 1] = 2.5     # an exact tie in every row
    qa, aa = a._quant(x)
    qb, ab = b._quant(x)
    assert np.array_equal(qa, qb) and np.array_equal(aa, ab)
    qc, ac = c._quant(x)
    assert np.array_equal(aa, ac)
    d = qc.astype(int) - qa.astype(int)
    assert np.abs(d).max() <= 1
    near = np.abs(x - np.floor(x) - 0.5) < oracle.decoder.NEAR_TIE_EPS[0]
    assert not d[~near].any()                       # nothing away from a tie moves
    assert 10 < int(np.abs(d[:, 1]).sum()) < 54     # about half of the exact ties move
    toks = [3, 1, 4, 1, 5]
    sa, sc = a.new_state(None), c.new_state(None)
    la, lc = a.prefill(sa, toks), c.prefill(sc, toks)
    assert np.abs(la - lc).max() < 0.05


def _scaled_permutation(rng_, n_out, n_in, perm, c):
    """int8 codes 127 at (n, perm[n]) for n < len(perm), zero elsewhere, with row scales c / 127:
    the projection computes y_n = c_n x_{perm[n]} exactly in real arithmetic."""
    w = np.zeros((n_out, n_in), np.int8)
    for n, k in enumerate(perm):
        w[n, k] = 127
    return w, (c.astype(np.float64) / 127.0).astype(F32)


def test_permutation_structured_whisper_w8a32_closed_form():
    """One W8A32 Whisper layer at position 0 whose v, o, xv, xo, fc1, fc2 are scaled
    permutations with a different scale on every row (q, k, xq, xk zero). With y = c * x[perm]
    for each of them and the encoder mean m_enc:
      x1 = x0 + c_o (c_v LN1(x0)[p_v] + b_v)[p_o] + b_o          (one cached row: weight 1)
      x2 = x1 + c_xo (c_xv m_enc[p_xv] + b_xv)[p_xo] + b_xo        (equal keys: uniform weights)
      x3 = x2 + c_2 gelu(c_1 LN3(x2)[p_1] + b_1)[p_2] + b_2
    Built from torch routines only. A row scale applied on the wrong axis or to the wrong row
    fails, since every permutation here moves every index."""
    cfg = synth.dataclasses.replace(synth.MODELS["tiny_whisper_w8a32"], n_layers=1)
    W = synth.make_weights(cfg, 5)
    W = _zero_projections(W)
    d, f = cfg.d_model, cfg.d_ff
    L = W["layers"][0]
    r = np.random.default_rng(9)
    perms, scales = {}, {}
    for key, (n_out, n_in) in {"v": (d, d), "o": (d, d), "xv": (d, d), "xo": (d, d), "fc1": (f, d),
                               "fc2": (d, f)}.items():
        m = min(n_out, n_in)
        perm = np.roll(np.arange(m), 1 + int(r.integers(0, m - 1)))   # a cyclic shift: no fixed point
        c = (0.5 + r.random(n_out)).astype(F32)
        L[key]["w"], L[key]["s"] = _scaled_permutation(r, n_out, n_in, perm[: min(n_out, m)], c)
        perms[key], scales[key] = perm, L[key]["s"].astype(np.float64) * 127.0
    dec = oracle.OracleDecoder(W, 16)
    enc = synth.encoder_hidden(cfg, 0, 5)
    st = dec.new_state(enc)
    tok = 31
    hidden, logits = dec.step([st], [tok], [0])
    T = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    ln = lambda x, g, b: torch.nn.functional.layer_norm(x, (d,), T(g), T(b), eps=float(F32(1e-5)))

    def P(key, x, n_out):
        y = torch.zeros(n_out, dtype=torch.float64)
        m = len(perms[key])
        y[:m] = T(scales[key][:m]) * x[torch.from_numpy(perms[key][:m])]
        return y

    x0 = T(W["tok_emb"][tok]) + T(W["pos_emb"][0])
    x1 = x0 + P("o", P("v", ln(x0, L["norm1_w"], L["norm1_b"]), d) + T(L["v"]["b"]), d) + T(L["o"]["b"])
    x2 = x1 + P("xo", P("xv", T(enc).mean(0), d) + T(L["xv"]["b"]), d) + T(L["xo"]["b"])
    g = torch.nn.functional.gelu(P("fc1", ln(x2, L["norm3_w"], L["norm3_b"]), f) + T(L["fc1"]["b"]),
                                 approximate="tanh")
    x3 = x2 + P("fc2", g, d) + T(L["fc2"]["b"])
    np.testing.assert_allclose(hidden[0], x3.numpy(), rtol=1e-5, atol=2e-6)
    ref = T(W["tok_emb"]) @ ln(x3, W["final_w"], W["final_b"])
    np.testing.assert_allclose(logits[0], ref.numpy(), rtol=1e-4, atol=1e-5)


def test_permutation_structured_qwen2_w8a8_closed_form():
    """One W8A8 Qwen2 layer at position 0 with q, k, v weights zero (every V row is b_v) and
    o, gate, up, down scaled permutations with a different scale on every row. With the
    pinned quantiser (q, a) = quant(.) and dequantised products acc * a * s:
      x1 = x0 + c_o dq(quant(b_v))[p_o]
      g = c_g dq(quant(h))[p_g], u = c_u dq(quant(h))[p_u] with h = RMS2(x1)
      x2 = x1 + c_d dq(quant(silu(g) u))[p_d]
    so each row scale, each permutation and the per-row activation scale are checked."""
    cfg = synth.dataclasses.replace(synth.MODELS["tiny_qwen2"], n_layers=1)
    W = synth.make_weights(cfg, 6)
    W = _zero_projections(W)
    d, f = cfg.d_model, cfg.d_ff
    L = W["layers"][0]
    r = np.random.default_rng(10)
    perms, cs = {}, {}
    for key, (n_out, n_in) in {"o": (d, d), "gate": (f, d), "up": (f, d), "down": (d, f)}.items():
        m = min(n_out, n_in)
        perm = np.roll(np.arange(m), 1 + int(r.integers(0, m - 1)))
        c = (0.5 + r.random(n_out)).astype(F32)
        L[key]["w"], L[key]["s"] = _scaled_permutation(r, n_out, n_in, perm, c)
        perms[key], cs[key] = perm, L[key]["s"]
    dec = oracle.OracleDecoder(W, 16)
    st = dec.new_state(None)
    tok = 5
    hidden, _ = dec.step([st], [tok], [0])

    def proj(key, x_row, n_out):
        """acc * a * s exactly as dequantised: acc_n = 127 q[perm[n]] (zero past the permutation)."""
        q, a = oracle.quantize_rows_i8_te(x_row[None, :])
        y = np.zeros(n_out, np.float64)
        m = len(perms[key])
        y[:m] = 127.0 * q[0, perms[key]].astype(np.float64) * float(a[0]) * cs[key][:m].astype(np.float64)
        return y.astype(F32)

    x0 = W["tok_emb"][tok]
    x1 = (x0 + proj("o", L["v"]["b"], d)).astype(F32)
    h = torch.nn.functional.rms_norm(torch.from_numpy(x1).double(), (d,), torch.from_numpy(L["norm2_w"]).double(),
                                     eps=float(F32(1e-6))).numpy().astype(F32)
    g = proj("gate", h, f)
    u = proj("up", h, f)
    m = (torch.nn.functional.silu(torch.from_numpy(g).double()).numpy().astype(F32) * u).astype(F32)
    x2 = (x1 + proj("down", m, d)).astype(F32)
    np.testing.assert_allclose(hidden[0], x2, rtol=1e-6, atol=1e-7)


def test_tie_log_and_flips():
    """The quantiser's tie bookkeeping: an activation within tie_eps of a rounding boundary is
    logged with its site, row, column and distance, and a flip rounds exactly that activation
    to the other neighbouring integer and changes nothing else."""
    cfg, W = _model("tiny_qwen2")
    dec = oracle.OracleDecoder(W, 8)
    x = np.array([[127.0, 2.5, 1.0, -3.4999], [127.0, 2.25, 1.0, 0.0]], F32)
    dec.tie_log, dec.tie_eps = [], {0: 1e-3}
    dec._site = 0
    q0, a0 = dec._quant(x)
    assert [(s, r, c) for s, r, c, _ in dec.tie_log] == [(0, 0, 1), (0, 0, 3)]
    dec.tie_log, dec.flips = None, {1: [(0, 1), (0, 3)]}
    dec._site = 1
    q1, a1 = dec._quant(x)
    assert np.array_equal(a0, a1)
    assert int(q1[0, 1]) == 3 and int(q0[0, 1]) == 2     # 2.5 rounds to even 2; flipped to 3
    assert int(q1[0, 3]) == -4 and int(q0[0, 3]) == -3   # -3.4999 rounds to -3; flipped to -4
    diff = q1.astype(int) != q0.astype(int)
    assert int(diff.sum()) == 2


@pytest.mark.parametrize("name", ["tiny_qwen2_gqa", "mid_qwen2_gqa"])
def test_grouped_query_attention_equals_mha_with_repeated_kv_heads(name):
    """Grouped-query attention (query head h reads K/V head h // group) is the multi-head
    decoder whose K and V projections repeat each K/V head's rows `group` times: same codes,
    scales and biases row for row, so every logit is the same bits. A wrong head mapping
    (h % H_kv instead of h // group) breaks it."""
    cfg_g, W = _model(name)
    cfg_m = synth.dataclasses.replace(cfg_g, n_kv_heads=0, name=name + "_as_mha")
    group = cfg_g.n_heads // cfg_g.kv_heads
    Wm = copy.deepcopy(W)
    Wm["config"] = cfg_m
    idx = np.concatenate([np.arange(h * 64, (h + 1) * 64) for h in range(cfg_g.kv_heads) for _ in range(group)])
    for L in Wm["layers"]:
        for key in ("k", "v"):
            p = L[key]
            L[key] = {"w": p["w"][idx], "s": p["s"][idx] if p["s"] is not None else None,
                      "b": p["b"][idx] if p["b"] is not None else None}
    toks = list(synth.token_ids(cfg_g, 0, 7))
    outs = []
    for Wx in (W, Wm):
        dec = oracle.OracleDecoder(Wx, 32)
        st = dec.new_state(None)
        lg = dec.prefill(st, toks)
        _, lg2 = dec.step([st], [5], [st.n])
        outs.append((lg, lg2))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])
    # the mapping matters: interleaved repetition (head h reads K/V head h % H_kv) differs
    idx_bad = np.concatenate([np.arange((h % cfg_g.kv_heads) * 64, (h % cfg_g.kv_heads + 1) * 64)
                              for h in range(cfg_g.n_heads)])
    Wb = copy.deepcopy(W)
    Wb["config"] = cfg_m
    for L, L0 in zip(Wb["layers"], W["layers"]):
        for key in ("k", "v"):
            p = L0[key]
            L[key] = {"w": p["w"][idx_bad], "s": p["s"][idx_bad], "b": p["b"][idx_bad]}
    dec = oracle.OracleDecoder(Wb, 32)
    st = dec.new_state(None)
    assert not np.array_equal(dec.prefill(st, toks), outs[0][0])
