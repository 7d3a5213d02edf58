"""Pins for the oracle's leaf operations (CPU only).

Each test checks the oracle against something other than itself: values the
pages print (tests/golden), closed forms, a library routine in f64 (torch CPU),
invariants, or brute force on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------- quantisation ----------------

def test_quant_golden_ties_even():
    g = _gold("quant_ties_even.json")
    for row in g["rows"]:
        q, a = oracle.quantize_rows_i8_te(np.array([row["x"]], dtype=F32))
        assert q[0].tolist() == row["q"]
        assert float(a[0]) == pytest.approx(row["a"], abs=0) or float(a[0]) == row["a"]
    # the half-away-from-zero reading is distinguishable on the first row
    q, _ = oracle.quantize_rows_i8_te(np.array([g["rows"][0]["x"]], dtype=F32))
    assert q[0].tolist() != g["half_away_from_zero_would_give"][0]


def test_quant_hand_value_non_power_of_two():
    # amax = 1 -> inv = 127 exactly; 0.5*127 = 63.5 (tie -> 64); -0.25*127 = -31.75 -> -32
    q, a = oracle.quantize_rows_i8_te(np.array([[1.0, 0.5, -0.25, 0.0]], dtype=F32))
    assert q[0].tolist() == [127, 64, -32, 0]
    assert a[0] == F32(1.0) / F32(127.0)


def test_quant_round_trip_and_error_bound():
    x = rng(1).standard_normal((64, 333)).astype(F32) * 3
    q, a = oracle.quantize_rows_i8_te(x)
    assert q.dtype == np.int8 and q.min() >= -127 and q.max() <= 127
    # the row max maps to +-127
    assert np.all(np.abs(q).max(axis=1) == 127)
    # dequantise then quantise again gives the same codes
    xr = oracle.dequantize_rows_i8(q, a)
    q2, a2 = oracle.quantize_rows_i8_te(xr)
    assert np.array_equal(q, q2)
    # reconstruction error at most half a step (plus f32 slack on the step itself)
    err = np.abs(xr.astype(np.float64) - x.astype(np.float64))
    assert np.all(err <= a.astype(np.float64)[:, None] * (0.5 + 1e-5) + 1e-30)


def test_quant_zero_row():
    q, a = oracle.quantize_rows_i8_te(np.zeros((2, 16), F32))
    assert not q.any() and not a.any()


def test_weight_quant_matches_offline_checkpoint_writer_and_bounds():
    w = rng(2).standard_normal((97, 131)).astype(F32) * F32(0.02)
    w[5] = 0.0
    q, s = oracle.quantize_weight_rows(w)
    q2, s2 = synth.quantize_weight_rows_offline(w)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)
    assert s[5] == 0 and not q[5].any()
    assert np.all(np.abs(q).max(axis=1)[s > 0] == 127)
    err = np.abs(q.astype(np.float64) * s[:, None] - w)
    assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 1e-5) + 1e-30)


def test_weight_quant_hand_values():
    w = np.array([[0.5, -1.0, 0.25], [2.54, 0.01, -1.27]], dtype=F32)
    q, s = oracle.quantize_weight_rows(w)
    assert s[0] == F32(1.0) / F32(127.0)
    # -1.0 / (1/127) = -127; 0.5 -> 63.5 -> 64 (even); 0.25 -> 31.75 -> 32
    assert q[0].tolist() == [64, -127, 32]
    assert s[1] == F32(2.54) / F32(127.0)
    assert q[1, 0] == 127 and q[1, 2] in (-63, -64)


def test_int8_dot_brute_force():
    r = rng(3)
    xq = r.integers(-127, 128, size=(3, 37)).astype(np.int8)
    wq = r.integers(-127, 128, size=(5, 37)).astype(np.int8)
    acc = oracle.int8_dot_acc(xq, wq)
    for m in range(3):
        for n in range(5):
            assert acc[m, n] == sum(int(xq[m, k]) * int(wq[n, k]) for k in range(37))
    # extreme magnitudes: 127*127*2816 stays exact
    big = np.full((1, 2816), 127, np.int8)
    assert oracle.int8_dot_acc(big, -big)[0, 0] == -127 * 127 * 2816


def test_w8a8_zero_activation_gives_bias_and_dequant_order():
    r = rng(4)
    wq = r.integers(-127, 128, size=(6, 16)).astype(np.int8)
    s = r.random(6).astype(F32) * F32(0.01)
    b = r.standard_normal(6).astype(F32)
    xq, a = oracle.quantize_rows_i8_te(np.zeros((1, 16), F32))
    y = oracle.linear_w8a8(xq, a, wq, s, b)
    assert np.array_equal(y[0], b)
    # nonzero: y = acc * a * s + b by brute force in Python floats
    x = r.standard_normal((2, 16)).astype(F32)
    xq, a = oracle.quantize_rows_i8_te(x)
    y = oracle.linear_w8a8(xq, a, wq, s, b)
    for m in range(2):
        for n in range(6):
            acc = sum(int(xq[m, k]) * int(wq[n, k]) for k in range(16))
            ref = acc * float(a[m]) * float(s[n]) + float(b[n])
            assert abs(float(y[m, n]) - ref) <= 1e-6 * max(1.0, abs(ref))


def test_w8a32_equals_dequantised_f32_linear():
    r = rng(5)
    w = r.standard_normal((33, 70)).astype(F32) * F32(0.02)
    q, s = oracle.quantize_weight_rows(w)
    x = r.standard_normal((4, 70)).astype(F32)
    b = r.standard_normal(33).astype(F32) * F32(0.01)
    wd = (q.astype(np.float64) * s[:, None]).astype(F32)
    np.testing.assert_allclose(oracle.linear_w8a32(x, q, s, b), oracle.linear_f32(x, wd, b),
                               rtol=1e-6, atol=1e-7)


def test_linear_golden_zero_weight_bias_only():
    g = _gold("linear_zero_weight.json")
    y = oracle.linear_f32(np.array([g["x"]], F32), np.array(g["w"], F32), np.array(g["b"], F32))
    assert y[0].tolist() == g["y"]


def test_linear_brute_force():
    r = rng(6)
    x = r.standard_normal((2, 9)).astype(F32)
    w = r.standard_normal((4, 9)).astype(F32)
    b = r.standard_normal(4).astype(F32)
    y = oracle.linear_f32(x, w, b)
    for m in range(2):
        for n in range(4):
            ref = math.fsum(float(x[m, k]) * float(w[n, k]) for k in range(9)) + float(b[n])
            assert float(y[m, n]) == float(F32(ref))


# ---------------- norms ----------------

def test_layer_norm_constant_row_gives_beta():
    g = rng(7).standard_normal(64).astype(F32)
    b = rng(8).standard_normal(64).astype(F32)
    y = oracle.layer_norm(np.full((1, 64), 3.25, F32), g, b, 1e-5)
    np.testing.assert_array_equal(y[0], b)


def test_layer_norm_matches_torch_f64():
    r = rng(9)
    x = r.standard_normal((5, 384)).astype(F32) * 2 + 1
    g = (1 + 0.02 * r.standard_normal(384)).astype(F32)
    b = (0.01 * r.standard_normal(384)).astype(F32)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (384,),
                                         torch.from_numpy(g).double(), torch.from_numpy(b).double(),
                                         eps=float(F32(1e-5))).numpy()
    np.testing.assert_allclose(oracle.layer_norm(x, g, b, 1e-5), ref, rtol=1e-6, atol=1e-6)


def test_rms_norm_closed_form_and_torch():
    # x = [3, 4]: mean(x^2) = 12.5 -> y = x / sqrt(12.5 + eps)
    y = oracle.rms_norm(np.array([[3.0, 4.0]], F32), np.ones(2, F32), 0.0)
    np.testing.assert_allclose(y[0], [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=1e-7)
    r = rng(10)
    x = r.standard_normal((4, 1024)).astype(F32)
    w = (1 + 0.02 * r.standard_normal(1024)).astype(F32)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x).double(), (1024,),
                                       torch.from_numpy(w).double(), eps=float(F32(1e-6))).numpy()
    np.testing.assert_allclose(oracle.rms_norm(x, w, 1e-6), ref, rtol=1e-6, atol=1e-7)


# ---------------- RoPE ----------------

def test_rope_identity_at_pos0_and_norm_preserving():
    x = rng(11).standard_normal((16, 64)).astype(F32)
    c, s = oracle.rope_cos_sin(0, 1e6)
    np.testing.assert_array_equal(oracle.apply_rope_neox(x, c, s), x)
    for pos in (1, 7, 1023, 4095):
        c, s = oracle.rope_cos_sin(pos, 1e6)
        y = oracle.apply_rope_neox(x, c, s)
        np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-6)


def test_rope_closed_form_one_hot():
    # e_0 at pos 1: frequency theta^0 = 1, so the angle is 1 rad and the pair is (0, 32)
    x = np.zeros((1, 64), F32)
    x[0, 0] = 1.0
    c, s = oracle.rope_cos_sin(1, 1e6)
    y = oracle.apply_rope_neox(x, c, s)
    assert y[0, 0] == F32(math.cos(1.0)) and y[0, 32] == F32(math.sin(1.0))
    assert np.count_nonzero(y) == 2
    # e_33 (second half of pair 1) at pos 5: angle = 5 * theta^(-2/64)
    x = np.zeros((1, 64), F32)
    x[0, 33] = 1.0
    ang = 5 * 1e6 ** (-2 / 64)
    c, s = oracle.rope_cos_sin(5, 1e6)
    y = oracle.apply_rope_neox(x, c, s)
    assert y[0, 1] == pytest.approx(-math.sin(ang), rel=1e-6)
    assert y[0, 33] == pytest.approx(math.cos(ang), rel=1e-6)


def test_rope_equals_complex_rotation():
    r = rng(12)
    x = r.standard_normal((4, 64)).astype(F32)
    pos = 321
    c, s = oracle.rope_cos_sin(pos, 1e6)
    y = oracle.apply_rope_neox(x, c, s)
    z = (x[:, :32].astype(np.float64) + 1j * x[:, 32:].astype(np.float64)) * (c + 1j * s.astype(np.float64))
    np.testing.assert_allclose(y[:, :32], z.real, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(y[:, 32:], z.imag, rtol=1e-6, atol=1e-6)


def test_rope_interleaved_pairing_mutation_is_detected():
    # the same rotation applied to interleaved pairs (2i, 2i+1) moves the result by O(0.1-1)
    r = rng(13)
    x = (np.arange(64, dtype=F32) + 1) * F32(0.07)
    x = x[None, :]
    pos = 3
    c, s = oracle.rope_cos_sin(pos, 1e4)
    y = oracle.apply_rope_neox(x, c, s)
    x0, x1 = x[0, 0::2].astype(np.float64), x[0, 1::2].astype(np.float64)
    inter = np.empty(64)
    inter[0::2] = x0 * c - x1 * s
    inter[1::2] = x0 * s + x1 * c
    assert np.max(np.abs(inter - y[0])) > 0.1


# ---------------- attention / softmax ----------------

def test_softmax_sums_to_one_and_fails_closed():
    r = rng(14)
    for n in (1, 2, 31, 1500, 4129):
        p = oracle.softmax_weights(r.standard_normal(n) * 10)
        assert abs(p.sum() - 1.0) < 1e-6 and np.all(p >= 0)
    assert oracle.softmax_weights(np.array([5.0]))[0] == 1.0
    bad = np.array([1.0, np.nan, 2.0])
    assert np.array_equal(oracle.softmax_weights(bad), np.zeros(3))
    assert np.array_equal(oracle.softmax_weights(np.array([np.inf, 1.0])), np.zeros(2))


def test_attention_golden_single_key():
    g = _gold("attention_single_key.json")
    out = oracle.attention_decode(np.array(g["q"], F32), np.array(g["k"], F32), np.array(g["v"], F32))
    assert out.tolist() == g["out"]


def test_attention_identical_keys_give_mean_of_v():
    r = rng(15)
    n, H = 9, 3
    k = np.repeat(r.standard_normal((1, H, 64)).astype(F32), n, axis=0)
    v = r.standard_normal((n, H, 64)).astype(F32)
    q = r.standard_normal((H, 64)).astype(F32)
    out = oracle.attention_decode(q, k, v)
    np.testing.assert_allclose(out, v.astype(np.float64).mean(axis=0), rtol=1e-6, atol=1e-7)


def test_attention_matches_torch_sdpa_f64():
    r = rng(16)
    n, H = 300, 4
    q = r.standard_normal((H, 64)).astype(F32)
    k = r.standard_normal((n, H, 64)).astype(F32)
    v = r.standard_normal((n, H, 64)).astype(F32)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double()[:, None, :], torch.from_numpy(k).double().transpose(0, 1),
        torch.from_numpy(v).double().transpose(0, 1))[:, 0, :].numpy()
    np.testing.assert_allclose(oracle.attention_decode(q, k, v), ref, rtol=1e-6, atol=1e-7)


# ---------------- activations / argmax ----------------

def test_gelu_tanh_matches_torch_and_closed_forms():
    x = np.linspace(-8, 8, 2001).astype(F32)
    ref = torch.nn.functional.gelu(torch.from_numpy(x).double(), approximate="tanh").numpy()
    np.testing.assert_allclose(oracle.gelu_tanh(x), ref, rtol=1e-6, atol=1e-7)
    assert oracle.gelu_tanh(np.array([0.0], F32))[0] == 0.0
    # gelu(x) - gelu(-x) = x for the tanh form (odd tanh)
    np.testing.assert_allclose(oracle.gelu_tanh(x) - oracle.gelu_tanh(-x), x, rtol=1e-6, atol=1e-6)


def test_silu_matches_torch():
    x = np.linspace(-20, 20, 801).astype(F32)
    ref = torch.nn.functional.silu(torch.from_numpy(x).double()).numpy()
    np.testing.assert_allclose(oracle.silu(x), ref, rtol=1e-6, atol=1e-7)


def test_argmax_golden_first_max():
    g = _gold("argmax_first_max.json")
    for case in g["cases"]:
        row = np.array([float(v) for v in case["row"]], F32)
        assert oracle.argmax_first(row) == case["argmax"]


def test_w8a32_brute_force_with_distinct_row_scales():
    """y_n = s_n * sum_k q_nk x_k + b_n with a different scale on every output row: a
    scale taken from the wrong row or applied along the input axis fails."""
    r = rng(12)
    q = r.integers(-127, 128, size=(5, 11)).astype(np.int8)
    s = (r.random(5) + 0.5).astype(F32) * F32(0.01)
    b = r.standard_normal(5).astype(F32)
    x = r.standard_normal((3, 11)).astype(F32)
    y = oracle.linear_w8a32(x, q, s, b)
    for m in range(3):
        for n in range(5):
            ref = float(s[n]) * math.fsum(int(q[n, k]) * float(x[m, k]) for k in range(11)) + float(b[n])
            assert abs(float(y[m, n]) - ref) <= 1e-6 * max(1.0, abs(ref))


def test_linear_with_cached_f64_weights_is_the_same_function():
    """The decoder passes each matrix's f64 copy (converted once); the result is the same bits."""
    r = rng(13)
    w = r.standard_normal((7, 19)).astype(F32)
    q = r.integers(-127, 128, size=(7, 19)).astype(np.int8)
    s = r.random(7).astype(F32)
    b = r.standard_normal(7).astype(F32)
    x = r.standard_normal((2, 19)).astype(F32)
    xq, a = oracle.quantize_rows_i8_te(x)
    assert np.array_equal(oracle.linear_f32(x, w, b), oracle.linear_f32(x, w, b, w64=w.astype(np.float64)))
    assert np.array_equal(oracle.linear_w8a32(x, q, s, b), oracle.linear_w8a32(x, q, s, b, w64=q.astype(np.float64)))
    assert np.array_equal(oracle.linear_w8a8(xq, a, q, s, b), oracle.linear_w8a8(xq, a, q, s, b, w64=q.astype(np.float64)))
    assert np.array_equal(oracle.int8_dot_acc(xq, q), oracle.int8_dot_acc(xq, q, w64=q.astype(np.float64)))
