"""Numerics of the TF32 tensor-core projections (CPU property checks).

Batches of 8 or more run larger f32 projections on TF32 tensor cores with split operands:
x = x_hi + x_lo and w = w_hi + w_lo (each part rounded to TF32, 10 explicit mantissa bits,
round to nearest with ties away from zero as cvt.rna does), products
x_hi w_hi + x_lo w_hi + x_hi w_lo accumulated in f32 (int8 weights are exact in TF32 and need
only the two x terms). These tests restate the split in numpy and check that one such dot
product lies within a few f32 ulps of the exact one, far inside the 2e-3 parity tolerance,
and that dropping a kept term is detected.
"""
import numpy as np

F = np.float32


def tf32(v: np.ndarray) -> np.ndarray:
    """Round f32 to TF32 (keep 10 mantissa bits), nearest with ties away from zero."""
    b = np.asarray(v, F).view(np.uint32).astype(np.uint64)
    b = (b + 0x1000) & 0xFFFFE000   # add half an ulp of the kept part to the magnitude, truncate
    return b.astype(np.uint32).view(F)


def split(v):
    hi = tf32(v)
    lo = tf32((np.asarray(v, F) - hi).astype(F))
    return hi, lo


def dot_3xtf32(w, x, int8_weights=False):
    xh, xl = split(x)
    if int8_weights:
        terms = [w.astype(np.float64) * xl, w.astype(np.float64) * xh]
    else:
        wh, wl = split(w)
        terms = [wh.astype(np.float64) * xl, wl.astype(np.float64) * xh, wh.astype(np.float64) * xh]
    # products of TF32 values are exact in f32's accumulator width; accumulate in f32
    acc = F(0.0)
    for k in range(len(x)):
        for t in terms:
            acc = F(acc + F(t[k]))
    return acc


def test_tf32_rounding_keeps_ten_bits():
    v = np.array([1.0 + 2.0 ** -10, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -12, -1.0 - 2.0 ** -11], F)
    got = tf32(v)
    assert got[0] == F(1.0 + 2.0 ** -10)          # representable
    assert got[1] == F(1.0 + 2.0 ** -10)          # tie, away from zero
    assert got[2] == F(1.0 + 2.0 ** -10)          # rounds up
    assert got[3] == F(-1.0 - 2.0 ** -10)         # tie away from zero on the negative side


def test_split_dot_within_f32_accuracy():
    rng = np.random.default_rng(3)
    for k in (64, 512, 2048):
        for int8_weights in (False, True):
            w = (np.rint(rng.standard_normal(k) * 40).clip(-127, 127).astype(F) if int8_weights
                 else (rng.standard_normal(k) * 0.05).astype(F))
            x = rng.standard_normal(k).astype(F)
            exact = float(np.dot(w.astype(np.float64), x.astype(np.float64)))
            got = float(dot_3xtf32(w, x, int8_weights))
            scale = float(np.sum(np.abs(w.astype(np.float64) * x)))
            assert abs(got - exact) <= 2.0 ** -20 * scale + 1e-30, (k, int8_weights, got, exact)
            assert abs(got - exact) <= 2e-3


def test_dropping_the_lo_term_is_detected():
    rng = np.random.default_rng(4)
    w = (rng.standard_normal(512) * 0.05).astype(F)
    x = rng.standard_normal(512).astype(F)
    exact = float(np.dot(w.astype(np.float64), x.astype(np.float64)))
    xh, _ = split(x)
    wh, _ = split(w)
    one_term = float(np.dot(wh.astype(np.float64), xh.astype(np.float64)))
    good = float(dot_3xtf32(w, x))
    assert abs(one_term - exact) > 20 * abs(good - exact)
