"""Numerics of the tied head's exact-integer product (CPU property checks).

The head writes each f32 row r (embedding rows once, hidden rows per step) with a row scale
s_r = amax_r / 127 as three base-254 int8 digits, v ~ s_r (d1 + d2/254 + d3/254^2), sums the
six digit products of weight >= 254^-2 exactly in int32, and combines them as
s_n s_b (A0 + (A1 + A2/254)/254) in f32 (the splitting idea of Ozaki et al. 2012 and Ootomo,
Ozaki, Yokota 2024, truncated to f32 accuracy). These tests restate that arithmetic in numpy
with f32 rounding at the same points and check the bounds the design relies on: the digit
representation error is below 2^-22 amax per element, the digits stay in [-127, 127], the
int32 sums cannot overflow for K <= 4096, and the logits are within a few f32 ulps of the
exact f64 dot product -- far inside the 2e-3 parity tolerance.
"""
import numpy as np
import pytest

F = np.float32


def digits3(row: np.ndarray):
    """Three base-254 digits of a row with f32 arithmetic: (d1, d2, d3, scale)."""
    row = row.astype(F)
    amax = F(np.max(np.abs(row)))
    inv = F(F(127.0) / amax) if amax > 0 else F(0.0)
    r0 = (row * inv).astype(F)
    e1 = np.clip(np.rint(r0), -127, 127).astype(F)
    r1 = ((r0 - e1).astype(F) * F(254.0)).astype(F)
    e2 = np.clip(np.rint(r1), -127, 127).astype(F)
    r2 = ((r1 - e2).astype(F) * F(254.0)).astype(F)
    e3 = np.clip(np.rint(r2), -127, 127).astype(F)
    return e1.astype(np.int64), e2.astype(np.int64), e3.astype(np.int64), F(amax / F(127.0))


def reconstruct(d1, d2, d3, s):
    return s.astype(np.float64) * (d1 + d2 / 254.0 + d3 / 254.0 ** 2)


def head_logit(w: np.ndarray, x: np.ndarray) -> np.float32:
    """One logit the way the tensor-core head forms it."""
    D1, D2, D3, sw = digits3(w)
    E1, E2, E3, sx = digits3(x)
    a0 = int(np.dot(D1, E1))
    a1 = int(np.dot(D1, E2) + np.dot(D2, E1))
    a2 = int(np.dot(D1, E3) + np.dot(D2, E2) + np.dot(D3, E1))
    for a in (a0, a1, a2):
        assert -2 ** 31 <= a < 2 ** 31
    u = F(F(a1) + F(F(a2) * F(1.0 / 254.0)))
    t = F(F(a0) + F(u * F(1.0 / 254.0)))
    return F(F(sw * sx) * t)


def _rows(rng, k, kind):
    if kind == "normal":
        return rng.standard_normal(k).astype(F)
    if kind == "outlier":  # one large element: small elements keep only absolute accuracy
        r = (rng.standard_normal(k) * 0.02).astype(F)
        r[rng.integers(k)] = F(50.0)
        return r
    if kind == "tiny":
        return (rng.standard_normal(k) * 1e-30).astype(F)
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["normal", "outlier", "tiny"])
def test_digit_representation_error_below_2_pow_minus_22_amax(kind):
    rng = np.random.default_rng([7, len(kind)])
    for k in (64, 384, 1280):
        row = _rows(rng, k, kind)
        d1, d2, d3, s = digits3(row)
        for d in (d1, d2, d3):
            assert np.all(np.abs(d) <= 127)
        amax = float(np.max(np.abs(row)))
        err = np.max(np.abs(reconstruct(d1, d2, d3, s) - row.astype(np.float64)))
        assert err <= 2.0 ** -22 * amax, (kind, k, err / amax)


def test_zero_row_gives_zero_digits_and_scale():
    d1, d2, d3, s = digits3(np.zeros(256, F))
    assert s == 0 and not d1.any() and not d2.any() and not d3.any()


def test_int32_sums_cannot_overflow_up_to_k_4096():
    # the largest accumulator sums three products of two digits of magnitude <= 127
    assert 3 * 127 * 127 * 4096 < 2 ** 31


@pytest.mark.parametrize("kind", ["normal", "outlier"])
def test_head_logits_match_exact_dot_product(kind):
    rng = np.random.default_rng([11, len(kind)])
    for k in (384, 512, 1024, 1280):
        for _ in range(20):
            w = (_rows(rng, k, kind) * F(0.02)).astype(F)   # embedding-like scale
            x = _rows(rng, k, "normal")
            exact = float(np.dot(w.astype(np.float64), x.astype(np.float64)))
            got = float(head_logit(w, x))
            # f32 rounding of the combination plus the representation errors of both rows
            bound = 4 * 2.0 ** -24 * abs(exact) + 2.0 ** -21 * (
                np.max(np.abs(w)) * np.sum(np.abs(x)) + np.max(np.abs(x)) * np.sum(np.abs(w)))
            assert abs(got - exact) <= bound, (kind, k, got, exact, bound)
            assert abs(got - exact) <= 2e-3   # far inside the logits' parity tolerance


def test_dropping_a_kept_product_is_detected():
    """A plausible slip (dropping D2 E2 from A2) breaks the bound on a normal row pair."""
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(1024) * 0.02).astype(F)
    x = rng.standard_normal(1024).astype(F)
    D1, D2, D3, sw = digits3(w)
    E1, E2, E3, sx = digits3(x)
    a0 = int(np.dot(D1, E1))
    a1 = int(np.dot(D1, E2) + np.dot(D2, E1))
    a2_bad = int(np.dot(D1, E3) + np.dot(D3, E1))
    bad = float(sw) * float(sx) * (a0 + (a1 + a2_bad / 254.0) / 254.0)
    exact = float(np.dot(w.astype(np.float64), x.astype(np.float64)))
    good = float(head_logit(w, x))
    assert abs(bad - exact) > 20 * abs(good - exact) + 1e-9


def coarse_logit(w: np.ndarray, x: np.ndarray) -> np.float32:
    """The int8 head's coarse logit: only the embedding row's first digit (its per-row int8
    quantisation) against the hidden row's three digits, combined like head_logit."""
    D1, _, _, sw = digits3(w)
    E1, E2, E3, sx = digits3(x)
    a0, a1, a2 = int(np.dot(D1, E1)), int(np.dot(D1, E2)), int(np.dot(D1, E3))
    u = F(F(a1) + F(F(a2) * F(1.0 / 254.0)))
    t = F(F(a0) + F(u * F(1.0 / 254.0)))
    return F(F(sw * sx) * t)


def int8_head_bound(w, x, coarse, c1=0.502, c2=0.002):
    """The kernel's bound on |exact head - coarse|: s_n s_b (c1 S1 + c2 S2) * 1.001 plus a few
    ulps of the coarse logit, with S1 = sum |E1|, S2 = sum |E2| of the hidden row's digits."""
    _, _, _, sw = digits3(w)
    E1, E2, _, sx = digits3(x)
    b = float(F(sw * sx)) * (c1 * float(np.abs(E1).sum()) + c2 * float(np.abs(E2).sum()))
    return b * 1.001 + 4e-6 * abs(float(coarse)) + 1e-30


@pytest.mark.parametrize("kind", ["normal", "outlier"])
def test_int8_head_bound_holds(kind):
    """Every exact-head logit lies within the bound of its coarse logit, so the candidates
    (coarse + bound >= the row's largest coarse - bound) contain the exact argmax."""
    rng = np.random.default_rng([13, len(kind)])
    worst = 0.0
    for k in (384, 1024, 1280):
        for _ in range(40):
            w = (_rows(rng, k, kind) * F(0.02)).astype(F)
            x = _rows(rng, k, "normal")
            c = coarse_logit(w, x)
            e = head_logit(w, x)
            bnd = int8_head_bound(w, x, c)
            assert abs(float(e) - float(c)) <= bnd, (kind, k, e, c, bnd)
            worst = max(worst, abs(float(e) - float(c)) / bnd)
    assert worst > 0.01   # the bound is not vacuous by orders of magnitude


def test_int8_head_without_the_bound_misses():
    """Mutation: taking the coarse logits as exact (no bound) is wrong on ordinary rows, so the
    re-score is needed; the bound itself holds on the same rows."""
    rng = np.random.default_rng(17)
    misses = 0
    for _ in range(200):
        w = (rng.standard_normal(64) * 0.02).astype(F)
        w[0] = F(0.08)   # a large element: coarse digits round away much of the small ones
        x = rng.standard_normal(64).astype(F)
        c = coarse_logit(w, x)
        err = abs(float(head_logit(w, x)) - float(c))
        assert err <= int8_head_bound(w, x, c)
        if err > int8_head_bound(w, x, c, c1=0.0, c2=0.0):
            misses += 1
    assert misses > 0


def test_int8_head_candidates_contain_the_argmax():
    """On a small vocabulary, the candidate rule keeps the exact head's argmax and few others."""
    rng = np.random.default_rng(19)
    V, k = 2000, 256
    E = (rng.standard_normal((V, k)) * 0.02).astype(F)
    x = rng.standard_normal(k).astype(F)
    exact = np.array([head_logit(E[n], x) for n in range(V)], np.float64)
    coarse = np.array([coarse_logit(E[n], x) for n in range(V)], np.float64)
    bound = np.array([int8_head_bound(E[n], x, coarse[n]) for n in range(V)])
    thr = np.max(coarse - bound)
    cand = np.nonzero(coarse + bound >= thr)[0]
    assert int(np.argmax(exact)) in set(cand.tolist())
    assert len(cand) < V // 10
