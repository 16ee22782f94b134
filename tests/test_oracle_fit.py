"""Pins of the data-free VQ fit oracle (oracle/fit.py) against what the
mathematics fixes: planted maxima, exact-rational nearest centroids, exact
means, Lloyd's monotone objective and planted clusters. CPU only."""
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import fit


def _bf16(a):
    return synth.bf16_bits(np.asarray(a, dtype=np.float32))


def test_scales_are_planted_group_maxima():
    # every 64-weight group holds values below 0.25 in magnitude and one planted value of
    # magnitude m (bf16- and fp16-exact); one group is all zeros
    g = synth.rng(500)
    rows, cols = 5, 256
    w = g.uniform(-0.25, 0.25, size=(rows, cols)).astype(np.float32)
    planted = np.zeros((rows, cols // 64), dtype=np.float32)
    for r in range(rows):
        for q in range(cols // 64):
            m = np.float32(0.5 + 0.125 * g.integers(0, 12))
            pos = 64 * q + int(g.integers(0, 64))
            w[r, pos] = m if g.integers(0, 2) else -m
            planted[r, q] = m
    w[3, 64:128] = 0.0
    planted[3, 1] = 0.0
    sc = fit.fit_scales(_bf16(w))
    assert np.array_equal(sc, planted.astype(np.float16).view(np.uint16))
    v = fit.subvectors(_bf16(w), sc, 4)
    assert np.all(v.reshape(rows, cols)[3, 64:128] == 0)                 # zero group: v = 0
    assert np.abs(v).max() <= 1.0                                       # |w| <= group max


def test_nearest_is_exact_argmin_on_tiny_inputs():
    # brute force with exact rationals over fp32 inputs: the chosen centroid's exact distance
    # is the smallest, up to fp32 rounding of near-ties
    g = synth.rng(501)
    v = g.uniform(-1, 1, size=(60, 4)).astype(np.float32)
    c = g.uniform(-1, 1, size=(9, 4)).astype(np.float32)
    got = fit.nearest(v, c)
    for i in range(len(v)):
        exact = [sum((Fraction(float(v[i, t])) - Fraction(float(c[k, t]))) ** 2 for t in range(4))
                 for k in range(len(c))]
        best = min(exact)
        assert exact[got[i]] <= best * (1 + Fraction(1, 10 ** 5)) + Fraction(1, 10 ** 12)
        second = sorted(exact)[1]
        if second > best * (1 + Fraction(1, 10 ** 4)):
            assert got[i] == exact.index(best)


def test_ties_go_to_the_lower_index():
    c = np.array([[0.5, 0.5], [0.25, 0.0], [0.5, 0.5], [0.25, 0.0]], dtype=np.float32)
    v = np.array([[0.5, 0.5], [0.25, 0.0], [0.375, 0.25]], dtype=np.float32)
    # the third point is equally far (exactly) from entries 0 and 1
    assert list(fit.nearest(v, c)) == [0, 1, 0]


def test_lloyd_update_is_the_exact_mean():
    # points with few significant bits: the fixed-point sums are exact and the centroid is the
    # fp32 rounding of the exact rational mean; an empty cluster keeps its value
    g = synth.rng(502)
    v = (g.integers(-1024, 1025, size=(37, 4)) / 1024.0).astype(np.float32)
    c = np.array([[0, 0, 0, 0], [5, 5, 5, 5]], dtype=np.float32)   # all points go to entry 0
    new, a = fit.lloyd_step(v, c)
    assert np.all(a == 0)
    for t in range(4):
        mean = sum(Fraction(float(x)) for x in v[:, t]) / len(v)
        assert new[0, t] == np.float32(float(mean))
    assert np.array_equal(new[1], c[1])


def test_lloyd_objective_never_increases():
    g = synth.rng(503)
    w = synth.weights(64, 1024, g)
    sc = fit.fit_scales(w)
    v_all = fit.subvectors(w, sc, 4)
    sample, init = synth.fit_draw(len(v_all), 4096, 64, g)
    v = v_all[sample]
    c = v_all[init].copy()
    prev = fit.sse(v, c)
    for _ in range(12):
        c, _ = fit.lloyd_step(v, c)
        cur = fit.sse(v, c)
        assert cur <= prev * (1 + 1e-6)
        prev = cur


@pytest.mark.parametrize("d,K", [(2, 16), (4, 8), (8, 4)])
def test_fit_recovers_planted_clusters(d, K):
    # Every 64-weight group starts with one subvector equal to centre 0 = (1, 0, ..., 0), so the
    # group scale is exactly 1 and v = w. The other subvectors are centre label + small noise,
    # labels seeded per position: a mistake in the subvector layout, the assignment or the
    # update breaks codes == labels.
    g = synth.rng(504, d, K)
    rows, cols = 8, 256
    centres = np.zeros((K, d), dtype=np.float32)
    centres[0, 0] = 1.0
    centres[1:] = g.uniform(-0.75, 0.75, size=(K - 1, d)).astype(np.float32)
    n_per_row = cols // d
    labels = g.integers(1, K, size=(rows, n_per_row))
    labels[:, ::64 // d] = 0
    noise = g.uniform(-1e-3, 1e-3, size=(rows, n_per_row, d)).astype(np.float32)
    noise[labels == 0] = 0
    w = (centres[labels] + noise).reshape(rows, cols)
    wb = _bf16(w)
    assert np.all(fit.fit_scales(wb) == np.float16(1.0).view(np.uint16))
    flat = labels.reshape(-1)
    sample = np.arange(rows * n_per_row, dtype=np.int32)
    init = np.array([int(np.flatnonzero(flat == k)[0]) for k in range(K)], dtype=np.int32)
    sc, cb, codes, hist = fit.fit(wb, d, K, sample, init, iters=3)
    assert np.array_equal(codes, labels.astype(np.uint16))
    cbf = cb.view(np.float16).astype(np.float32)
    assert np.abs(cbf - centres).max() < 3e-3          # means of centre + noise, in fp16
    assert np.array_equal(hist[2], hist[3])            # converged: a further step changes nothing


def _f32_of_fraction(fr: Fraction) -> np.float32:
    """The fp32 number nearest the rational fr (ties to even), by exact integer arithmetic."""
    if fr == 0:
        return np.float32(0.0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()   # 2^e <= a < 2^(e+2)
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    q = max(e, -126) - 23                       # spacing of fp32 numbers near a
    n = a / (Fraction(2) ** q)
    fl = n.numerator // n.denominator
    rem = n - fl
    r = fl + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1) else 0)
    return np.float32(sign * float(Fraction(r) * Fraction(2) ** q))


def test_lloyd_update_is_the_exact_mean_on_realistic_points():
    # the points a real fit sees: bf16 N(0, 0.02) weights over their fp16 group maxima (F1), so full
    # fp32 significands and magnitudes down to the smallest bf16 weights of a group. Each centroid
    # the step moves must be the fp32 rounding (to nearest even) of the exact rational mean of its
    # points as they are, without any fixed-point rounding of the points before the sum.
    g = synth.rng(505)
    w = synth.weights(128, 1024, g)
    sc = fit.fit_scales(w)
    for d, K in ((4, 64), (2, 32), (8, 16)):
        v_all = fit.subvectors(w, sc, d)
        # every subvector with a component that is not a multiple of 2^-40 joins the sample
        v64 = v_all.astype(np.float64)
        fine = np.nonzero((np.rint(v64 * 2.0 ** 40) * 2.0 ** -40 != v64).any(axis=1))[0]
        assert len(fine) > 0
        sample = np.union1d(g.choice(v_all.shape[0], size=4096, replace=False), fine)
        v = v_all[sample]
        c = v[g.choice(len(v), size=K, replace=False)].copy()
        new, a = fit.lloyd_step(v, c)
        small = len(fine)
        for k in range(K):
            pts = v[a == k]
            if len(pts) == 0:
                assert np.array_equal(new[k], c[k])
                continue
            for t in range(d):
                exact = sum(Fraction(float(x)) for x in pts[:, t]) / len(pts)
                assert new[k, t] == _f32_of_fraction(exact), (d, K, k, t, small)
