"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- closed forms, library routines, hand-worked fixtures, brute force
on tiny inputs, or invariants -- chosen so that a dropped term, a wrong sign or
index, or a transposed operand fails at least one of them."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------- number formats

def test_f16_decode_exhaustive(oracle_lib):
    # library routine: numpy's IEEE binary16 decoder, all 65536 patterns
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle_lib.f16_to_f64(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_decode_exhaustive(oracle_lib):
    # library routine: a bf16 pattern is the top half of an fp32 pattern
    bits = np.arange(65536, dtype=np.uint32)
    ref = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = oracle_lib.bf16_to_f64(bits.astype(np.uint16))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_round_nearest_even(oracle_lib):
    # library routine: torch's fp32 -> bf16 conversion is round-to-nearest-even;
    # fp32 inputs are exact doubles, so one rounding happens on both sides.
    g = np.random.default_rng(5)
    v = np.concatenate([
        g.standard_normal(2000).astype(np.float32),
        (g.standard_normal(500) * 1e-39).astype(np.float32),          # bf16 subnormals
        (g.standard_normal(500) * 3e38).astype(np.float32),            # near overflow
        np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, -(1.0 + 2**-8), 2**-133, 3 * 2**-134,
                  3.3895314e38, 0.0, -0.0], dtype=np.float32),         # ties and edges
    ])
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle_lib.f64_to_bf16(v.astype(np.float64))
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ packing

def _golden_pack_cases():
    cases = []
    with open(os.path.join(GOLDEN, "pack_lsb_first.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, ncode, codes, words = [s.strip() for s in line.split("|")]
            c = np.zeros(int(ncode), dtype=np.uint16)
            for kv in codes.split():
                j, v = kv.split(":")
                c[int(j)] = int(v)
            w = np.array([int(h, 16) for h in words.split()], dtype=np.uint32)
            cases.append((int(bits), c, w))
    return cases


@pytest.mark.parametrize("case", range(5))
def test_pack_golden(oracle_lib, case):
    bits, codes, words = _golden_pack_cases()[case]
    got = oracle_lib.pack(codes[None, :], bits)
    assert got.shape == (1, len(words))
    assert np.array_equal(got[0], words)
    assert np.array_equal(oracle_lib.unpack_row(words, len(codes), bits), codes)


def test_pack_rows_are_row_local(oracle_lib):
    # a second row restarts at its own word 0 (row-local packing)
    c = np.zeros((2, 32), dtype=np.uint16)
    c[1, 0] = 1
    got = oracle_lib.pack(c, 3)
    assert got.shape == (2, 3)
    assert got[1, 0] == 1 and got[0].sum() == 0


@pytest.mark.parametrize("bits", list(range(1, 17)))
def test_pack_roundtrip_and_size(oracle_lib, bits):
    g = synth.rng(11, bits)
    rows, ncode = 5, 96
    codes = synth.raw_codes((rows, ncode), bits, g)
    codes[0, :] = (1 << bits) - 1          # all-ones codes
    codes[1, :] = 0
    packed = oracle_lib.pack(codes, bits)
    # closed form: 32 codes of b bits are exactly b words
    assert packed.shape == (rows, ncode // 32 * bits)
    assert np.array_equal(oracle_lib.unpack(packed, ncode, bits), codes)
    # all-ones codes fill every bit of their row
    assert np.all(packed[0] == 0xFFFFFFFF)


@pytest.mark.parametrize("d,K,bpw", [(4, 256, 2.25), (4, 512, 2.5), (2, 2048, 5.75), (2, 256, 4.25)])
def test_bits_per_weight_closed_form(oracle_lib, d, K, bpw):
    # 2.25 bpw: d=4, K=256 (Qwen3.5-397B-A17B-VQ-2.4bpw card, "Methodology")
    # 2.5 bpw: d=4, K=512 (Qwen3.5-397B-A17B-VQ-2.6bpw card, "Methodology")
    # 5.75 bpw: d=2, K=2048 (gemma-4-26b-a4b-it-VQ-6.2bpw card, "How it was built")
    # 4.25 bpw: d=2, K=256 with a 64-group fp16 scale (the single-GEMV workload)
    bits = int(math.log2(K))
    rows, cols = 8, 512
    g = synth.rng(3)
    codes = synth.raw_codes((rows, cols // d), bits, g)
    packed = oracle_lib.pack(codes, bits)
    scale_bytes = rows * (cols // 64) * 2
    measured = (packed.nbytes + scale_bytes) * 8 / (rows * cols)
    assert measured == bpw
    # codebook doubling at d=4 costs +0.25 bpw (gemma card, "How it was built")
    assert bits / d + 0.25 == bpw


def test_skipzero_pack_keeps_live_rows_byte_identical(oracle_lib):
    # vq-skipzero (Qwen3.5-397B-A17B-VQ-2.4bpw card, "Changelog 2026-10-01"):
    # dropping dead rows leaves the live rows' bytes unchanged.
    g = synth.rng(7)
    E, rows, ncode, bits = 3, 70, 64, 10
    codes = synth.raw_codes((E, rows, ncode), bits, g)
    bm = synth.live_bitmap(E, rows, 9, g)
    full = oracle_lib.pack(codes, bits)
    sz = oracle_lib.pack(codes, bits, bm)
    live = np.array([(bm[e, r // 32] >> (r % 32)) & 1 for e in range(E) for r in range(rows)], dtype=bool)
    assert sz.shape[0] == E * (rows - 9)
    assert np.array_equal(sz, full[live])


# ------------------------------------------------------------------ dequant

def _module(oracle_lib, codes, bits, d, codebook, scales, bitmap=None):
    E, rows, ncode = codes.shape
    words = oracle_lib.pack(codes, bits, bitmap)
    sc = oracle_lib.compact_rows(scales, bitmap)
    return oracle_lib.Module(E, rows, ncode * d, d, bits, words, sc, codebook, bitmap)


def test_dequant_d1_affine(oracle_lib):
    # d=1, K=8 (3-bit, group 64: the affine fall-through geometry of the
    # Qwen3.5-397B-A17B-VQ-2.4bpw card, "2026-09-20 correction"): a codebook
    # c_q = q - z turns VQ dequant into affine dequant s*q + bias, bias = -s*z.
    g = synth.rng(21)
    rows, cols, bits, z = 6, 192, 3, 4
    q = synth.raw_codes((1, rows, cols), bits, g)
    cb = synth.f16_bits(np.arange(8, dtype=np.float32) - z).reshape(8, 1)
    s_bits = synth.scales(rows, cols // 64, g)
    m = _module(oracle_lib, q, bits, 1, cb, s_bits[None])
    W = oracle_lib.dequant(m, 0)
    s = s_bits.view(np.float16).astype(np.float64)
    s_full = np.repeat(s, 64, axis=1)
    affine = s_full * q[0].astype(np.float64) + (-s_full * z)
    assert np.array_equal(W, affine)


def _golden_affine_cases():
    rows = []
    with open(os.path.join(os.path.dirname(__file__), "golden", "affine_3bit_group64.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            sc, b, ws = (x.strip() for x in line.split("|"))
            rows.append((float(sc), float(b), [float(v) for v in ws.split()]))
    return rows


def test_dequant_affine_biases_golden(oracle_lib):
    # one row per fixture line: its 64 weights cycle q = 0..7 in group 0 (scale and bias of the line);
    # a second group of each row checks that the bias is taken per group
    cases = _golden_affine_cases()
    assert len(cases) == 4
    rows, cols, bits = len(cases), 128, 3
    q = np.tile(np.arange(8, dtype=np.uint16), cols // 8)[None, None, :].repeat(rows, axis=1)
    cb = synth.f16_bits(np.arange(8, dtype=np.float32)).reshape(8, 1)           # identity codebook
    sc = synth.f16_bits(np.array([[c[0], 1.0] for c in cases], dtype=np.float32))
    bi = synth.f16_bits(np.array([[c[1], 0.0] for c in cases], dtype=np.float32))
    m = _module(oracle_lib, q, bits, 1, cb, sc[None])
    m.biases = bi
    W = oracle_lib.dequant(m, 0)
    for r, (_, _, want) in enumerate(cases):
        assert list(W[r, :8]) == want and list(W[r, 56:64]) == want
        assert list(W[r, 64:72]) == [float(v) for v in range(8)]                # group 1: s = 1, b = 0


def test_dequant_affine_biases_equal_zero_point_form(oracle_lib):
    # with b = -s * z (exact in fp16) the biased identity codebook equals the zero-point codebook
    # c_q = q - z without biases, the form pinned by test_dequant_d1_affine
    g = synth.rng(24)
    rows, cols, bits, z = 5, 192, 3, 3
    q = synth.raw_codes((1, rows, cols), bits, g)
    s_bits = synth.f16_bits(2.0 ** g.integers(-6, 2, size=(rows, cols // 64)).astype(np.float32))
    s = s_bits.view(np.float16).astype(np.float32)
    ident = synth.f16_bits(np.arange(8, dtype=np.float32)).reshape(8, 1)
    zp = synth.f16_bits(np.arange(8, dtype=np.float32) - z).reshape(8, 1)
    m_b = _module(oracle_lib, q, bits, 1, ident, s_bits[None])
    m_b.biases = synth.f16_bits(-s * z)
    m_z = _module(oracle_lib, q, bits, 1, zp, s_bits[None])
    assert np.array_equal(oracle_lib.dequant(m_b, 0), oracle_lib.dequant(m_z, 0))


def test_affine_biases_dead_rows_and_gemv_linearity(oracle_lib):
    # dead rows stay exactly zero with biases; the GEMV of a biased module is the unbiased GEMV
    # plus b times each group's activation sum (linearity of the dot product)
    g = synth.rng(25)
    E, rows, cols, bits = 2, 40, 192, 3
    q = synth.raw_codes((E, rows, cols), bits, g)
    bm = synth.live_bitmap(E, rows, 6, g)
    cb = synth.f16_bits(np.arange(8, dtype=np.float32)).reshape(8, 1)
    sc = synth.scales(E * rows, cols // 64, g).reshape(E, rows, cols // 64)
    m0 = _module(oracle_lib, q, bits, 1, cb, sc, bm)
    m1 = _module(oracle_lib, q, bits, 1, cb, sc, bm)
    b = synth.f16_bits(g.normal(0, 0.5, size=(len(m1.scales), cols // 64)))
    m1.biases = b
    W1 = oracle_lib.dequant(m1, 1)
    dead = [r for r in range(rows) if not (bm[1, r // 32] >> (r % 32)) & 1]
    assert dead and all(np.all(W1[r] == 0) for r in dead)
    x = synth.activations(3, cols, g)
    y0, y1 = oracle_lib.gemv(m0, 1, x), oracle_lib.gemv(m1, 1, x)
    xs = oracle_lib.bf16_to_f64(x).reshape(3, cols // 64, 64).sum(axis=2)          # [T, groups]
    live = [r for r in range(rows) if r not in dead]
    bl = b.view(np.float16).astype(np.float64)[sum(1 for rr in range(rows)
                                                     if (bm[0, rr // 32] >> (rr % 32)) & 1):]
    for i, r in enumerate(live):
        assert np.allclose(y1[:, r], y0[:, r] + xs @ bl[i], rtol=0, atol=1e-12)


def test_dequant_column_mapping(oracle_lib):
    # closed form: codebook entry k = (k, -k, 2k, -2k) (exact in fp16),
    # scales 2^(group index) per row r times (r + 1): W[r, c] is fixed by
    # code(r, c // d), component c % d and group c // 64. A transposed or
    # shifted index breaks the pattern.
    d, bits, rows, cols = 4, 5, 3, 256
    K = 1 << bits
    k = np.arange(K, dtype=np.float32)
    cb = synth.f16_bits(np.stack([k, -k, 2 * k, -2 * k], axis=1))
    g = synth.rng(4)
    codes = synth.raw_codes((1, rows, cols // d), bits, g)
    sc = np.array([[(r + 1) * 2.0**gi for gi in range(cols // 64)] for r in range(rows)], dtype=np.float32)
    m = _module(oracle_lib, codes, bits, d, cb, synth.f16_bits(sc)[None])
    W = oracle_lib.dequant(m, 0)
    mult = np.array([1, -1, 2, -2])
    for r in range(rows):
        for c in range(cols):
            expect = codes[0, r, c // d] * mult[c % d] * (r + 1) * 2.0 ** (c // 64)
            assert W[r, c] == expect


def test_dequant_dead_rows_exact_zero(oracle_lib):
    g = synth.rng(8)
    E, rows, cols, d, bits = 2, 64, 128, 2, 8
    codes = synth.raw_codes((E, rows, cols // d), bits, g)
    bm = synth.live_bitmap(E, rows, 8, g)
    cb = synth.codebook(1 << bits, d, g)
    sc = synth.scales(E * rows, cols // 64, g).reshape(E, rows, -1)
    m = _module(oracle_lib, codes, bits, d, cb, sc, bm)
    m_full = _module(oracle_lib, codes, bits, d, cb, sc, None)
    for e in range(E):
        W = oracle_lib.dequant(m, e)
        Wf = oracle_lib.dequant(m_full, e)
        for r in range(rows):
            live = (bm[e, r // 32] >> (r % 32)) & 1
            if live:
                assert np.array_equal(W[r], Wf[r])
            else:
                assert np.all(W[r] == 0.0) and not np.any(np.signbit(W[r]))


# ------------------------------------------------------------------ GEMV

def test_gemv_brute_force_exact(oracle_lib):
    # brute force on a tiny input with exact rational arithmetic
    g = synth.rng(9)
    rows, cols, d, bits = 5, 64, 2, 4
    codes = synth.raw_codes((1, rows, cols // d), bits, g)
    cb = synth.codebook(1 << bits, d, g)
    sc = synth.scales(rows, 1, g)[None]
    x = synth.activations(3, cols, g)
    m = _module(oracle_lib, codes, bits, d, cb, sc)
    y = oracle_lib.gemv(m, 0, x)
    cbv = cb.view(np.float16).astype(np.float64)
    scv = sc[0].view(np.float16).astype(np.float64)
    xv = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(3):
        for r in range(rows):
            exact = sum(Fraction(cbv[codes[0, r, c // d], c % d]) * Fraction(scv[r, 0]) * Fraction(xv[t, c])
                        for c in range(cols))
            assert abs(y[t, r] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))


def test_gemv_one_hot_selects_column(oracle_lib):
    # x = e_c gives y[r] = W[r, c]: pins rows vs columns (rows != cols here)
    g = synth.rng(10)
    rows, cols, d, bits = 7, 128, 4, 6
    codes = synth.raw_codes((1, rows, cols // d), bits, g)
    cb = synth.codebook(1 << bits, d, g)
    sc = synth.scales(rows, cols // 64, g)[None]
    m = _module(oracle_lib, codes, bits, d, cb, sc)
    W = oracle_lib.dequant(m, 0)
    for c in (0, 5, 63, 64, 127):
        x = np.zeros((1, cols), dtype=np.uint16)
        x[0, c] = 0x3F80          # bf16 1.0
        y = oracle_lib.gemv(m, 0, x)
        assert np.array_equal(y[0], W[:, c])


# ------------------------------------------------------------------ routing

def _brute_topk(row, k):
    key = [((1, 0.0) if math.isnan(v) else (0, -float(v)), e) for e, v in enumerate(row)]
    return [e for _, e in sorted(key)[:k]]


def test_route_topk_brute_force(oracle_lib):
    g = np.random.default_rng(12)
    T, E, k = 9, 13, 4
    l = g.standard_normal((T, E)).astype(np.float32)
    l[1, 3] = l[1, 7] = l[1].max() + 1         # tie at the top: lower index first
    l[2, :] = 0.0
    l[2, 5] = -0.0                              # -0 == +0: index decides
    l[3, 2] = np.nan                            # NaN ranks last
    l[4, :] = np.nan
    ids, w, counts, offsets, perm = oracle_lib.route(l, k)
    for t in range(T):
        assert list(ids[t]) == _brute_topk(l[t], k)


def test_route_weights(oracle_lib):
    from scipy.special import softmax
    g = np.random.default_rng(13)
    T, E, k = 6, 40, 7
    l = g.standard_normal((T, E)).astype(np.float32)
    ids, w, *_ = oracle_lib.route(l, k, renorm=True)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    for t in range(T):
        for j in range(1, k):
            assert math.isclose(w[t, 0] / w[t, j], math.exp(float(l[t, ids[t, 0]]) - float(l[t, ids[t, j]])),
                                rel_tol=1e-13)
    ids0, w0, *_ = oracle_lib.route(l, k, renorm=False)
    ref = softmax(l.astype(np.float64), axis=1)
    assert np.array_equal(ids0, ids)
    assert np.allclose(w0, np.take_along_axis(ref, ids0, axis=1), rtol=1e-13, atol=0)


def test_route_bucketing_invariants(oracle_lib):
    g = synth.rng(14)
    T, E, k = 50, 16, 3
    l = synth.logits_zipf(T, E, 1.1, g)
    ids, w, counts, offsets, perm = oracle_lib.route(l, k)
    flat = ids.ravel()
    assert offsets[0] == 0 and offsets[E] == T * k
    assert np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.bincount(flat, minlength=E), counts)
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    for e in range(E):
        b = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[b] == e)
        assert np.all(np.diff(b) > 0)
    assert all(len(set(r)) == k for r in ids)


def test_route_rejects_bad_k(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.route(np.zeros((2, 4), dtype=np.float32), 5)


# ------------------------------------------------------------------ MoE layer

def _layer(oracle_lib, E, H, I, d, bits, seed, identical=False):
    g = synth.rng(seed)
    mods = []
    for rows, cols in ((I, H), (I, H), (H, I)):
        n_e = 1 if identical else E
        codes = synth.raw_codes((n_e, rows, cols // d), bits, g)
        sc = synth.scales(n_e * rows, cols // 64, g).reshape(n_e, rows, -1)
        if identical:
            codes = np.repeat(codes, E, axis=0)
            sc = np.repeat(sc, E, axis=0)
        cb = synth.codebook(1 << bits, d, g)
        mods.append(_module(oracle_lib, codes, bits, d, cb, sc))
    return mods


def _dense_swiglu(oracle_lib, mods, e, x):
    Wg, Wu, Wd = (oracle_lib.dequant(m, e) for m in mods)
    g = Wg @ x
    u = Wu @ x
    return Wd @ (g / (1.0 + np.exp(-g)) * u)


def test_moe_identical_experts_is_dense_swiglu(oracle_lib):
    E, H, I, T, k = 6, 128, 64, 3, 3
    mods = _layer(oracle_lib, E, H, I, 2, 5, 30, identical=True)
    g = synth.rng(31)
    x = synth.activations(T, H, g)
    l = synth.logits_normal(T, E, g)
    y = oracle_lib.moe(*mods, x, l, k)
    xv = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(T):
        ref = _dense_swiglu(oracle_lib, mods, 0, xv[t])
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-14)


def test_moe_weighted_sum_of_selected_experts(oracle_lib):
    E, H, I, T, k = 5, 128, 256, 4, 2
    mods = _layer(oracle_lib, E, H, I, 4, 6, 40)
    g = synth.rng(41)
    x = synth.activations(T, H, g)
    l = synth.logits_normal(T, E, g)
    xv = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for renorm in (True, False):
        y = oracle_lib.moe(*mods, x, l, k, renorm=renorm)
        ids, w, *_ = oracle_lib.route(l, k, renorm=renorm)
        for t in range(T):
            ref = sum(w[t, j] * _dense_swiglu(oracle_lib, mods, ids[t, j], xv[t]) for j in range(k))
            assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-14)
    # k = 1 with renorm: the single selected expert with weight exactly 1
    y1 = oracle_lib.moe(*mods, x, l, 1)
    for t in range(T):
        e = int(np.argmax(l[t]))
        assert np.allclose(y1[t], _dense_swiglu(oracle_lib, mods, e, xv[t]), rtol=1e-12, atol=1e-14)


def test_moe_token_subset_matches_full(oracle_lib):
    E, H, I, T, k = 4, 64, 64, 5, 2
    mods = _layer(oracle_lib, E, H, I, 2, 4, 50)
    g = synth.rng(51)
    x = synth.activations(T, H, g)
    l = synth.logits_normal(T, E, g)
    full = oracle_lib.moe(*mods, x, l, k)
    sub = oracle_lib.moe(*mods, x, l, k, tokens=np.array([4, 1]))
    assert np.array_equal(sub, full[[4, 1]])
