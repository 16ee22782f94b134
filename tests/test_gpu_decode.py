"""GPU parity of the decode path against the CPU oracle, through the C ABI.

Bit-exact: code unpacking, dequantised weights, routing ids, bucket offsets
and the pair permutation. Floating point: relative L2 <= 2e-3 and
max|err| <= 1e-2 * max|y_ref| (fp32 outputs); bf16 outputs must be the
round-to-nearest-even image of the fp32 outputs."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, lib_module, oracle_module, row_words_fn, small_module
from synth import workloads as wl

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu

GEOS = [(1, 3), (1, 4), (2, 8), (2, 10), (2, 11), (4, 8), (4, 9), (4, 11), (4, 13), (8, 12)]


def _cols(d):
    return 512 if d == 8 else 256


def _live_mask(md, e):
    if md.bitmap is None:
        return np.ones(md.rows, dtype=bool)
    return np.array([(md.bitmap[e, r // 32] >> (r % 32)) & 1 for r in range(md.rows)], dtype=bool)


def _bf16_of(y32: torch.Tensor) -> np.ndarray:
    return y32.to(torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("d,bits", GEOS)
def test_unpack_and_dequant_bit_exact(d, bits):
    E, rows, cols = 3, 77, _cols(d)
    md = small_module(E, rows, cols, d, bits, n_dead=9, seed=100 * d + bits)
    om, lm = oracle_module(md), lib_module(md)
    ow = om.words
    start = 0
    for e in range(E):
        live = _live_mask(md, e)
        codes = vq.unpack(lm, e).cpu().numpy().view(np.uint16)
        ref = oracle.unpack(ow[start:start + live.sum()], cols // d, bits)
        start += live.sum()
        assert np.array_equal(codes[live], ref)
        assert np.all(codes[~live] == 0xFFFF)
        W = vq.dequant(lm, e).cpu().numpy().astype(np.float64)
        assert np.array_equal(W, oracle.dequant(om, e))


@pytest.mark.parametrize("d,bits", GEOS)
@pytest.mark.parametrize("T", [1, 5, 8, 13])
def test_gemv_small(d, bits, T):
    E, rows, cols = 2, 80, _cols(d)
    md = small_module(E, rows, cols, d, bits, n_dead=7, seed=7 * d + bits)
    om, lm = oracle_module(md), lib_module(md)
    x = synth.activations(T, cols, synth.rng(5, T))
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    for e in range(E):
        ref = oracle.gemv(om, e, x)
        y = vq.gemv(lm, e, xt, out_dtype=torch.float32)
        yb = vq.gemv(lm, e, xt, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert_close(got, ref, what=f"gemv d{d} b{bits} T{T} e{e}")
        dead = ~_live_mask(md, e)
        assert np.all(got[:, dead] == 0) and not np.any(np.signbit(got[:, dead]))
        assert np.array_equal(yb.view(torch.int16).cpu().numpy().view(np.uint16), _bf16_of(y))


def test_gemv_single_512x1024_d2k256():
    s = wl.GEMV_D2K256
    md = wl.module_data(1, s.rows, s.cols, s.geo, 0, (s.seed, 0), raw=True)
    om, lm = oracle_module(md), lib_module(md)
    x = synth.activations(s.T, s.cols, synth.rng(s.seed, 1))
    y = vq.gemv(lm, 0, torch.from_numpy(x.view(np.int16)).cuda())
    assert_close(y.cpu().numpy(), oracle.gemv(om, 0, x), what="gemv 512x1024")


@pytest.mark.parametrize("T,E,k,zipf", [(1, 512, 10, None), (8, 512, 10, None), (16, 256, 8, None),
                                        (300, 64, 6, None), (4096, 256, 8, 1.1), (2048, 512, 10, None),
                                        (33, 2000, 4, None)])
def test_route_bit_exact(T, E, k, zipf):
    g = synth.rng(70, T, E)
    lg = synth.logits_zipf(T, E, zipf, g) if zipf else synth.logits_normal(T, E, g)
    if T >= 8:
        lg[3, 5] = lg[3, 9] = lg[3].max() + 1.0      # tie at the top
        lg[4, 2] = np.nan
        lg[5, :] = 0.0
        lg[5, 7] = -0.0
    for renorm in (True, False):
        ids, w, counts, offsets, perm = oracle.route(lg, k, renorm)
        gi, gw, go, gp = vq.route(torch.from_numpy(lg).cuda(), k, renorm)
        assert np.array_equal(gi.cpu().numpy(), ids)
        assert np.array_equal(go.cpu().numpy(), offsets)
        assert np.array_equal(gp.cpu().numpy(), perm)
        ok = np.isfinite(w).all(axis=1)
        np.testing.assert_allclose(gw.cpu().numpy()[ok], w[ok], rtol=2e-6, atol=1e-7)


def _small_layer(E, H, I, geos, dead=(0, 0, 0), seed=0):
    mds = []
    for i, (rows, cols) in enumerate(((I, H), (I, H), (H, I))):
        mds.append(small_module(E, rows, cols, *geos[i], n_dead=dead[i], seed=seed * 10 + i))
    return mds


@pytest.mark.parametrize("geos,dead", [
    (((2, 8), (2, 8), (2, 8)), (0, 0, 0)),
    (((2, 10), (2, 10), (8, 12)), (13, 11, 0)),
    (((4, 9), (4, 11), (4, 9)), (0, 0, 5)),
    (((1, 3), (1, 3), (2, 8)), (0, 0, 0)),
])
@pytest.mark.parametrize("T", [1, 4, 19])
def test_moe_decode_small(geos, dead, T):
    E, k, H, I = 8, 3, 512, 256
    mds = _small_layer(E, H, I, geos, dead, seed=T)
    oms = [oracle_module(m) for m in mds]
    layer = vq.MoELayer(*[lib_module(m) for m in mds])
    g = synth.rng(80, T)
    x = synth.activations(T, H, g)
    lg = synth.logits_normal(T, E, g)
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    lt = torch.from_numpy(lg).cuda()
    for renorm in (True, False):
        ref = oracle.moe(*oms, x, lg, k, renorm)
        y = layer.decode(xt, lt, k, renorm)
        yb = layer.decode(xt, lt, k, renorm, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert_close(y.cpu().numpy(), ref, what=f"moe decode {geos} T{T}")
        assert layer.check(vq.VQ_MODE_DECODE) == vq.VQ_OK
        assert np.array_equal(yb.view(torch.int16).cpu().numpy().view(np.uint16), _bf16_of(y))


def _full_layer(spec):
    mds = wl.layer_modules(spec, raw=False, row_words=row_words_fn())
    return mds, [oracle_module(m) for m in mds], vq.MoELayer(*[lib_module(m) for m in mds])


@pytest.mark.parametrize("spec,T,sample", [
    (wl.DECODE_D2K256, 1, None), (wl.DECODE_D2K256, 8, [0, 5, 7]),
    (wl.DECODE_D4K512, 16, [0, 9, 15]), (wl.DECODE_D4K2048, 16, [2, 11]),
    (wl.SKIPZERO_MIXED, 1, None),
])
def test_moe_decode_full_size(spec, T, sample):
    mds, oms, layer = _full_layer(spec)
    x, lg = wl.layer_inputs(spec, T)
    y = layer.decode(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda(), spec.top_k)
    torch.cuda.synchronize()
    tok = np.arange(T) if sample is None else np.array(sample)
    ref = oracle.moe(*oms, x, lg, spec.top_k, tokens=tok)
    assert_close(y.cpu().numpy()[tok], ref, what=f"{spec.name} T{T}")
    del layer
    torch.cuda.empty_cache()


@pytest.mark.parametrize("d,bits", GEOS)
@pytest.mark.parametrize("T", [1, 9])
def test_gemv_staged_path(d, bits, T):
    # 1024 columns (16 groups) and 300 rows with skipzero: the TMA-staged kernel (d = 8: the register kernel)
    # path (several 256-row items, a ragged last item, compacted live rows)
    E, rows, cols = 3, 300, 1024
    md = small_module(E, rows, cols, d, bits, n_dead=37, seed=11 * d + bits)
    om, lm = oracle_module(md), lib_module(md)
    x = synth.activations(T, cols, synth.rng(6, T))
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    for e in range(E):
        y = vq.gemv(lm, e, xt)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert_close(got, oracle.gemv(om, e, x), what=f"staged gemv d{d} b{bits} T{T} e{e}")
        dead = ~_live_mask(md, e)
        assert np.all(got[:, dead] == 0)
