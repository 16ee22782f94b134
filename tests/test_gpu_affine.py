"""GPU parity of the affine arm (per-group biases) against the CPU oracle, through the C ABI.

The cards' fallback format "affine 3-bit, group 64" (Qwen3.5-397B-A17B-VQ-2.4bpw card, Changelog
2026-09-20) gives no formula; the library reads it as w = s * q + b with an fp16 scale and an fp16 bias
per (row, 64 weights): d = 1, the identity codebook C[q] = q, plus the bias. The same bias can sit on
any VQ module (w = s * C[q] + b). The oracle's biased dequantisation is pinned by its own CPU tests.

Checked here: one-hot activations give the weights themselves (decode GEMV: fp32 of s * C[q] + b,
rounded once; prefill GEMM: its fp16 rounding, one fused multiply-add), and the GEMV, the decode layer
and the prefill layer meet the usual float bar with biased modules, alone and mixed with plain ones."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, lib_module, oracle_module, small_module

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu

BF16_ONE = 0x3F80


def _biased(md, seed, affine=False):
    """(oracle module, library module) of md with seeded biases; affine=True also swaps in the identity
    codebook C[q] = q (d = 1), the plain affine format."""
    g = synth.rng(1100, seed)
    if affine:
        assert md.d == 1
        md.codebook = synth.f16_bits(np.arange(1 << md.bits, dtype=np.float32)).reshape(-1, 1)
        # affine scales are small (the group's range / 2^bits): U(0.5, 2) / 64
        md.scales = synth.f16_bits(synth.rng(1101, seed).uniform(0.5, 2.0, md.scales.shape).astype(np.float32) / 64)
    b = synth.biases(md.E * md.rows, md.cols // 64, g).reshape(md.E, md.rows, md.cols // 64)
    om = oracle_module(md)
    om.biases = oracle.compact_rows(b, md.bitmap)
    base = lib_module(md)
    bl = vq.pack_scales(b, md.bitmap)
    lm = vq.Module(base.E, base.rows, base.cols, base.d, base.bits, base.codes, base.scales, base.codebook,
                   base.live_bitmap, base.live_rank, torch.from_numpy(bl.view(np.int16)).to(base.codes.device))
    return om, lm


def _one_hot(cols):
    x = np.zeros((cols, cols), dtype=np.uint16)
    x[np.arange(cols), np.arange(cols)] = BF16_ONE
    return torch.from_numpy(x.view(np.int16)).cuda()


GEOS = [(1, 3, True), (2, 8, False), (4, 9, False), (2, 10, False)]


@pytest.mark.parametrize("d,bits,affine", GEOS)
@pytest.mark.parametrize("cols,rows", [(1024, 300), (256, 80)])   # TMA-staged kernel (d = 8: register); register kernel
def test_gemv_weights_bit_exact_with_bias(d, bits, affine, cols, rows):
    md = small_module(2, rows, cols, d, bits, n_dead=17, seed=1110 + 16 * d + bits)
    om, lm = _biased(md, d * 100 + bits, affine)
    xt = _one_hot(cols)
    for e in range(2):
        y = vq.gemv(lm, e, xt).cpu().numpy()
        W = oracle.dequant(om, e).astype(np.float32)   # the exact s * C[q] + b rounded once to fp32
        assert np.array_equal(y.T, W), f"d{d} b{bits} e{e}: {np.count_nonzero(y.T != W)} weights differ"


@pytest.mark.parametrize("d,bits,affine", [g for g in GEOS if vq.packed_words(1, 1024 // g[0], g[1]) % 4 == 0])
def test_prefill_gemm_weights_bit_exact_with_bias(d, bits, affine):
    cols, rows = 1024, 320
    md = small_module(2, rows, cols, d, bits, n_dead=11, seed=1120 + 16 * d + bits)
    om, lm = _biased(md, 200 + d * 100 + bits, affine)
    xt = _one_hot(cols)
    for e in range(2):
        y, _, _ = vq.gemm(lm, e, xt)
        W = oracle.dequant(om, e).astype(np.float16).astype(np.float64)   # one rounding to fp16
        assert np.array_equal(y.cpu().numpy().astype(np.float64).T, W)


@pytest.mark.parametrize("T", [1, 9])
@pytest.mark.parametrize("d,bits,affine", GEOS)
def test_gemv_with_bias(d, bits, affine, T):
    md = small_module(2, 300, 1024, d, bits, n_dead=21, seed=1130 + d + bits)
    om, lm = _biased(md, 300 + d + bits, affine)
    x = synth.activations(T, 1024, synth.rng(1131, T))
    y = vq.gemv(lm, 1, torch.from_numpy(x.view(np.int16)).cuda())
    assert_close(y.cpu().numpy(), oracle.gemv(om, 1, x), what=f"biased gemv d{d} b{bits} T{T}")


LAYERS = [
    # (gate, up, down): (d, bits, affine, biased)
    (((1, 3, True, True), (1, 3, True, True), (1, 3, True, True)), (0, 0, 0)),        # an affine 3-bit layer
    (((2, 8, False, True), (2, 8, False, True), (2, 8, False, False)), (0, 0, 0)),    # biased gate/up, plain down
    (((2, 10, False, True), (2, 10, False, False), (4, 9, False, True)), (13, 0, 0)),  # mixed, skipzero gate
]


@pytest.mark.parametrize("li", range(len(LAYERS)))
@pytest.mark.parametrize("path,T", [("decode", 1), ("decode", 7), ("prefill", 150)])
def test_layer_with_bias(li, path, T):
    E, k, H, I = 8, 3, 1024, 512
    mods, dead = LAYERS[li]
    oms, lms = [], []
    for i, ((d, bits, affine, biased), (rows, cols)) in enumerate(zip(mods, ((I, H), (I, H), (H, I)))):
        md = small_module(E, rows, cols, d, bits, n_dead=dead[i], seed=1140 + 10 * li + i)
        if biased:
            om, lm = _biased(md, 400 + 10 * li + i, affine)
        else:
            om, lm = oracle_module(md), lib_module(md)
        oms.append(om)
        lms.append(lm)
    layer = vq.MoELayer(*lms)
    g = synth.rng(1150, li, T)
    x = synth.activations(T, H, g)
    lg = synth.logits_normal(T, E, g)
    fn = layer.decode if path == "decode" else layer.prefill
    y = fn(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda(), k)
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy(), oracle.moe(*oms, x, lg, k), what=f"{path} layer{li} T{T}")
