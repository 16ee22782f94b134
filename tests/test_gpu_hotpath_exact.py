"""Bit-exact checks of the weight decoding inside the hot-path kernels themselves.

The format (Qwen3.5-397B-A17B-VQ-2.4bpw card, "Methodology": row-local, LSB-first 32-code blocks in
uint32 words; Qwen3.5-397B-A17B-VQ-2.6bpw card, "Methodology": one fp16 scale per (row, 64 weights))
fixes every dequantised weight W[r, c] = fp16(centroid) * fp16(scale), an exact fp32 product.

Driving a GEMM with one-hot activation rows (token t = e_t, bf16 1.0) makes its output the weight
matrix itself: y[t, r] = W[r, t]. In the decode GEMV one product of an fp16 centroid and 1.0 enters the
fp32 sum of its group, and the fp32 group scale multiplies it, so y must equal the oracle's W bit for
bit. In the prefill GEMM the weight tile is the fp16 rounding of the product (round to nearest even),
so y must equal RNE-fp16 of the oracle's W bit for bit. Every column of every row is covered, so the
codes that straddle word and 32-code-block boundaries (9-, 10-, 11- and 13-bit codes), the swizzled
8-bit layout and the skipzero rows are all exercised in the kernels that run on the hot path."""
import numpy as np
import pytest
import torch

import oracle
from helpers import lib_module, oracle_module, small_module

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu

GEOS = [(1, 3), (1, 4), (2, 8), (2, 10), (2, 11), (4, 8), (4, 9), (4, 11), (4, 13), (8, 12)]
BF16_ONE = 0x3F80


def _one_hot(cols):
    x = np.zeros((cols, cols), dtype=np.uint16)
    x[np.arange(cols), np.arange(cols)] = BF16_ONE
    return torch.from_numpy(x.view(np.int16)).cuda()


def _live(md, e):
    if md.bitmap is None:
        return np.ones(md.rows, dtype=bool)
    return np.array([(md.bitmap[e, r // 32] >> (r % 32)) & 1 for r in range(md.rows)], dtype=bool)


@pytest.mark.parametrize("d,bits", GEOS)
@pytest.mark.parametrize("cols,rows", [(1024, 300), (256, 80)])   # TMA-staged kernel (d = 8: register); register kernel
def test_gemv_weights_bit_exact(d, bits, cols, rows):
    md = small_module(3, rows, cols, d, bits, n_dead=29, seed=600 + 16 * d + bits)
    om, lm = oracle_module(md), lib_module(md)
    xt = _one_hot(cols)
    for e in range(md.E):
        y = vq.gemv(lm, e, xt).cpu().numpy().astype(np.float64)   # [cols tokens, rows]
        W = oracle.dequant(om, e)
        assert np.array_equal(y.T, W), f"d{d} b{bits} e{e}: {np.count_nonzero(y.T != W)} weights differ"
        dead = ~_live(md, e)
        assert not np.any(np.signbit(y[:, dead]))


def _fp16_rne(W):
    return W.astype(np.float16).astype(np.float64)   # numpy rounds binary64 -> binary16 to nearest even


@pytest.mark.parametrize("d,bits", [g for g in GEOS if vq.packed_words(1, 1024 // g[0], g[1]) % 4 == 0])
def test_prefill_gemm_weights_bit_exact(d, bits):
    # two modules sharing each weight-tile pass (the gate/up instantiation) and one alone (down's)
    cols, rows = 1024, 320
    md0 = small_module(2, rows, cols, d, bits, n_dead=23, seed=700 + 16 * d + bits)
    md1 = small_module(2, rows, cols, d, bits, n_dead=0, seed=701 + 16 * d + bits)
    om0, om1 = oracle_module(md0), oracle_module(md1)
    lm0, lm1 = lib_module(md0), lib_module(md1)
    xt = _one_hot(cols)
    pair = (d, bits) != (4, 13)   # two 8192-entry codebooks and their stages do not fit shared memory
    if not pair:
        with pytest.raises(vq.VQError) as ei:
            vq.gemm(lm0, 0, xt, m1=lm1)
        assert ei.value.status == vq.VQ_ERR_UNSUPPORTED
    for e in range(2):
        W0, W1 = _fp16_rne(oracle.dequant(om0, e)), _fp16_rne(oracle.dequant(om1, e))
        z, none, _ = vq.gemm(lm0, e, xt)
        assert none is None
        assert np.array_equal(z.cpu().numpy().astype(np.float64).T, W0)
        if not pair:
            continue
        y0, y1, _ = vq.gemm(lm0, e, xt, m1=lm1)
        y0, y1 = y0.cpu().numpy().astype(np.float64), y1.cpu().numpy().astype(np.float64)
        assert np.array_equal(y0.T, W0), f"gate-like d{d} b{bits} e{e}: {np.count_nonzero(y0.T != W0)} differ"
        assert np.array_equal(y1.T, W1), f"up-like d{d} b{bits} e{e}: {np.count_nonzero(y1.T != W1)} differ"
