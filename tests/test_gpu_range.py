"""GPU parity over bf16's whole range, through the C ABI, against the CPU oracle.

The runtime the VQ model cards describe takes bf16 activations (Qwen3.8-Flash-Next-VQ-4.4bpw card,
Changelog 2026-09-17: bf16 I/O), while the tensor cores read fp16 operands. The library scales each
operand row by a power of two before its fp16 rounding and undoes it in fp32, so tokens far outside
fp16's range, tokens with outliers and batches that mix magnitudes must all meet the usual bar. It is
checked token by token (relative L2 <= 2e-3, max|err| <= 1e-2 * max|y_ref| for each token), so a
small token next to a large one cannot hide behind it."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, lib_module, oracle_module, small_module

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu


def _cases(T, H, seed):
    """(name, bf16 activations [T, H]) for the range cases."""
    g = synth.rng(500, seed, T, H)
    ng = H // 64
    mixed = g.integers(-30, 18, size=T)
    out = [
        ("tiny 2^-20", synth.activations_scaled(T, H, g, log2_token=np.full(T, -20))),
        ("huge 2^17", synth.activations_scaled(T, H, g, log2_token=np.full(T, 17))),
        ("outlier 3e5", synth.activations_scaled(T, H, g, outliers=[(t, (37 * t + 5) % H, 3.0e5) for t in range(T)])),
        ("mixed 2^-30..2^17", synth.activations_scaled(T, H, g, log2_token=mixed)),
        # groups of one token 2^40 apart: below fp16's range for one, above it for another
        ("groups 2^-24..2^16", synth.activations_scaled(T, H, g, log2_group=g.integers(-24, 17, size=(T, ng)))),
    ]
    return out


def _per_token(got, ref, what):
    for t in range(ref.shape[0]):
        assert_close(got[t], ref[t], what=f"{what} token {t}")


@pytest.mark.parametrize("cols,rows", [(1024, 300), (256, 80)])   # TMA-staged (d = 8: register) and register kernels
@pytest.mark.parametrize("d,bits", [(2, 8), (4, 9), (2, 10), (8, 12), (1, 4)])
def test_gemv_range(cols, rows, d, bits):
    md = small_module(2, rows, cols, d, bits, n_dead=11, seed=510 + d * bits)
    om, lm = oracle_module(md), lib_module(md)
    T = 9
    for name, x in _cases(T, cols, d * 100 + bits):
        xt = torch.from_numpy(x.view(np.int16)).cuda()
        for e in range(2):
            y = vq.gemv(lm, e, xt)
            torch.cuda.synchronize()
            _per_token(y.cpu().numpy(), oracle.gemv(om, e, x), f"gemv d{d}b{bits} {cols} {name} e{e}")


def _layer(E, H, I, geos, dead, seed):
    mds = [small_module(E, rows, cols, *geos[i], n_dead=dead[i], seed=seed * 10 + i)
           for i, (rows, cols) in enumerate(((I, H), (I, H), (H, I)))]
    return [oracle_module(m) for m in mds], vq.MoELayer(*[lib_module(m) for m in mds])


LAYERS = [
    (8, 3, 512, 256, ((2, 8), (2, 8), (2, 8)), (0, 0, 0)),
    (8, 2, 1024, 512, ((2, 10), (2, 10), (8, 12)), (21, 17, 0)),
    (6, 2, 512, 512, ((4, 9), (4, 9), (4, 9)), (0, 0, 5)),
]


@pytest.mark.parametrize("li", range(len(LAYERS)))
@pytest.mark.parametrize("path", ["decode", "prefill"])
def test_moe_range(li, path):
    E, k, H, I, geos, dead = LAYERS[li]
    oms, layer = _layer(E, H, I, geos, dead, seed=520 + li)
    T = 7 if path == "decode" else 150
    g = synth.rng(521, li, T)
    lg = synth.logits_normal(T, E, g)
    lt = torch.from_numpy(lg).cuda()
    fn = layer.decode if path == "decode" else layer.prefill
    for name, x in _cases(T, H, 10 * li + (path == "prefill")):
        ref = oracle.moe(*oms, x, lg, k)
        y = fn(torch.from_numpy(x.view(np.int16)).cuda(), lt, k)
        torch.cuda.synchronize()
        _per_token(y.cpu().numpy(), ref, f"{path} layer{li} {name}")
        assert layer.check(vq.VQ_MODE_DECODE if path == "decode" else vq.VQ_MODE_PREFILL) == vq.VQ_OK


def test_zero_token_gives_zero():
    # an all-zero activation row (and +-0 mixed in) gives exactly zero outputs on both paths
    oms, layer = _layer(8, 512, 256, ((2, 8), (2, 8), (2, 8)), (0, 0, 0), seed=530)
    T, k = 4, 3
    g = synth.rng(531)
    x = synth.activations(T, 512, g)
    x[1] = 0
    x[2, ::2] = 0x8000   # -0
    x[2, 1::2] = 0
    lg = synth.logits_normal(T, 8, g)
    xt, lt = torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda()
    for fn in (layer.decode, layer.prefill):
        y = fn(xt, lt, k).cpu().numpy()
        assert np.all(y[1] == 0) and np.all(y[2] == 0)
        assert_close(y[[0, 3]], oracle.moe(*oms, x, lg, k, tokens=np.array([0, 3])), what="other tokens")
