"""vq_moe_decode_noalloc: the decode layer for callers that cannot allocate
device memory (a host framework that owns every allocation, or a thin C FFI
without a CUDA memory API). Its scratch is a static device array inside the
library; this checks, through the C ABI, that two calls in a row reproduce
vq_moe_decode and the CPU oracle (same tolerance as the other parity tests)
and that a batch too large for the static scratch is refused.

Collected last on purpose, so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, lib_module, oracle_module, small_module

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu

VQ_ERR_WORKSPACE = 4


def _layer():
    E, H, I = 16, 1024, 512
    mds = [small_module(E, I, H, 2, 8, seed=900), small_module(E, I, H, 2, 8, seed=901),
           small_module(E, H, I, 2, 8, seed=902)]
    layer = vq.MoELayer(*[lib_module(m) for m in mds])
    layer.oracle_modules = [oracle_module(m) for m in mds]
    return layer


def _noalloc(layer, x, lg, k, y):
    return vq._L().vq_moe_decode_noalloc(ctypes.byref(layer._s), x.data_ptr(), x.shape[0], lg.data_ptr(), k, 1,
                                         y.data_ptr(), vq.VQ_F32, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_decode_twice():
    layer = _layer()
    T, k = 5, 4
    g = synth.rng(903)
    xh = synth.activations(T, layer.hidden, g)
    lgh = synth.logits_normal(T, layer.E, g)
    x = torch.from_numpy(xh.view(np.int16)).cuda()
    lg = torch.from_numpy(lgh).cuda()
    ref = layer.decode(x, lg, k).cpu().numpy()
    want = oracle.moe(*layer.oracle_modules, xh, lgh, k)
    for _ in range(2):
        y = torch.full((T, layer.hidden), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(layer, x, lg, k, y) == 0
        torch.cuda.synchronize()
        assert_close(y.cpu().numpy(), ref, what="noalloc decode vs vq_moe_decode")
        assert_close(y.cpu().numpy(), want, what="noalloc decode vs the oracle")


def test_noalloc_rejects_batch_beyond_static_scratch():
    layer = _layer()
    T, k = 2000, 4
    assert layer.workspace_size(T, k, vq.VQ_MODE_DECODE) > (16 << 20)
    x = torch.zeros((T, layer.hidden), dtype=torch.int16, device="cuda")
    lg = torch.zeros((T, layer.E), dtype=torch.float32, device="cuda")
    y = torch.zeros((T, layer.hidden), dtype=torch.float32, device="cuda")
    assert _noalloc(layer, x, lg, k, y) == VQ_ERR_WORKSPACE
