"""Failure detection on the GPU without a fault: a barrier wait that runs out.

Every wait of the pipelined kernels on an on-chip barrier is bounded. vq_set_wait_limit(0) makes every
wait give up at once, so every CTA with work stops at its first wait; with a bound of a few polls, a
wait gives up or not depending on timing, and a CTA may stop with copies and tensor-core operations
in flight, which it lets complete before it frees its tensor memory and returns. Either way the call
itself returns VQ_OK (it only queues work), vq_moe_check reports VQ_ERR_DEVICE_CHECK whenever a wait
gave up (always with a bound of 0), and the next call on the same workspace, with the default bound,
is correct again (checked against the oracle)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, lib_module, oracle_module, small_module

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu


def _layer():
    # every module streamed through the TMA-staged GEMV in decode (16-byte rows, 8-group scale boxes)
    E, H, I = 8, 1024, 512
    mds = [small_module(E, rows, cols, 2, 8, seed=800 + i) for i, (rows, cols) in enumerate(((I, H), (I, H), (H, I)))]
    return [oracle_module(m) for m in mds], vq.MoELayer(*[lib_module(m) for m in mds])


@pytest.mark.parametrize("limit", [0, 2])
@pytest.mark.parametrize("path", ["decode", "prefill"])
def test_wait_that_runs_out_is_reported_and_the_next_call_is_correct(path, limit):
    oms, layer = _layer()
    T, k = (5, 3) if path == "decode" else (200, 3)
    g = synth.rng(801, T)
    x = synth.activations(T, layer.hidden, g)
    lg = synth.logits_normal(T, layer.E, g)
    xt, lt = torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda()
    fn = layer.decode if path == "decode" else layer.prefill
    mode = vq.VQ_MODE_DECODE if path == "decode" else vq.VQ_MODE_PREFILL
    y = torch.zeros((T, layer.hidden), dtype=torch.float32, device="cuda")
    vq.set_wait_limit(limit)
    try:
        fn(xt, lt, k, out=y)   # queues the work; the waits give up on the GPU
    finally:
        vq.set_wait_limit(None)
    st = layer.check(mode)
    if limit == 0:
        assert st == vq.VQ_ERR_DEVICE_CHECK
    else:
        assert st in (vq.VQ_OK, vq.VQ_ERR_DEVICE_CHECK)
        if st == vq.VQ_OK:   # no wait ran out: the result is complete
            assert_close(y.cpu().numpy(), oracle.moe(*oms, x, lg, k), what=f"{path} with {limit} polls")
    y = fn(xt, lt, k)   # same workspace, default bound
    torch.cuda.synchronize()
    assert layer.check(mode) == vq.VQ_OK
    assert_close(y.cpu().numpy(), oracle.moe(*oms, x, lg, k), what=f"{path} after a give-up")
