"""GPU edge cases of the decode and routing paths, through the C ABI: the
extremes of top_k, an empty batch, workspace reuse across batches of
different sizes (the partial-sum slices of one call must not leak into the
next), and bitwise repeatability."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, lib_module, oracle_module, small_module
from synth import workloads as wl

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,k", [(40, 64, 1), (40, 64, 32), (3, 32, 32), (257, 48, 32)])
def test_route_top_k_extremes(T, E, k):
    g = synth.rng(71, T, E, k)
    lg = synth.logits_normal(T, E, g)
    ids, w, counts, offsets, perm = oracle.route(lg, k, True)
    gi, gw, go, gp = vq.route(torch.from_numpy(lg).cuda(), k, True)
    assert np.array_equal(gi.cpu().numpy(), ids)
    assert np.array_equal(go.cpu().numpy(), offsets)
    assert np.array_equal(gp.cpu().numpy(), perm)
    np.testing.assert_allclose(gw.cpu().numpy(), w, rtol=2e-6, atol=1e-7)


def _layer(E=64, H=512, I=256, geo=(2, 8), seed=5):
    mds = [small_module(E, r, c, *geo, n_dead=0, seed=seed + i) for i, (r, c) in enumerate(((I, H), (I, H), (H, I)))]
    return mds, vq.MoELayer(*[lib_module(m) for m in mds])


def test_empty_batch_launches_nothing():
    _, layer = _layer()
    x = torch.empty((0, layer.hidden), dtype=torch.int16, device="cuda")
    lg = torch.empty((0, layer.E), dtype=torch.float32, device="cuda")
    assert layer.decode(x, lg, 4).shape == (0, layer.hidden)
    assert layer.prefill(x, lg, 4).shape == (0, layer.hidden)
    torch.cuda.synchronize()


def test_workspace_reuse_across_batch_sizes():
    mds, layer = _layer()
    oms = [oracle_module(m) for m in mds]
    k = 6
    ws = layer.workspace(64, k, vq.VQ_MODE_DECODE, "cuda")   # large enough for every call below
    g = synth.rng(72)
    calls = []
    for T in (8, 1, 33, 8):
        x = synth.activations(T, layer.hidden, g)
        lg = synth.logits_normal(T, layer.E, g)
        calls.append((x, lg))
    outs = []
    for x, lg in calls:
        y = layer.decode(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda(), k, workspace=ws)
        torch.cuda.synchronize()
        outs.append(y.cpu().numpy())
        assert_close(outs[-1], oracle.moe(*oms, x, lg, k), what=f"decode T{x.shape[0]} after reuse")
    # the first and the last call have different inputs; rerunning the first reproduces it bit for bit
    x, lg = calls[0]
    y = layer.decode(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda(), k, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy(), outs[0])


def test_decode_bitwise_repeatable():
    _, layer = _layer(geo=(4, 9), seed=9)
    T, k = 16, 8
    g = synth.rng(73)
    x = torch.from_numpy(synth.activations(T, layer.hidden, g).view(np.int16)).cuda()
    lg = torch.from_numpy(synth.logits_normal(T, layer.E, g)).cuda()
    ys = [layer.decode(x, lg, k).cpu().numpy() for _ in range(3)]
    assert all(np.array_equal(ys[0], y) for y in ys[1:])


def test_decode_step_replays_from_a_cuda_graph():
    # the decode step allocates nothing and only launches on its stream: it can be captured
    # once into a CUDA graph and replayed, with outputs bit-identical to eager calls
    E, k, H, I = 16, 4, 512, 256
    oms, layer = _layer(E, H, I, seed=31)
    g = synth.rng(93)
    xs, lgs = [], []
    for _ in range(3):
        x = synth.activations(5, H, g)
        xs.append(torch.from_numpy(x.view(np.int16)).cuda())
        lgs.append(torch.from_numpy(synth.logits_normal(5, E, g)).cuda())
    ws = layer.workspace(5, k, vq.VQ_MODE_DECODE, "cuda")
    outs = [torch.empty((5, H), dtype=torch.float32, device="cuda") for _ in range(3)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        layer.decode(xs[0], lgs[0], k, out=outs[0], workspace=ws, stream=s)   # warm-up outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s):
            for i in range(3):
                layer.decode(xs[i], lgs[i], k, out=outs[i], workspace=ws, stream=s)
    for o in outs:
        o.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for i in range(3):
        want = layer.decode(xs[i], lgs[i], k)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], want)
    del graph


@pytest.mark.parametrize("T", [256, 2048])
def test_skipzero_layer_decode_bitwise_repeatable_from_the_first_call(T):
    # the full-size skipzero + mixed-geometry layer (live bitmaps, d=2/10-bit gate/up, d=8/12-bit down): the
    # first call on a fresh workspace and the calls after it give the same bits (16 calls: a race that
    # changed a few sums in about one call in eight shows up here)
    from helpers import row_words_fn
    mds = wl.layer_modules(wl.SKIPZERO_MIXED, raw=False, row_words=row_words_fn())
    layer = vq.MoELayer(*[lib_module(m) for m in mds])
    del mds
    x, lg = wl.layer_inputs(wl.SKIPZERO_MIXED, T)
    xt, lt = torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda()
    outs = [layer.decode(xt, lt, wl.SKIPZERO_MIXED.top_k).cpu().numpy().view(np.uint32).copy() for _ in range(16)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    del layer
    torch.cuda.empty_cache()
