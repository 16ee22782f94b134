"""GPU parity of the prefill path (tcgen05 grouped GEMM) against the CPU oracle,
through the C ABI: relative L2 <= 2e-3 and max|err| <= 1e-2 * max|y_ref|;
bf16 outputs are the round-to-nearest-even image of the fp32 outputs."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, lib_module, oracle_module, row_words_fn, small_module
from synth import workloads as wl

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu


def _layer(E, H, I, geos, dead=(0, 0, 0), seed=0):
    mds = []
    for i, (rows, cols) in enumerate(((I, H), (I, H), (H, I))):
        mds.append(small_module(E, rows, cols, *geos[i], n_dead=dead[i], seed=seed * 10 + i))
    return [oracle_module(m) for m in mds], vq.MoELayer(*[lib_module(m) for m in mds])


def _bf16_of(y32):
    return y32.to(torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16)


CASES = [
    # (E, k, H, I, geometries, dead rows)
    (8, 3, 512, 320, ((2, 8), (2, 8), (2, 8)), (0, 0, 0)),          # ragged gate/up tile (320 = 2.5 x 128 rows)
    (8, 3, 320, 256, ((2, 8), (2, 8), (2, 8)), (0, 0, 0)),          # ragged down tile (320 = 2.5 x 128 rows)
    (8, 3, 512, 512, ((4, 9), (4, 9), (4, 9)), (0, 0, 0)),
    (8, 2, 512, 256, ((2, 10), (2, 10), (8, 12)), (21, 17, 0)),      # skipzero gate/up + d=8 down
    (6, 2, 1024, 512, ((4, 11), (4, 11), (4, 11)), (0, 0, 9)),
    (8, 3, 512, 256, ((1, 3), (1, 3), (2, 10)), (0, 0, 0)),
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("T", [1, 7, 64, 300])
def test_prefill_small(case, T):
    E, k, H, I, geos, dead = CASES[case]
    oms, layer = _layer(E, H, I, geos, dead, seed=case + 3 * T)
    g = synth.rng(81, case, T)
    x = synth.activations(T, H, g)
    lg = synth.logits_normal(T, E, g)
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    lt = torch.from_numpy(lg).cuda()
    ref = oracle.moe(*oms, x, lg, k)
    y = layer.prefill(xt, lt, k)
    yb = layer.prefill(xt, lt, k, out_dtype=torch.bfloat16)
    yd = layer.decode(xt, lt, k)
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy(), ref, what=f"prefill case{case} T{T}")
    assert layer.check(vq.VQ_MODE_PREFILL) == vq.VQ_OK
    assert np.array_equal(yb.view(torch.int16).cpu().numpy().view(np.uint16), _bf16_of(y))
    assert_close(y.cpu().numpy(), yd.cpu().numpy().astype(np.float64), what="prefill vs decode")


def test_prefill_buckets_span_several_token_tiles():
    # 4 experts, top-2 of 1200 tokens: ~600 tokens per bucket -> 5 ragged 128-token gate/up tiles
    # and 3 ragged 256-token down tiles
    E, k, H, I = 4, 2, 512, 256
    oms, layer = _layer(E, H, I, ((2, 8), (2, 8), (2, 8)), seed=77)
    g = synth.rng(82)
    x = synth.activations(1200, H, g)
    lg = synth.logits_normal(1200, E, g)
    y = layer.prefill(torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda(), k)
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy(), oracle.moe(*oms, x, lg, k), what="multi-tile buckets")


@pytest.mark.parametrize("T,chunk", [(600, 256), (700, 700), (1000, 333), (5, 2)])
def test_prefill_chunked_matches_one_call(T, chunk):
    # chunk after chunk through one chunk-sized workspace: every token's output equals the
    # one-call prefill bit for bit (it depends only on its own row), and the oracle on samples
    E, k, H, I = 8, 3, 512, 256
    oms, layer = _layer(E, H, I, ((2, 8), (2, 8), (2, 8)), seed=91)
    g = synth.rng(83, T, chunk)
    x = synth.activations(T, H, g)
    lg = synth.logits_normal(T, E, g)
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    lt = torch.from_numpy(lg).cuda()
    y = layer.prefill(xt, lt, k)
    ws = torch.empty(layer.workspace_size(min(T, chunk), k, vq.VQ_MODE_PREFILL) + 256, dtype=torch.uint8,
                     device="cuda")
    yc = layer.prefill_chunked(xt, lt, k, chunk=chunk, workspace=ws)
    yb = layer.prefill_chunked(xt, lt, k, chunk=chunk, out_dtype=torch.bfloat16, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(yc.cpu().numpy().view(np.uint32), y.cpu().numpy().view(np.uint32))
    assert np.array_equal(yb.view(torch.int16).cpu().numpy().view(np.uint16), _bf16_of(y))   # bf16 rows offset right
    tok = np.unique(np.array([0, chunk - 1, chunk % T, T // 2, T - 1]) % T)
    assert_close(yc.cpu().numpy()[tok], oracle.moe(*oms, x, lg, k, tokens=tok), what=f"chunked T{T} c{chunk}")
    if T > chunk:
        assert layer.workspace_size(chunk, k, vq.VQ_MODE_PREFILL) < layer.workspace_size(T, k, vq.VQ_MODE_PREFILL)


def test_prefill_rejects_unaligned_geometry():
    # d=4 / 9-bit needs cols to be a multiple of 512 for whole 16-byte code chunks
    E, H, I = 4, 256, 512
    _, layer = _layer(E, H, I, ((4, 9), (4, 9), (4, 9)))
    x = torch.zeros((2, H), dtype=torch.int16, device="cuda")
    lg = torch.zeros((2, E), dtype=torch.float32, device="cuda")
    with pytest.raises(vq.VQError):
        layer.prefill(x, lg, 2)


@pytest.mark.parametrize("spec,T,n_sample", [
    (wl.PREFILL_D4K512, 4096, 256),    # a seeded 256-token subset of the Zipf(1.1) layer (2048 expert pairs)
    (wl.SKIPZERO_MIXED, 2048, 64),
])
def test_prefill_full_size(spec, T, n_sample):
    mds = wl.layer_modules(spec, raw=False, row_words=row_words_fn())
    oms = [oracle_module(m) for m in mds]
    layer = vq.MoELayer(*[lib_module(m) for m in mds])
    x, lg = wl.layer_inputs(spec, T)
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    lt = torch.from_numpy(lg).cuda()
    y = layer.prefill(xt, lt, spec.top_k)
    torch.cuda.synchronize()
    tok = np.sort(synth.rng(84, T).choice(T, size=n_sample, replace=False))
    tok[0], tok[-1] = 0, T - 1   # the first and the last token are always in
    tok = np.unique(tok)
    ref = oracle.moe(*oms, x, lg, spec.top_k, tokens=tok)
    got = y.cpu().numpy()[tok]
    assert_close(got, ref, what=f"{spec.name} T{T}")
    for i in range(len(tok)):   # and token by token
        assert_close(got[i], ref[i], what=f"{spec.name} T{T} token {tok[i]}")
    # in ragged chunks through a chunk-sized workspace: the same outputs bit for bit
    yc = layer.prefill_chunked(xt, lt, spec.top_k, chunk=T // 2 + 7)
    torch.cuda.synchronize()
    assert np.array_equal(yc.cpu().numpy().view(np.uint32), y.cpu().numpy().view(np.uint32))
    del yc
    # every token: decode path and prefill path agree
    yd = layer.decode(xt, lt, spec.top_k)
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy(), yd.cpu().numpy().astype(np.float64), what="prefill vs decode, all tokens")
    del layer
    torch.cuda.empty_cache()
