"""GPU parity of the data-free VQ fit (vq_fit) with the CPU oracle (oracle/fit.py)
through the C ABI: scales, codebook and codes bit for bit (every decision is
taken in fp32 by the same definition on both sides; centroid sums are exact)."""
import numpy as np
import pytest
import torch

import synth
from oracle import fit as ofit

import vector_quantized_moe_b200 as vq

pytestmark = pytest.mark.gpu


def _run(w, d, K, sample, init, iters):
    wt = torch.from_numpy(w.view(np.int16)).cuda()
    st = torch.from_numpy(sample).cuda()
    it = torch.from_numpy(init).cuda()
    sc, cb, codes, ws = vq.fit(wt, d, K, st, it, iters)
    torch.cuda.synchronize()
    assert vq.fit_check(ws) == vq.VQ_OK
    return (sc.cpu().numpy().view(np.uint16), cb.cpu().numpy().view(np.uint16), codes.cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("rows,cols,d,K,n_sample,iters", [
    (64, 512, 4, 64, 2048, 5),        # d4, small codebook
    (48, 1024, 2, 256, 4096, 4),      # d2K256 geometry
    (24, 512, 8, 32, 1024, 3),
    (40, 256, 1, 8, 1024, 6),         # d=1 (3-bit scalar codebook)
    (32, 640, 4, 512, 4096, 3),       # d4K512 geometry, ragged row count of blocks
    (64, 512, 8, 4096, 4096, 2),      # K*d = 32768: the largest centroid table
    (16, 128, 2, 8, 8, 0),            # no Lloyd step: the initial points, rounded
])
def test_fit_bit_exact(rows, cols, d, K, n_sample, iters):
    g = synth.rng(700, rows, cols, d, K)
    w = synth.weights(rows, cols, g)
    w[0, :64] = 0                                   # an all-zero group: scale 0, v = 0
    sample, init = synth.fit_draw(rows * cols // d, n_sample, K, g)
    sc, cb, codes = _run(w, d, K, sample, init, iters)
    osc, ocb, ocodes, _ = ofit.fit(w, d, K, sample, init, iters)
    assert np.array_equal(sc, osc)
    assert np.array_equal(cb, ocb)
    assert np.array_equal(codes, ocodes)


def test_fit_full_size_expert_tensor():
    # one d4K512 expert tensor of the Qwen3.5 VQ card's geometry (2048 x 6144), 64K-point
    # sample, 8 Lloyd steps: scales and codebook in full, codes on sampled subvectors
    rows, cols, d, K = 2048, 6144, 4, 512
    g = synth.rng(701)
    w = synth.weights(rows, cols, g)
    sample, init = synth.fit_draw(rows * cols // d, 65536, K, g)
    sc, cb, codes = _run(w, d, K, sample, init, 8)
    osc = ofit.fit_scales(w)
    assert np.array_equal(sc, osc)
    v_all = ofit.subvectors(w, osc, d)
    c = v_all[init].copy()
    for _ in range(8):
        c, _ = ofit.lloyd_step(v_all[sample], c)
    assert np.array_equal(cb, c.astype(np.float16).view(np.uint16))
    pick = np.sort(g.choice(len(v_all), size=20000, replace=False))
    ref = ofit.nearest(v_all[pick], cb.view(np.float16).astype(np.float32))
    assert np.array_equal(codes.reshape(-1)[pick], ref.astype(np.uint16))


def test_fit_codes_feed_the_expert_path():
    # the fit's outputs, packed, go through the library's dequant: W_hat = scale * codebook[code]
    rows, cols, d, K, bits = 32, 512, 4, 256, 8
    g = synth.rng(702)
    w = synth.weights(rows, cols, g)
    sample, init = synth.fit_draw(rows * cols // d, 2048, K, g)
    sc, cb, codes = _run(w, d, K, sample, init, 4)
    words = vq.pack(codes[None], bits)
    m = vq.Module.from_host(1, rows, cols, d, bits, words, sc, cb)
    wh = vq.dequant(m, 0).cpu().numpy()
    ref = cb.view(np.float16).astype(np.float32)[codes.astype(np.int64)].reshape(rows, cols) * \
        np.repeat(sc.view(np.float16).astype(np.float32), 64, axis=1)
    assert np.array_equal(wh, ref)
    # and the fit beats its own starting point on the sample
    v = ofit.subvectors(w, sc, d)[sample]
    assert ofit.sse(v, cb.view(np.float16).astype(np.float32)) < ofit.sse(v, ofit.subvectors(w, sc, d)[init])


def test_fit_index_out_of_range_sets_error_word():
    rows, cols, d, K = 8, 256, 4, 8
    g = synth.rng(703)
    w = synth.weights(rows, cols, g)
    sample, init = synth.fit_draw(rows * cols // d, 64, K, g)
    sample[5] = rows * cols // d + 3                # past the last subvector: skipped, reported
    wt = torch.from_numpy(w.view(np.int16)).cuda()
    _, _, _, ws = vq.fit(wt, d, K, torch.from_numpy(sample).cuda(), torch.from_numpy(init).cuda(), 2)
    torch.cuda.synchronize()
    assert vq.fit_check(ws) == vq.VQ_ERR_DEVICE_CHECK


def test_fit_duplicate_start_and_empty_centroids():
    # two identical initial centroids: in the first step the second loses every tie, gets no
    # point and keeps its value (later steps move the first, and the second may then win points)
    rows, cols, d, K = 32, 512, 4, 16
    g = synth.rng(704)
    w = synth.weights(rows, cols, g)
    sample, init = synth.fit_draw(rows * cols // d, 1024, K, g)
    init[3] = init[1]
    for iters in (1, 4):
        sc, cb, codes = _run(w, d, K, sample, init, iters)
        osc, ocb, ocodes, hist = ofit.fit(w, d, K, sample, init, iters)
        assert np.array_equal(cb, ocb) and np.array_equal(codes, ocodes) and np.array_equal(sc, osc)
        if iters == 1:
            assert np.array_equal(cb[3], hist[0][3].astype(np.float16).view(np.uint16))
            assert not np.array_equal(cb[1], cb[3])


def test_fit_all_zero_tensor():
    # every scale 0, every subvector 0: all codes go to entry 0, the codebook stays the start
    rows, cols, d, K = 8, 256, 2, 8
    w = np.zeros((rows, cols), dtype=np.uint16)
    sample = np.arange(0, rows * cols // d, 2, dtype=np.int32)
    init = sample[:K].copy()
    sc, cb, codes = _run(w, d, K, sample, init, 3)
    assert not sc.any() and not cb.any() and not codes.any()
