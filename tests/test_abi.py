"""CPU tests of the C ABI: the library loads, exports every symbol the header
declares, and its host-side packing matches the oracle bit for bit. No call
here launches GPU work."""
import ctypes

import numpy as np
import pytest

import oracle
import synth

import vector_quantized_moe_b200 as vq


def test_header_symbols_exported():
    names = vq.header_functions()
    assert len(names) >= 13
    lib = ctypes.CDLL(vq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for s in range(7):
        assert vq.status_str(s)
    assert vq.status_str(1).startswith("VQ_ERR_ARG")


def test_geometries():
    for d, b in ((2, 8), (2, 10), (4, 9), (4, 11), (8, 12), (1, 3)):
        assert vq.geometry_supported(d, b)
    assert not vq.geometry_supported(3, 8)
    assert not vq.geometry_supported(2, 16)


@pytest.mark.parametrize("ncode,bits", [(32, 3), (64, 8), (96, 9), (128, 10), (64, 11), (32, 12), (64, 13), (32, 16)])
def test_packed_words_closed_form(ncode, bits):
    assert vq.packed_words(7, ncode, bits) == 7 * (ncode // 32) * bits
    assert vq.packed_words(1, 33, bits) == 0


@pytest.mark.parametrize("bits", [1, 3, 4, 8, 9, 10, 11, 12, 13, 16])
def test_pack_matches_oracle(bits):
    g = synth.rng(60, bits)
    E, rows, ncode = 3, 37, 96
    codes = synth.raw_codes((E, rows, ncode), bits, g)
    bm = synth.live_bitmap(E, rows, 5, g)
    for b in (None, bm):
        assert np.array_equal(vq.pack(codes, bits, b), oracle.pack(codes, bits, b))


def test_pack_scales_and_rank():
    g = synth.rng(61)
    E, rows, ng = 4, 70, 3
    sc = synth.scales(E * rows, ng, g).reshape(E, rows, ng)
    bm = synth.live_bitmap(E, rows, 11, g)
    assert np.array_equal(vq.pack_scales(sc, bm), oracle.compact_rows(sc, bm))
    rank = vq.live_rank(bm, rows)
    # rank[e, w] = live rows before (e, 32*w), counted by brute force
    live = [[(bm[e, r // 32] >> (r % 32)) & 1 for r in range(rows)] for e in range(E)]
    for e in range(E):
        for w in range(bm.shape[1]):
            assert rank[e, w] == sum(sum(live[x]) for x in range(e)) + sum(live[e][: 32 * w])


def test_pack_rejects_out_of_range_code():
    codes = np.zeros((1, 1, 32), dtype=np.uint16)
    codes[0, 0, 5] = 8
    with pytest.raises(vq.VQError):
        vq.pack(codes, 3)


def test_live_rank_rejects_bits_beyond_rows():
    bm = np.array([[0xFFFFFFFF]], dtype=np.uint32)
    with pytest.raises(vq.VQError):
        vq.live_rank(bm, 20)


def _null_module(**kw):
    m = dict(E=2, rows=64, cols=128, d=2, bits=8, codes=256, scales=512, codebook=1024, live_bitmap=None,
             live_rank=None)
    m.update(kw)
    return vq.vq_module(m["E"], m["rows"], m["cols"], m["d"], m["bits"], m["codes"], m["scales"], m["codebook"],
                        m["live_bitmap"], m["live_rank"], m.get("live_rows", 0), m.get("biases"))


@pytest.mark.parametrize("kw,status", [
    (dict(codes=None), 1), (dict(cols=100), 1), (dict(d=3), 1), (dict(bits=7), 3), (dict(codes=264), 2),
    (dict(live_bitmap=4096), 1), (dict(E=0), 1), (dict(biases=4097), 2),
])
def test_argument_errors_before_launch(kw, status):
    # fake (never dereferenced) pointers: validation fails before any CUDA call
    m = _null_module(**kw)
    rc = vq._L().vq_gemv(ctypes.byref(m), 0, 4096, 1, 8192, 0, None)
    assert rc == status


def test_workspace_size_monotone():
    m = _null_module()
    down = _null_module(rows=128, cols=64)
    L = vq.vq_moe_layer(m, m, down)
    a = vq._L().vq_moe_workspace_size(ctypes.byref(L), 4, 1, 0)
    b = vq._L().vq_moe_workspace_size(ctypes.byref(L), 64, 1, 0)
    assert 0 < a < b
    assert vq._L().vq_moe_workspace_size(ctypes.byref(L), 4, 3, 0) == 0   # top_k > E


def test_prefill_chunked_validates_before_launch():
    # fake (never dereferenced) pointers: chunk < 1 fails validation, an empty prompt queues nothing
    m = _null_module()
    down = _null_module(rows=128, cols=64)
    L = vq.vq_moe_layer(m, m, down)
    f = vq._L().vq_moe_prefill_chunked
    assert f(ctypes.byref(L), 4096, 4, 8192, 1, 1, 0, 16384, 0, 65536, 1 << 20, None) == 1
    assert f(ctypes.byref(L), 4096, 4, 8192, 1, 1, -3, 16384, 0, 65536, 1 << 20, None) == 1
    assert f(ctypes.byref(L), None, 0, None, 1, 1, 5, None, 0, 65536, 1 << 20, None) == 0


def test_fit_argument_errors_before_launch():
    # fake (never dereferenced) pointers: every check fails before any CUDA call
    f = vq._L().vq_fit
    ok = dict(w=4096, rows=8, cols=256, d=4, K=8, sample=8192, n=64, init=12288, iters=2, sc=16384, cb=20480,
              codes=24576, ws=65536, nws=1 << 20)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["w"], a["rows"], a["cols"], a["d"], a["K"], a["sample"], a["n"], a["init"], a["iters"], a["sc"],
                 a["cb"], a["codes"], a["ws"], a["nws"], None)
    assert call(d=3) == 1
    assert call(cols=100) == 1
    assert call(K=1) == 1                          # VQ_ERR_ARG
    assert call(K=128) == 1                        # K > n_sample
    assert call(K=8192, n=1 << 14, d=8) == 1       # K * d beyond the shared-memory table
    assert call(w=4098) == 2                       # VQ_ERR_ALIGN
    assert call(ws=65600) == 4                     # VQ_ERR_WORKSPACE (misaligned)
    assert call(nws=16) == 4                       # too small
    assert vq._L().vq_fit_workspace_size(8, 3) == 0
    assert vq._L().vq_fit_workspace_size(512, 4) > 512 * 4 * 12


def test_status_constants_match_header():
    import os
    import re
    text = open(os.path.join(os.path.dirname(vq.__file__), "..", "include", "vq_moe.h")).read()
    enum = dict((n, int(v)) for n, v in re.findall(r"(VQ_(?:OK|ERR_[A-Z_]+)) = (\d+)", text))
    assert len(enum) == 7
    for name, value in enum.items():
        assert getattr(vq, name) == value, name


def test_wait_limit_argument_checked():
    with pytest.raises(vq.VQError):
        vq.set_wait_limit(1 << 33)
    vq.set_wait_limit(0)
    vq.set_wait_limit(None)


def test_gemm_argument_errors_before_launch():
    # fake (never dereferenced) pointers: validation fails before any CUDA call
    f = vq._L().vq_gemm
    m = _null_module()
    other = _null_module(rows=128)
    assert f(ctypes.byref(m), None, 2, 4096, 4, 8192, None, 65536, 1 << 20, None) == 1      # expert out of range
    assert f(ctypes.byref(m), ctypes.byref(other), 0, 4096, 4, 8192, 16384, 65536, 1 << 20, None) == 1   # shapes
    assert f(ctypes.byref(m), ctypes.byref(m), 0, 4096, 4, 8192, None, 65536, 1 << 20, None) == 1   # y1 missing
    assert f(ctypes.byref(m), None, 0, 4098, 4, 8192, None, 65536, 1 << 20, None) == 2      # misaligned x
    assert f(ctypes.byref(m), None, 0, 4096, 4, 8192, None, 65600, 1 << 20, None) == 4      # misaligned workspace
    assert vq._L().vq_gemm_workspace_size(ctypes.byref(m), 4) > 4 * 128 * 2
    assert vq._L().vq_gemm_workspace_size(ctypes.byref(_null_module(d=3)), 4) == 0

