"""Test helpers: build the oracle's and the library's view of the same seeded
inputs. Raw codes are packed separately by each side (oracle.pack vs the
library's vq_pack); large modules share directly drawn packed words."""
from __future__ import annotations

import numpy as np

from synth.workloads import Geometry, ModuleData, module_data


def oracle_module(md: ModuleData):
    import oracle   # imported here so that the library-side helpers never load the oracle
    if md.codes is not None:
        words = oracle.pack(md.codes, md.bits, md.bitmap)
        sc = oracle.compact_rows(md.scales, md.bitmap)
    else:
        words, sc = md.words, md.scales
    return oracle.Module(md.E, md.rows, md.cols, md.d, md.bits, words, sc, md.codebook, md.bitmap)


def lib_module(md: ModuleData, device="cuda"):
    import vector_quantized_moe_b200 as vq
    if md.codes is not None:
        words = vq.pack(md.codes, md.bits, md.bitmap)
        sc = vq.pack_scales(md.scales, md.bitmap)
    else:
        words, sc = md.words, md.scales
    return vq.Module.from_host(md.E, md.rows, md.cols, md.d, md.bits, words, sc, md.codebook, md.bitmap,
                               device=device)


def small_module(E, rows, cols, d, bits, n_dead=0, seed=0):
    return module_data(E, rows, cols, Geometry(d, bits), n_dead, (seed, 99), raw=True)


def row_words_fn():
    import vector_quantized_moe_b200 as vq
    return lambda cols, geo: vq.packed_words(1, cols // geo.d, geo.bits)


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.linalg.norm(ref.ravel()))
    return float(np.linalg.norm((got - ref).ravel())) / (den if den > 0 else 1.0)


def assert_close(got, ref, rel=2e-3, maxfrac=1e-2, what=""):
    """The floating-point bar: relative L2 <= rel and max|err| <= maxfrac * max|ref|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    r = rel_l2(got, ref)
    m = float(np.max(np.abs(got - ref))) if got.size else 0.0
    top = float(np.max(np.abs(ref))) if ref.size else 0.0
    assert r <= rel, f"{what}: relative L2 {r:.3e} > {rel:.1e}"
    assert m <= maxfrac * top + 1e-30, f"{what}: max|err| {m:.3e} > {maxfrac:.0e} * {top:.3e}"
    return r, m
