"""The synthetic workloads: shapes, geometries, seeds and input distributions of
the MoE layers the VQ model cards describe (random numbers only; no method
arithmetic). Packed words are drawn directly for large modules because every
bit pattern of a packed row is a valid row of uniform random codes."""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np

from . import (activations, codebook, live_bitmap, logits_normal, logits_zipf, random_words, raw_codes, rng,
               scales)


@dataclass(frozen=True)
class Geometry:
    d: int
    bits: int


@dataclass(frozen=True)
class LayerSpec:
    name: str
    E: int
    top_k: int
    hidden: int
    inter: int
    gate: Geometry
    up: Geometry
    down: Geometry
    dead_gate: int = 0        # dead output rows per expert (skipzero)
    dead_up: int = 0
    dead_down: int = 0
    zipf_s: Optional[float] = None   # router logits Zipf-skewed with this exponent, else N(0, 1)
    batches: Tuple[int, ...] = ()
    seed: int = 0


@dataclass(frozen=True)
class GemvSpec:
    name: str
    rows: int
    cols: int
    geo: Geometry
    T: int = 1
    seed: int = 0


D2K256 = Geometry(2, 8)
D2K1024 = Geometry(2, 10)
D4K512 = Geometry(4, 9)
D4K2048 = Geometry(4, 11)
D8K4096 = Geometry(8, 12)

# Single VQ GEMV: 512 x 1024, d=2, K=256, one token.
GEMV_D2K256 = GemvSpec("gemv_d2k256_512x1024", 512, 1024, D2K256, 1, 0)

# MoE decode, d=2/K=256 everywhere: 512 experts top-10, hidden 4096, inter 1024.
DECODE_D2K256 = LayerSpec("moe_decode_d2k256_e512k10_h4096_i1024", 512, 10, 4096, 1024, D2K256, D2K256, D2K256,
                          batches=(1, 8), seed=0)

# MoE decode, d=4/K=512 (9-bit) and the promoted d=4/K=2048 (11-bit) layer:
# 256 experts top-8, hidden 6144, inter 2048, 16 tokens.
DECODE_D4K512 = LayerSpec("moe_decode_d4k512_e256k8_h6144_i2048", 256, 8, 6144, 2048, D4K512, D4K512, D4K512,
                          batches=(16,), seed=0)
DECODE_D4K2048 = LayerSpec("moe_decode_d4k2048_e256k8_h6144_i2048", 256, 8, 6144, 2048, D4K2048, D4K2048, D4K2048,
                           batches=(16,), seed=1)

# MoE prefill, d=4/K=512: 4096 tokens, 256 experts top-8 with Zipf(1.1) router logits.
PREFILL_D4K512 = LayerSpec("moe_prefill_d4k512_e256k8_h6144_i2048_zipf1.1", 256, 8, 6144, 2048, D4K512, D4K512,
                           D4K512, zipf_s=1.1, batches=(4096,), seed=0)

# Skipzero + mixed geometry: gate/up d=2/K=1024 with 127 of 1024 rows dead
# (12.43%), down d=8/K=4096; 512 experts top-10, hidden 4096, inter 1024.
SKIPZERO_MIXED = LayerSpec("moe_skipzero_d2k1024_d8k4096_e512k10_h4096_i1024", 512, 10, 4096, 1024, D2K1024, D2K1024,
                           D8K4096, dead_gate=127, dead_up=127, batches=(1, 2048), seed=0)

ALL_LAYERS = (DECODE_D2K256, DECODE_D4K512, DECODE_D4K2048, PREFILL_D4K512, SKIPZERO_MIXED)


@dataclass
class ModuleData:
    """Host arrays of one module. `codes` (raw, [E, rows, ncode]) is set for
    raw draws; `words` (packed live rows) for direct word draws."""
    E: int
    rows: int
    cols: int
    d: int
    bits: int
    codebook: np.ndarray
    scales: np.ndarray                 # [E, rows, cols/64] (raw) or [live rows, cols/64] (words)
    bitmap: Optional[np.ndarray] = None
    codes: Optional[np.ndarray] = None
    words: Optional[np.ndarray] = None


def module_data(E: int, rows: int, cols: int, geo: Geometry, n_dead: int, seed: Tuple[int, ...],
                raw: bool, row_words: Optional[int] = None) -> ModuleData:
    """One module's seeded inputs. raw=True draws codes [E, rows, cols/d] and
    full scales; raw=False draws `row_words` packed words per live row."""
    g = rng(*seed)
    cb = codebook(1 << geo.bits, geo.d, g)
    bm = live_bitmap(E, rows, n_dead, g) if n_dead else None
    ngroups = cols // 64
    if raw:
        codes = raw_codes((E, rows, cols // geo.d), geo.bits, g)
        sc = scales(E * rows, ngroups, g).reshape(E, rows, ngroups)
        return ModuleData(E, rows, cols, geo.d, geo.bits, cb, sc, bm, codes=codes)
    assert row_words is not None
    n_live = E * (rows - n_dead)
    words = random_words(n_live, row_words, g)
    sc = scales(n_live, ngroups, g)
    return ModuleData(E, rows, cols, geo.d, geo.bits, cb, sc, bm, words=words)


def layer_inputs(spec: LayerSpec, T: int, seed_offset: int = 0):
    """(x bf16 bits [T, hidden], router logits fp32 [T, E]) for a batch of T tokens."""
    g = rng(spec.seed, 1000 + seed_offset, T)
    x = activations(T, spec.hidden, g)
    if spec.zipf_s is not None:
        lg = logits_zipf(T, spec.E, spec.zipf_s, g)
    else:
        lg = logits_normal(T, spec.E, g)
    return x, lg


def layer_modules(spec: LayerSpec, raw: bool, row_words=None):
    """gate, up, down ModuleData. row_words(cols, geo) gives packed words per row when raw=False."""
    out = []
    for i, (rows, cols, geo, dead) in enumerate(((spec.inter, spec.hidden, spec.gate, spec.dead_gate),
                                                  (spec.inter, spec.hidden, spec.up, spec.dead_up),
                                                  (spec.hidden, spec.inter, spec.down, spec.dead_down))):
        rw = None if raw else row_words(cols, geo)
        out.append(module_data(spec.E, rows, cols, geo, dead, (spec.seed, i), raw, rw))
    return out
