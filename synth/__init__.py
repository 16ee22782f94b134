"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module only draws random numbers and stores them in the bit formats the
VQ-MoE layer consumes (fp16 codebooks and scales, bf16 activations, fp32
router logits, uint16 raw codes, uint32 packed words, uint32 live-row bitmaps).
It holds none of the method's arithmetic: no packing, unpacking, dequantisation,
routing or matmul. Sizes that depend on the packed format (words per row) are
passed in by the caller.

Distributions follow the workloads of the VQ-MoE model cards:
  * codebook entries N(0, 0.02) stored as fp16,
  * group scales U(0.5, 2) stored as fp16 (one per row and 64 weights),
  * codes uniform over the K = 2**bits codebook entries,
  * activations N(0, 1) stored as bf16,
  * router logits N(0, 1) fp32, or Zipf(s)-skewed: -s*ln(rank_e) + Gumbel(0, 1),
  * skipzero: a seeded random set of dead output rows per (expert, module),
  * expert weights for the data-free fit: N(0, 0.02) stored as bf16 (a bf16
    checkpoint), the k-means subsample and its initial centroids drawn as
    subvector indices.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rng", "bf16_bits", "f16_bits", "codebook", "scales", "biases", "raw_codes",
    "live_bitmap", "random_words", "activations", "activations_scaled", "logits_normal", "logits_zipf",
    "weights", "fit_draw",
]


def rng(*seed: int) -> np.random.Generator:
    """A PCG64 generator from an entropy tuple, e.g. rng(seed, module_id)."""
    return np.random.default_rng(np.random.SeedSequence(list(seed)))


def bf16_bits(a) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(a, dtype=np.float32))
    if nan.any():
        r[nan] = 0x7FC0
    return r


def f16_bits(a) -> np.ndarray:
    """Values -> IEEE binary16 bit patterns (uint16), numpy's round to nearest even."""
    return np.asarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def codebook(K: int, d: int, g: np.random.Generator, sigma: float = 0.02) -> np.ndarray:
    """fp16 codebook [K, d] with entries N(0, sigma)."""
    return f16_bits(g.normal(0.0, sigma, size=(K, d)).astype(np.float32))


def scales(n_rows: int, n_groups: int, g: np.random.Generator, lo: float = 0.5, hi: float = 2.0) -> np.ndarray:
    """fp16 group scales [n_rows, n_groups] drawn U(lo, hi)."""
    return f16_bits(g.uniform(lo, hi, size=(n_rows, n_groups)).astype(np.float32))


def biases(n_rows: int, n_groups: int, g: np.random.Generator, sigma: float = 0.02) -> np.ndarray:
    """fp16 group biases [n_rows, n_groups] drawn N(0, sigma) (the affine arm's offsets)."""
    return f16_bits(g.normal(0.0, sigma, size=(n_rows, n_groups)).astype(np.float32))


def raw_codes(shape, bits: int, g: np.random.Generator) -> np.ndarray:
    """uint16 codes uniform over [0, 2**bits)."""
    return g.integers(0, 1 << bits, size=shape, dtype=np.uint16)


def live_bitmap(E: int, rows: int, n_dead: int, g: np.random.Generator) -> np.ndarray:
    """uint32 [E, ceil(rows/32)]; bit (r % 32) of word r // 32 is 1 when row r is live.

    Exactly n_dead rows per expert are dead, chosen by a seeded permutation.
    Bits beyond `rows` in the last word are 0.
    """
    nw = (rows + 31) // 32
    out = np.zeros((E, nw), dtype=np.uint32)
    for e in range(E):
        live = np.ones(rows, dtype=bool)
        live[g.permutation(rows)[:n_dead]] = False
        padded = np.zeros(nw * 32, dtype=np.uint64)
        padded[:rows] = live
        w = padded.reshape(nw, 32) << np.arange(32, dtype=np.uint64)
        out[e] = w.sum(axis=1).astype(np.uint32)
    return out


def random_words(n_rows: int, words_per_row: int, g: np.random.Generator) -> np.ndarray:
    """Uniform random uint32 words [n_rows, words_per_row].

    Every bit pattern of a packed row is a valid row of uniform random codes
    when the row has no padding bits, so this draws packed codes directly for
    large workloads without materialising the raw codes.
    """
    return g.integers(0, 1 << 32, size=(n_rows, words_per_row), dtype=np.uint32)


def activations(T: int, H: int, g: np.random.Generator) -> np.ndarray:
    """bf16 activations [T, H] drawn N(0, 1)."""
    return bf16_bits(g.standard_normal((T, H), dtype=np.float32))


def activations_scaled(T: int, H: int, g: np.random.Generator, log2_token=None, log2_group=None,
                       outliers=()) -> np.ndarray:
    """bf16 activations [T, H] over bf16's range (the bf16 I/O of the cards'
    runtime): N(0, 1) times 2**log2_token[t] times 2**log2_group[t, c // 64]
    (integer exponents; each factor is exact), then each (t, c, value) of
    `outliers` written over its element, all rounded to bf16."""
    x = g.standard_normal((T, H)).astype(np.float32).astype(np.float64)
    if log2_token is not None:
        x = x * np.exp2(np.asarray(log2_token, dtype=np.float64))[:, None]
    if log2_group is not None:
        x = x * np.repeat(np.exp2(np.asarray(log2_group, dtype=np.float64)), 64, axis=1)
    for t, c, v in outliers:
        x[t, c] = v
    return bf16_bits(x.astype(np.float32))


def logits_normal(T: int, E: int, g: np.random.Generator) -> np.ndarray:
    """fp32 router logits [T, E] drawn N(0, 1)."""
    return g.standard_normal((T, E), dtype=np.float32)


def logits_zipf(T: int, E: int, s: float, g: np.random.Generator) -> np.ndarray:
    """Zipf(s)-skewed router logits: -s*ln(rank_e) + Gumbel(0, 1) noise.

    rank is a seeded permutation of 1..E, so top-k of a row is a draw without
    replacement from Zipf(s) over the experts (Gumbel-top-k).
    """
    rank = g.permutation(E).astype(np.float64) + 1.0
    base = -s * np.log(rank)
    gum = g.gumbel(0.0, 1.0, size=(T, E))
    return (base[None, :] + gum).astype(np.float32)


def weights(rows: int, cols: int, g: np.random.Generator, sigma: float = 0.02) -> np.ndarray:
    """A bf16 weight tensor [rows, cols] (bit patterns), entries N(0, sigma)."""
    return bf16_bits(g.normal(0.0, sigma, size=(rows, cols)))


def fit_draw(n_sub: int, n_sample: int, K: int, g: np.random.Generator):
    """The k-means subsample (n_sample distinct subvector indices, sorted) and
    K distinct initial centroids drawn from it (subvector indices), int32."""
    sample = np.sort(g.choice(n_sub, size=n_sample, replace=False)).astype(np.int32)
    init = sample[g.choice(n_sample, size=K, replace=False)].astype(np.int32)
    return sample, init
