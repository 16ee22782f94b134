"""CPU oracle of the data-free VQ fit (test infrastructure; see oracle/__init__.py
for who may use it). Plain numpy, float32 where the method decides an integer
(a code), float64 / exact integers elsewhere.

What the VQ model cards state ("Methodology" of Qwen3.5-397B-A17B-VQ-2.6bpw,
Qwen3.8-Flash-Next-VQ-4.4bpw and GLM-5.3-Flash-VQ-2.7bpw): codebooks are fit in pure
weight space by k-means / Lloyd over the weight subvectors (d consecutive
weights of a row), with no Hessian, activation statistics or calibration data;
k-means runs on a drawn subsample; each subvector stores the index of one
entry of a per-tensor fp16 codebook of K entries, and each (row, 64 weights)
group has an fp16 scale.

Readings of what the cards leave open:
  F1 scale: s[r, g] = fp16(max |w| over the group's 64 weights); the
     subvector the codebook sees is v = w / s (fp32), v = 0 where s = 0.
  F2 distance: squared Euclidean in fp32, sum over components in order,
     each difference, square and sum rounded on its own (no fused multiply-add);
     ties go to the lower index.
  F3 Lloyd step: every sample point goes to its nearest centroid; a centroid
     with points becomes their mean, computed exactly (each component as a
     fixed-point integer round(v * 2^40), summed exactly, then
     fp32(sum * 2^-40 / count) in fp64); a centroid with none keeps its value.
  F4 the subsample and the K initial centroids (sample points) are drawn by
     the caller and passed in; the cards' fit is unseeded or seeded at 1234.
  F5 after the iterations the codebook is rounded to fp16, and every subvector
     of the tensor takes the index of its nearest fp16 entry (F2).
"""
from __future__ import annotations

import numpy as np

FIX_SHIFT = 40   # fixed-point fraction bits of the exact centroid sums (F3)


def bf16_to_f32(w_bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to float32, exactly."""
    return (w_bits.astype(np.uint32) << 16).view(np.float32)


def fit_scales(w_bits: np.ndarray) -> np.ndarray:
    """F1: fp16 scale per (row, 64 weights) = the group's largest |w|. Returns
    fp16 bit patterns (uint16) [rows, cols / 64]."""
    w = bf16_to_f32(w_bits)
    rows, cols = w.shape
    amax = np.abs(w).reshape(rows, cols // 64, 64).max(axis=2)
    return amax.astype(np.float16).view(np.uint16)


def subvectors(w_bits: np.ndarray, scales_bits: np.ndarray, d: int) -> np.ndarray:
    """F1: all normalised subvectors v [rows * cols / d, d] (fp32), row-major:
    subvector i = (row i // (cols/d), weights d*(i % (cols/d)) .. + d)."""
    w = bf16_to_f32(w_bits)
    rows, cols = w.shape
    s = np.repeat(scales_bits.view(np.float16).astype(np.float32), 64, axis=1)   # [rows, cols]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s != 0, w / np.where(s != 0, s, np.float32(1)), np.float32(0)).astype(np.float32)
    return v.reshape(rows * (cols // d), d)


def sq_dist(v: np.ndarray, c: np.ndarray) -> np.ndarray:
    """F2: [n, K] fp32 squared distances, component by component, unfused."""
    acc = np.zeros((v.shape[0], c.shape[0]), dtype=np.float32)
    for t in range(v.shape[1]):
        diff = (v[:, None, t] - c[None, :, t]).astype(np.float32)
        acc = (acc + (diff * diff).astype(np.float32)).astype(np.float32)
    return acc


def nearest(v: np.ndarray, c: np.ndarray, chunk: int = 4096) -> np.ndarray:
    """F2: index of the nearest centroid of each row of v (first of equals)."""
    out = np.empty(v.shape[0], dtype=np.int64)
    for i in range(0, v.shape[0], chunk):
        out[i:i + chunk] = np.argmin(sq_dist(v[i:i + chunk], c), axis=1)
    return out


def lloyd_step(v: np.ndarray, c: np.ndarray):
    """F3: one assignment + update. Returns (new centroids, assignment)."""
    a = nearest(v, c)
    K, d = c.shape
    q = np.rint(v * np.float32(2.0 ** FIX_SHIFT)).astype(np.int64)   # exact: |v| <= 1
    sums = np.zeros((K, d), dtype=np.int64)
    np.add.at(sums, a, q)
    cnt = np.bincount(a, minlength=K).astype(np.int64)
    new = c.copy()
    has = cnt > 0
    mean = (sums[has].astype(np.float64) * 2.0 ** -FIX_SHIFT) / cnt[has, None].astype(np.float64)
    new[has] = mean.astype(np.float32)
    return new, a


def fit(w_bits: np.ndarray, d: int, K: int, sample: np.ndarray, init: np.ndarray, iters: int):
    """The whole fit of one tensor: F1 scales, F3 Lloyd on the sample points
    (subvector indices `sample`, initial centroids = subvectors `init`),
    F5 fp16 codebook and codes of every subvector.
    Returns (scales fp16 bits [rows, cols/64], codebook fp16 bits [K, d],
    codes uint16 [rows, cols/d], centroid history [iters + 1][K, d] fp32)."""
    rows, cols = w_bits.shape
    sc = fit_scales(w_bits)
    v_all = subvectors(w_bits, sc, d)
    v = v_all[sample]
    c = v_all[init].copy()
    hist = [c.copy()]
    for _ in range(iters):
        c, _ = lloyd_step(v, c)
        hist.append(c.copy())
    cb = c.astype(np.float16)
    codes = nearest(v_all, cb.astype(np.float32)).astype(np.uint16).reshape(rows, cols // d)
    return sc, cb.view(np.uint16), codes, hist


def sse(v: np.ndarray, c: np.ndarray) -> float:
    """Sum over points of the squared distance to the nearest centroid, in fp64."""
    a = nearest(v, c)
    diff = v.astype(np.float64) - c[a].astype(np.float64)
    return float((diff * diff).sum())
