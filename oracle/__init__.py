"""CPU oracle for the VQ-MoE expert path (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this package. The CUDA library never does, and nothing here
imports the library: the two share no code.

The arithmetic lives in vq_oracle.c (plain C, double precision); this file
builds it with gcc and marshals numpy arrays through ctypes. The data-free
VQ fit (k-means over weight subvectors) is oracle/fit.py, plain numpy. Each function
says which passage of the VQ model cards it follows; the readings of silent
points are listed in vq_oracle.c's header and in fit.py's.

Parity status: every function below is pinned by tests/test_oracle.py against
closed forms, library routines, hand-worked fixtures or brute force, except
the end-to-end MoE layer on real checkpoints (no real artifacts exist here),
which is "parity unpinned" against the pages' own models.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vq_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libvqoracle.so")


def build(force: bool = False) -> str:
    """Compile vq_oracle.c into oracle/_build/libvqoracle.so (gcc, OpenMP)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                           "-Wall", "-Wno-unknown-pragmas", _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


class _Module(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int32), ("rows", ctypes.c_int32), ("cols", ctypes.c_int32),
                ("d", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("words", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("codebook", ctypes.c_void_p), ("bitmap", ctypes.c_void_p), ("biases", ctypes.c_void_p)]


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.vqo_f16_to_f64.restype = ctypes.c_double
        lib.vqo_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.vqo_bf16_to_f64.restype = ctypes.c_double
        lib.vqo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.vqo_f64_to_bf16.restype = ctypes.c_uint16
        lib.vqo_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.vqo_row_words.restype = ctypes.c_size_t
        lib.vqo_row_words.argtypes = [I, I]
        lib.vqo_pack_row.argtypes = [P, I, I, P]
        lib.vqo_unpack_row.argtypes = [P, I, I, P]
        lib.vqo_pack.restype = ctypes.c_long
        lib.vqo_pack.argtypes = [P, I, I, I, I, P, P]
        lib.vqo_compact_u16.restype = ctypes.c_long
        lib.vqo_compact_u16.argtypes = [P, I, I, I, P, P]
        lib.vqo_dequant.argtypes = [ctypes.POINTER(_Module), I, P]
        lib.vqo_gemv.argtypes = [ctypes.POINTER(_Module), I, P, I, P]
        lib.vqo_route.restype = I
        lib.vqo_route.argtypes = [P, I, I, I, I, P, P, P, P, P]
        lib.vqo_moe.restype = I
        lib.vqo_moe.argtypes = [ctypes.POINTER(_Module)] * 3 + [I, I, P, P, I, I, I, P, I, P]
        lib.vqo_num_threads.restype = I
        lib.vqo_set_num_threads.argtypes = [I]
        lib.vqo_set_num_threads.restype = None
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return _L().vqo_num_threads()


def set_num_threads(n: int) -> None:
    """OpenMP threads for the oracle's loops (the CPU baseline times one and all)."""
    _L().vqo_set_num_threads(int(n))


def f16_to_f64(bits) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).ravel()
    f = _L().vqo_f16_to_f64
    return np.array([f(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def bf16_to_f64(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).ravel()
    f = _L().vqo_bf16_to_f64
    return np.array([f(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def f64_to_bf16(vals) -> np.ndarray:
    """float64 -> bfloat16 bit patterns, round to nearest even."""
    v = np.asarray(vals, dtype=np.float64).ravel()
    f = _L().vqo_f64_to_bf16
    return np.array([f(float(x)) for x in v], dtype=np.uint16).reshape(np.shape(vals))


def row_words(ncode: int, bits: int) -> int:
    """uint32 words of one packed row (ncode a multiple of 32)."""
    return int(_L().vqo_row_words(ncode, bits))


def pack(codes: np.ndarray, bits: int, bitmap: Optional[np.ndarray] = None) -> np.ndarray:
    """Pack uint16 codes [E, rows, ncode] (or [rows, ncode]) into the live rows'
    words [live_rows, row_words]; dead rows (bitmap bit 0) are dropped."""
    c = _c(codes, np.uint16)
    if c.ndim == 2:
        c = c[None]
    E, rows, ncode = c.shape
    assert ncode % 32 == 0
    nw = row_words(ncode, bits)
    bm = None if bitmap is None else _c(bitmap, np.uint32)
    out = np.zeros((E * rows, nw), dtype=np.uint32)
    n = _L().vqo_pack(_p(c), E, rows, ncode, bits, _p(bm), _p(out))
    return out[:n]


def unpack_row(words: np.ndarray, ncode: int, bits: int) -> np.ndarray:
    """Codes of one packed row."""
    w = _c(words, np.uint32)
    out = np.zeros(ncode, dtype=np.uint16)
    _L().vqo_unpack_row(_p(w), ncode, bits, _p(out))
    return out


def unpack(words: np.ndarray, ncode: int, bits: int) -> np.ndarray:
    """Codes [n_rows, ncode] of packed rows [n_rows, row_words]."""
    w = _c(words, np.uint32)
    return np.stack([unpack_row(w[i], ncode, bits) for i in range(w.shape[0])]) if w.shape[0] else \
        np.zeros((0, ncode), dtype=np.uint16)


def compact_rows(a: np.ndarray, bitmap: Optional[np.ndarray]) -> np.ndarray:
    """Keep the live rows of a uint16 per-row array [E, rows, n] (skipzero)."""
    x = _c(a, np.uint16)
    E, rows, n = x.shape
    out = np.zeros((E * rows, n), dtype=np.uint16)
    bm = None if bitmap is None else _c(bitmap, np.uint32)
    k = _L().vqo_compact_u16(_p(x), E, rows, n, _p(bm), _p(out))
    return out[:k]


@dataclass
class Module:
    """One VQ module (a (layer, projection) tensor shared by E experts).

    words: packed live rows [n_live, row_words] uint32, expert-major
    scales: fp16 bits [n_live, cols // 64]
    codebook: fp16 bits [2**bits, d]
    bitmap: uint32 [E, ceil(rows / 32)] or None (all rows live)
    biases: fp16 bits [n_live, cols // 64] or None: an affine offset per group (w = s * C[q] + b)
    """
    E: int
    rows: int
    cols: int
    d: int
    bits: int
    words: np.ndarray
    scales: np.ndarray
    codebook: np.ndarray
    bitmap: Optional[np.ndarray] = None
    biases: Optional[np.ndarray] = None

    def _struct(self):
        self._keep = (_c(self.words, np.uint32), _c(self.scales, np.uint16), _c(self.codebook, np.uint16),
                      None if self.bitmap is None else _c(self.bitmap, np.uint32),
                      None if self.biases is None else _c(self.biases, np.uint16))
        w, s, cb, bm, b = self._keep
        return _Module(self.E, self.rows, self.cols, self.d, self.bits, _p(w), _p(s), _p(cb), _p(bm), _p(b))


def dequant(m: Module, e: int) -> np.ndarray:
    """Dense weights [rows, cols] of expert e (float64, exact); dead rows 0."""
    W = np.zeros((m.rows, m.cols), dtype=np.float64)
    s = m._struct()
    _L().vqo_dequant(ctypes.byref(s), e, _p(W))
    return W


def gemv(m: Module, e: int, x_bf16: np.ndarray) -> np.ndarray:
    """y [T, rows] = x [T, cols] . W_e^T accumulated in float64."""
    x = _c(x_bf16, np.uint16)
    T = x.shape[0]
    y = np.zeros((T, m.rows), dtype=np.float64)
    s = m._struct()
    _L().vqo_gemv(ctypes.byref(s), e, _p(x), T, _p(y))
    return y


def route(logits: np.ndarray, k: int, renorm: bool = True):
    """Top-k routing and expert bucketing.

    Returns ids [T, k] int32, w [T, k] float64, counts [E], offsets [E+1],
    perm [T*k] (pair p = t*k + j, grouped by expert, increasing p per expert).
    """
    l = _c(logits, np.float32)
    T, E = l.shape
    ids = np.zeros((T, k), dtype=np.int32)
    w = np.zeros((T, k), dtype=np.float64)
    counts = np.zeros(E, dtype=np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    perm = np.zeros(T * k, dtype=np.int32)
    rc = _L().vqo_route(_p(l), T, E, k, int(bool(renorm)), _p(ids), _p(w), _p(counts), _p(offsets), _p(perm))
    if rc != 0:
        raise ValueError("bad routing arguments")
    return ids, w, counts, offsets, perm


def moe(gate: Module, up: Module, down: Module, x_bf16: np.ndarray, logits: np.ndarray, k: int,
        renorm: bool = True, tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """MoE SwiGLU layer outputs y [len(tokens), hidden] in float64 for the
    listed tokens (all tokens when None)."""
    x = _c(x_bf16, np.uint16)
    l = _c(logits, np.float32)
    T, H = x.shape
    E = l.shape[1]
    tok = np.arange(T, dtype=np.int32) if tokens is None else _c(tokens, np.int32)
    y = np.zeros((len(tok), H), dtype=np.float64)
    sg, su, sd = gate._struct(), up._struct(), down._struct()
    rc = _L().vqo_moe(ctypes.byref(sg), ctypes.byref(su), ctypes.byref(sd), H, gate.rows, _p(x), _p(l), E,
                      k, int(bool(renorm)), _p(tok), len(tok), _p(y))
    if rc != 0:
        raise ValueError("bad MoE arguments")
    return y
