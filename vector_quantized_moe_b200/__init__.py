"""Python binding of libvqmoe.so, the B200 (sm_100a) VQ-MoE expert-path library.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels; PyTorch provides device memory and streams. The library is loaded on
first use; every call raises ImportError when it has not been built
(python -m vector_quantized_moe_b200.build). There is no fallback.

Names follow include/vq_moe.h.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvqmoe.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "vq_moe.h")

VQ_OK = 0
VQ_ERR_ARG, VQ_ERR_ALIGN, VQ_ERR_UNSUPPORTED, VQ_ERR_WORKSPACE, VQ_ERR_CUDA, VQ_ERR_DEVICE_CHECK = 1, 2, 3, 4, 5, 6
VQ_F32, VQ_BF16 = 0, 1
VQ_MODE_DECODE, VQ_MODE_PREFILL = 0, 1


class VQError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {_L().vq_status_str(status).decode()}")
        self.status = status


class vq_module(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int32), ("rows", ctypes.c_int32), ("cols", ctypes.c_int32),
                ("d", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("codebook", ctypes.c_void_p),
                ("live_bitmap", ctypes.c_void_p), ("live_rank", ctypes.c_void_p), ("live_rows", ctypes.c_int64),
                ("biases", ctypes.c_void_p)]


class vq_moe_layer(ctypes.Structure):
    _fields_ = [("gate", vq_module), ("up", vq_module), ("down", vq_module)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m vector_quantized_moe_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_int64
    MP = ctypes.POINTER(vq_module)
    LP = ctypes.POINTER(vq_moe_layer)
    sig = {
        "vq_status_str": (ctypes.c_char_p, [ctypes.c_int]),
        "vq_geometry_supported": (ctypes.c_int, [I32, I32]),
        "vq_packed_words": (SZ, [I64, I32, I32]),
        "vq_pack": (ctypes.c_int, [P, I32, I32, I32, I32, P, P, SZ, ctypes.POINTER(SZ)]),
        "vq_pack_scales": (ctypes.c_int, [P, I32, I32, I32, P, P, SZ, ctypes.POINTER(SZ)]),
        "vq_live_rank": (ctypes.c_int, [P, I32, I32, P]),
        "vq_unpack": (ctypes.c_int, [MP, I32, P, P]),
        "vq_dequant": (ctypes.c_int, [MP, I32, P, P]),
        "vq_gemv": (ctypes.c_int, [MP, I32, P, I32, P, I32, P]),
        "vq_gemm_workspace_size": (SZ, [MP, I32]),
        "vq_gemm": (ctypes.c_int, [MP, MP, I32, P, I32, P, P, P, SZ, P]),
        "vq_route": (ctypes.c_int, [P, I32, I32, I32, I32, P, P, P, P, P]),
        "vq_moe_workspace_size": (SZ, [LP, I32, I32, I32]),
        "vq_moe_decode": (ctypes.c_int, [LP, P, I32, P, I32, I32, P, I32, P, SZ, P]),
        "vq_moe_prefill": (ctypes.c_int, [LP, P, I32, P, I32, I32, P, I32, P, SZ, P]),
        "vq_moe_prefill_chunked": (ctypes.c_int, [LP, P, I32, P, I32, I32, I32, P, I32, P, SZ, P]),
        "vq_set_trace_events": (ctypes.c_int, [P, I32]),
        "vq_set_wait_limit": (ctypes.c_int, [I64]),
        "vq_moe_check": (ctypes.c_int, [P, P]),
        "vq_moe_decode_noalloc": (ctypes.c_int, [LP, P, I32, P, I32, I32, P, I32, P]),
        "vq_fit_workspace_size": (SZ, [I32, I32]),
        "vq_fit": (ctypes.c_int, [P, I32, I32, I32, I32, P, I32, P, I32, P, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib_handle = None


def _L():
    """The loaded libvqmoe.so (loads it on first use; raises ImportError if missing)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


def header_functions() -> list:
    """Names of the functions include/vq_moe.h declares."""
    txt = open(HEADER_PATH).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(vq_[a-z_0-9]+)\s*\(", txt)))


def _check(status: int, where: str):
    if status != VQ_OK:
        raise VQError(status, where)


def status_str(status: int) -> str:
    return _L().vq_status_str(status).decode()


def geometry_supported(d: int, bits: int) -> bool:
    return bool(_L().vq_geometry_supported(d, bits))


def packed_words(rows: int, ncode: int, bits: int) -> int:
    return int(_L().vq_packed_words(rows, ncode, bits))


# ------------------------------------------------------------------ host packing

def pack(codes: np.ndarray, bits: int, live_bitmap: Optional[np.ndarray] = None) -> np.ndarray:
    """Pack uint16 codes [E, rows, ncode] -> words [live rows, row_words] (vq_pack)."""
    c = np.ascontiguousarray(codes, dtype=np.uint16)
    if c.ndim == 2:
        c = c[None]
    E, rows, ncode = c.shape
    bm = None if live_bitmap is None else np.ascontiguousarray(live_bitmap, dtype=np.uint32)
    rw = packed_words(1, ncode, bits)
    out = np.zeros((E * rows, max(rw, 1)), dtype=np.uint32)
    n = ctypes.c_size_t(0)
    _check(_L().vq_pack(c.ctypes.data, E, rows, ncode, bits, None if bm is None else bm.ctypes.data,
                        out.ctypes.data, out.size, ctypes.byref(n)), "vq_pack")
    return out[: n.value]


def pack_scales(scales: np.ndarray, live_bitmap: Optional[np.ndarray] = None) -> np.ndarray:
    """Keep the live rows of fp16 scales [E, rows, ngroups] (vq_pack_scales)."""
    s = np.ascontiguousarray(scales, dtype=np.uint16)
    E, rows, ng = s.shape
    bm = None if live_bitmap is None else np.ascontiguousarray(live_bitmap, dtype=np.uint32)
    out = np.zeros((E * rows, ng), dtype=np.uint16)
    n = ctypes.c_size_t(0)
    _check(_L().vq_pack_scales(s.ctypes.data, E, rows, ng, None if bm is None else bm.ctypes.data,
                               out.ctypes.data, out.size, ctypes.byref(n)), "vq_pack_scales")
    return out[: n.value]


def live_rank(live_bitmap: np.ndarray, rows: int) -> np.ndarray:
    """Rank table [E, ceil(rows/32)] for a live bitmap (vq_live_rank)."""
    bm = np.ascontiguousarray(live_bitmap, dtype=np.uint32)
    out = np.zeros_like(bm)
    _check(_L().vq_live_rank(bm.ctypes.data, bm.shape[0], rows, out.ctypes.data), "vq_live_rank")
    return out


# ------------------------------------------------------------------ device side

def _torch():
    import torch
    return torch


def _stream(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


class Module:
    """One VQ module on the device (vq_module). Tensors are kept alive here."""

    def __init__(self, E, rows, cols, d, bits, codes, scales, codebook, live_bitmap=None, live_rank_t=None,
                 biases=None):
        self.E, self.rows, self.cols, self.d, self.bits = E, rows, cols, d, bits
        self.codes, self.scales, self.codebook = codes, scales, codebook
        self.live_bitmap, self.live_rank = live_bitmap, live_rank_t
        self.biases = biases

    @classmethod
    def from_host(cls, E, rows, cols, d, bits, words, scales, codebook, live_bitmap=None, device="cuda",
                  biases=None):
        """Upload packed words [live rows, row_words], fp16 scale bits [live rows, cols/64],
        fp16 codebook bits [2^bits, d], an optional live bitmap [E, ceil(rows/32)] and optional
        fp16 bias bits [live rows, cols/64] (the affine arm)."""
        torch = _torch()
        up = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)
        bm = rk = None
        if live_bitmap is not None:
            bm = up(live_bitmap.astype(np.uint32), np.int32)
            rk = up(live_rank(live_bitmap, rows), np.int32)
        return cls(E, rows, cols, d, bits, up(words.astype(np.uint32), np.int32), up(scales, np.int16),
                   up(codebook, np.int16), bm, rk, None if biases is None else up(biases, np.int16))

    def struct(self) -> vq_module:
        return vq_module(self.E, self.rows, self.cols, self.d, self.bits, _ptr(self.codes), _ptr(self.scales),
                         _ptr(self.codebook), _ptr(self.live_bitmap), _ptr(self.live_rank),
                         int(self.scales.shape[0]), _ptr(self.biases))


def unpack(m: Module, expert: int, stream=None):
    """Codes [rows, cols/d] (uint16 bits in an int16 tensor); dead rows 0xFFFF (vq_unpack)."""
    torch = _torch()
    out = torch.empty((m.rows, m.cols // m.d), dtype=torch.int16, device=m.codes.device)
    s = m.struct()
    _check(_L().vq_unpack(ctypes.byref(s), expert, out.data_ptr(), _stream(stream)), "vq_unpack")
    return out


def dequant(m: Module, expert: int, stream=None):
    """Dequantised weights [rows, cols] fp32 (vq_dequant)."""
    torch = _torch()
    out = torch.empty((m.rows, m.cols), dtype=torch.float32, device=m.codes.device)
    s = m.struct()
    _check(_L().vq_dequant(ctypes.byref(s), expert, out.data_ptr(), _stream(stream)), "vq_dequant")
    return out


def _dt(out_dtype):
    torch = _torch()
    return VQ_F32 if out_dtype == torch.float32 else VQ_BF16


def gemv(m: Module, expert: int, x, out_dtype=None, out=None, stream=None):
    """y [T, rows] = x [T, cols] (bf16) . W_expert^T (vq_gemv)."""
    torch = _torch()
    out_dtype = out_dtype or torch.float32
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, m.rows), dtype=out_dtype, device=x.device)
    s = m.struct()
    _check(_L().vq_gemv(ctypes.byref(s), expert, x.data_ptr(), T, out.data_ptr(), _dt(out.dtype), _stream(stream)),
           "vq_gemv")
    return out


def gemm(m0: Module, expert: int, x, m1: Optional[Module] = None, workspace=None, stream=None):
    """The prefill path's tcgen05 GEMM for one expert (vq_gemm): y0 [T, rows] = x . W0_expert^T and,
    with m1, y1 = x . W1_expert^T (fp32). Returns (y0, y1 or None, workspace)."""
    torch = _torch()
    T = x.shape[0]
    y0 = torch.empty((T, m0.rows), dtype=torch.float32, device=x.device)
    y1 = torch.empty((T, m0.rows), dtype=torch.float32, device=x.device) if m1 is not None else None
    s0 = m0.struct()
    s1 = m1.struct() if m1 is not None else None
    n = int(_L().vq_gemm_workspace_size(ctypes.byref(s0), T))
    if n == 0:
        raise VQError(VQ_ERR_ARG, "vq_gemm_workspace_size")
    ws = workspace if workspace is not None else torch.empty(n + 256, dtype=torch.uint8, device=x.device)
    base = ws.data_ptr()
    aligned = (base + 255) // 256 * 256
    _check(_L().vq_gemm(ctypes.byref(s0), None if s1 is None else ctypes.byref(s1), expert, x.data_ptr(), T,
                        y0.data_ptr(), _ptr(y1), aligned, ws.numel() - (aligned - base), _stream(stream)), "vq_gemm")
    return y0, y1, ws


def route(logits, top_k: int, renorm: bool = True, stream=None):
    """(ids [T,k] int32, weights [T,k] fp32, offsets [E+1] int32, perm [T*k] int32) (vq_route)."""
    torch = _torch()
    T, E = logits.shape
    dev = logits.device
    ids = torch.empty((T, top_k), dtype=torch.int32, device=dev)
    w = torch.empty((T, top_k), dtype=torch.float32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * top_k, dtype=torch.int32, device=dev)
    _check(_L().vq_route(logits.data_ptr(), T, E, top_k, int(bool(renorm)), ids.data_ptr(), w.data_ptr(),
                         offsets.data_ptr(), perm.data_ptr(), _stream(stream)), "vq_route")
    return ids, w, offsets, perm


def fit(w, d: int, K: int, sample, init, iters: int, workspace=None, stream=None):
    """Data-free VQ fit of one bf16 tensor w [rows, cols] (16-bit bit patterns on the device):
    (scales fp16 bits [rows, cols/64], codebook fp16 bits [K, d], codes uint16 [rows, cols/d] as
    int16 tensors) from `iters` Lloyd steps over the subvectors `sample` starting at the
    subvectors `init` (int32 device tensors) (vq_fit)."""
    torch = _torch()
    rows, cols = w.shape
    dev = w.device
    scales = torch.empty((rows, cols // 64), dtype=torch.int16, device=dev)
    codebook = torch.empty((K, d), dtype=torch.int16, device=dev)
    codes = torch.empty((rows, cols // d), dtype=torch.int16, device=dev)
    n = int(_L().vq_fit_workspace_size(K, d))
    if n == 0:
        raise VQError(1, "vq_fit_workspace_size")
    ws = workspace if workspace is not None else torch.empty(n + 256, dtype=torch.uint8, device=dev)
    base = ws.data_ptr()
    aligned = (base + 255) // 256 * 256
    _check(_L().vq_fit(w.data_ptr(), rows, cols, d, K, sample.data_ptr(), sample.numel(), init.data_ptr(), iters,
                       scales.data_ptr(), codebook.data_ptr(), codes.data_ptr(), aligned, ws.numel() - (aligned - base),
                       _stream(stream)), "vq_fit")
    return scales, codebook, codes, ws


def fit_check(workspace, stream=None) -> int:
    """Status of the error word of a vq_fit workspace returned by fit() (vq_moe_check)."""
    base = (workspace.data_ptr() + 255) // 256 * 256
    return int(_L().vq_moe_check(base, _stream(stream)))


def set_trace_events(events) -> None:
    """Record the given torch.cuda.Event objects at the stage boundaries of the
    next MoE calls on this thread (vq_set_trace_events); None switches it off."""
    global _trace_keep
    if events is None:
        _trace_keep = None
        _check(_L().vq_set_trace_events(None, 0), "vq_set_trace_events")
        return
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _trace_keep = arr
    _check(_L().vq_set_trace_events(arr, len(events)), "vq_set_trace_events")


_trace_keep = None


def set_wait_limit(polls: Optional[int]) -> None:
    """Bound the barrier waits of the kernels this thread launches (vq_set_wait_limit);
    None restores the default."""
    _check(_L().vq_set_wait_limit(-1 if polls is None else int(polls)), "vq_set_wait_limit")


class MoELayer:
    """A SwiGLU MoE layer of three VQ modules (vq_moe_layer)."""

    def __init__(self, gate: Module, up: Module, down: Module):
        self.gate, self.up, self.down = gate, up, down
        self.hidden, self.inter, self.E = gate.cols, gate.rows, gate.E
        self._s = vq_moe_layer(gate.struct(), up.struct(), down.struct())
        self._ws = {}

    def workspace_size(self, T: int, top_k: int, mode: int) -> int:
        return int(_L().vq_moe_workspace_size(ctypes.byref(self._s), T, top_k, mode))

    def workspace(self, T: int, top_k: int, mode: int, device=None):
        """A cached device workspace large enough for (T, top_k, mode)."""
        torch = _torch()
        n = self.workspace_size(T, top_k, mode)
        if n == 0:
            raise VQError(1, "vq_moe_workspace_size")
        cur = self._ws.get(mode)
        if cur is None or cur.numel() < n:
            cur = torch.empty(n + 256, dtype=torch.uint8, device=device or self.gate.codes.device)
            self._ws[mode] = cur
        return cur

    def _run(self, fn, name, mode, x, logits, top_k, renorm, out, out_dtype, workspace, stream):
        torch = _torch()
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.hidden), dtype=out_dtype or torch.float32, device=x.device)
        ws = workspace if workspace is not None else self.workspace(T, top_k, mode, x.device)
        base = ws.data_ptr()
        aligned = (base + 255) // 256 * 256
        nbytes = ws.numel() - (aligned - base)
        _check(fn(ctypes.byref(self._s), x.data_ptr(), T, logits.data_ptr(), top_k, int(bool(renorm)),
                  out.data_ptr(), _dt(out.dtype), aligned, nbytes, _stream(stream)), name)
        return out

    def check(self, mode: int, stream=None) -> int:
        """Status of the device error word of the cached workspace for `mode` (vq_moe_check)."""
        ws = self._ws.get(mode)
        if ws is None:
            return VQ_OK
        base = (ws.data_ptr() + 255) // 256 * 256
        return int(_L().vq_moe_check(base, _stream(stream)))

    def decode(self, x, logits, top_k: int, renorm: bool = True, out=None, out_dtype=None, workspace=None,
               stream=None):
        """y [T, hidden] for decode-sized batches (vq_moe_decode)."""
        return self._run(_L().vq_moe_decode, "vq_moe_decode", VQ_MODE_DECODE, x, logits, top_k, renorm, out,
                         out_dtype, workspace, stream)

    def prefill(self, x, logits, top_k: int, renorm: bool = True, out=None, out_dtype=None, workspace=None,
                stream=None):
        """y [T, hidden] for prefill-sized batches (vq_moe_prefill, tcgen05 grouped GEMM)."""
        return self._run(_L().vq_moe_prefill, "vq_moe_prefill", VQ_MODE_PREFILL, x, logits, top_k, renorm, out,
                         out_dtype, workspace, stream)

    def prefill_chunked(self, x, logits, top_k: int, chunk: int = 2048, renorm: bool = True, out=None,
                        out_dtype=None, workspace=None, stream=None):
        """y [T, hidden] for a long prompt, `chunk` tokens at a time through one chunk-sized
        workspace (vq_moe_prefill_chunked)."""
        torch = _torch()
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.hidden), dtype=out_dtype or torch.float32, device=x.device)
        ws = workspace if workspace is not None else self.workspace(max(1, min(T, chunk)), top_k, VQ_MODE_PREFILL,
                                                                     x.device)
        base = ws.data_ptr()
        aligned = (base + 255) // 256 * 256
        nbytes = ws.numel() - (aligned - base)
        _check(_L().vq_moe_prefill_chunked(ctypes.byref(self._s), x.data_ptr(), T, logits.data_ptr(), top_k,
                                            int(bool(renorm)), int(chunk), out.data_ptr(), _dt(out.dtype), aligned,
                                            nbytes, _stream(stream)), "vq_moe_prefill_chunked")
        return out
