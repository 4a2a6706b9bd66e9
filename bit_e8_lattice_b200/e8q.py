"""Thin ctypes binding of libe8q (include/e8q.h), same entry-point names.

Argument marshalling only: torch provides device memory and streams, every
step of the path runs in the library's CUDA kernels.  There is no CPU
fallback: if ``libe8q.so`` is missing or no CUDA device is present the calls
raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libe8q.so")

E8Q_OK = 0
E8Q_F32, E8Q_BF16 = 0, 1
DEQUANT = {"none": 0, "rotated": 1, "original": 2}

ESC_DTYPE = np.dtype([("group", "<u4"), ("core", "<u2"), ("root", "u1"), ("reserved", "u1")])
OVF_DTYPE = np.dtype([("group", "<u4"), ("coord2", "<i2", (8,))])


class E8qError(RuntimeError):
    pass


class Matrix(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("signs", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("scale", ctypes.c_void_p), ("dequant", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("rht_block", ctypes.c_int32), ("in_dtype", ctypes.c_int32)]


class EncodeArgs(ctypes.Structure):
    _fields_ = [("kappa", ctypes.c_float), ("dequant", ctypes.c_int32), ("scale_in", ctypes.c_int32),
                ("esc", ctypes.c_void_p), ("esc_cap", ctypes.c_int64), ("ovf", ctypes.c_void_p),
                ("ovf_cap", ctypes.c_int64), ("esc_row_ptr", ctypes.c_void_p), ("ovf_row_ptr", ctypes.c_void_p),
                ("counters", ctypes.c_void_p), ("flags", ctypes.c_int32), ("reserved", ctypes.c_int32)]


ENCODE_CORE_ONLY = 1
ENCODE_SHAPE_GAIN = 2


class EncodedC(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("signs", ctypes.c_void_p),
                ("esc", ctypes.c_void_p), ("esc_row_ptr", ctypes.c_void_p), ("ovf", ctypes.c_void_p),
                ("ovf_row_ptr", ctypes.c_void_p), ("esc_count", ctypes.c_int64), ("ovf_count", ctypes.c_int64),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("group_base", ctypes.c_int64),
                ("rht_block", ctypes.c_int32), ("reserved", ctypes.c_int32)]


COUNTER_FIELDS = ("n_escape", "n_overflow", "n_nonfinite", "n_dropped", "n_clamped", "err")

_lib = None


def lib():
    """Load libe8q.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise E8qError(f"{LIB_PATH} is missing; build it with `python -m bit_e8_lattice_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.e8q_status_string.argtypes = [ctypes.c_int]
        L.e8q_status_string.restype = ctypes.c_char_p
        L.e8q_init.restype = ctypes.c_int
        L.e8q_core_table.argtypes = [vp]
        L.e8q_core_table.restype = ctypes.c_int
        L.e8q_escape_lookup.argtypes = [vp, i64, vp]
        L.e8q_escape_lookup.restype = ctypes.c_int
        L.e8q_encode_workspace_bytes.argtypes = [ctypes.POINTER(Matrix), i32]
        L.e8q_encode_workspace_bytes.restype = sz
        L.e8q_project_encode.argtypes = [ctypes.POINTER(Matrix), i32, ctypes.POINTER(EncodeArgs), vp, sz, vp]
        L.e8q_project_encode.restype = ctypes.c_int
        L.e8q_project_encode_noalloc.argtypes = [ctypes.POINTER(Matrix), i32, ctypes.POINTER(EncodeArgs), vp]
        L.e8q_project_encode_noalloc.restype = ctypes.c_int
        L.e8q_decode.argtypes = [ctypes.POINTER(EncodedC), i32, vp, vp]
        L.e8q_decode.restype = ctypes.c_int
        L.e8q_gemv_workspace_bytes.argtypes = [ctypes.POINTER(EncodedC), i32]
        L.e8q_gemv_workspace_bytes.restype = sz
        L.e8q_dequant_gemv.argtypes = [ctypes.POINTER(EncodedC), vp, i32, vp, vp, sz, vp]
        L.e8q_dequant_gemv.restype = ctypes.c_int
        L.e8q_gemm_workspace_bytes.argtypes = [ctypes.POINTER(EncodedC), i32]
        L.e8q_gemm_workspace_bytes.restype = sz
        L.e8q_dequant_gemm.argtypes = [ctypes.POINTER(EncodedC), vp, i32, vp, vp, sz, vp]
        L.e8q_dequant_gemm.restype = ctypes.c_int
        L.e8q_ste_backward.argtypes = [vp, vp, i64, vp]
        L.e8q_ste_backward.restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != E8Q_OK:
        raise E8qError(f"{what}: {lib().e8q_status_string(rc).decode()} ({rc})")


def _stream_handle(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require_cuda(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise E8qError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise E8qError(f"{name} must be contiguous")


def core_table() -> np.ndarray:
    """The library's host-built core table (doubled coordinates), [65536][8]."""
    out = np.zeros((65536, 8), np.int8)
    _check(lib().e8q_core_table(out.ctypes.data_as(ctypes.c_void_p)), "e8q_core_table")
    return out


def escape_lookup(P: np.ndarray) -> np.ndarray:
    """The encode kernels' encoding word of given doubled E8 points [n][8]
    (host table; see e8q_escape_lookup in e8q.h)."""
    P = np.ascontiguousarray(np.asarray(P).reshape(-1, 8).astype(np.int8))
    out = np.zeros(P.shape[0], np.uint32)
    _check(lib().e8q_escape_lookup(P.ctypes.data_as(ctypes.c_void_p), P.shape[0], out.ctypes.data_as(ctypes.c_void_p)),
           "e8q_escape_lookup")
    return out


def init():
    _check(lib().e8q_init(), "e8q_init")


# --------------------------------------------------------------------------
# encoded matrices
# --------------------------------------------------------------------------
@dataclass
class Encoded:
    """One encoded matrix: views into the buffers of its encode call."""
    idx: torch.Tensor            # uint16 bits stored as int16 [rows][cols/8]
    scale: torch.Tensor          # float32 [rows]
    signs: torch.Tensor          # int8 [cols]
    esc: torch.Tensor            # uint8 [cap*8] (whole call)
    esc_row_ptr: torch.Tensor    # int64 [rows+1] (slice of the call's CSR)
    ovf: torch.Tensor            # uint8 [cap*20]
    ovf_row_ptr: torch.Tensor    # int64 [rows+1]
    rows: int
    cols: int
    group_base: int
    rht_block: int = 0
    esc_count: int = 0           # readable records (the encode call's capacity bound)
    ovf_count: int = 0

    def c(self) -> EncodedC:
        return EncodedC(_ptr(self.idx), _ptr(self.scale), _ptr(self.signs), _ptr(self.esc), _ptr(self.esc_row_ptr),
                        _ptr(self.ovf), _ptr(self.ovf_row_ptr), self.esc_count, self.ovf_count, self.rows, self.cols,
                        self.group_base, self.rht_block, 0)


@dataclass
class EncodeResult:
    idx: List[torch.Tensor]
    scale: List[torch.Tensor]
    dequant: List[Optional[torch.Tensor]]
    esc: torch.Tensor
    ovf: torch.Tensor
    esc_row_ptr: torch.Tensor
    ovf_row_ptr: torch.Tensor
    counters: torch.Tensor        # uint64 as int64 [6] on the device
    encoded: List[Encoded]
    group_base: List[int]
    row_base: List[int]
    esc_cap: int
    ovf_cap: int
    workspace: torch.Tensor = field(repr=False, default=None)

    def read_counters(self) -> dict:
        v = self.counters.cpu().numpy().view(np.uint64)
        return {k: int(x) for k, x in zip(COUNTER_FIELDS, v)}

    def escape_records(self) -> np.ndarray:
        n = min(self.read_counters()["n_escape"], self.esc_cap)
        return np.frombuffer(self.esc[: 8 * n].cpu().numpy().tobytes(), ESC_DTYPE)

    def overflow_records(self) -> np.ndarray:
        n = min(self.read_counters()["n_overflow"], self.ovf_cap)
        return np.frombuffer(self.ovf[: 20 * n].cpu().numpy().tobytes(), OVF_DTYPE)


class Encoder:
    """Pre-allocated outputs for repeated project+encode calls on matrices of
    fixed shapes (one launch per call)."""

    def __init__(self, shapes: Sequence[tuple], signs: Sequence[torch.Tensor], in_dtype=torch.bfloat16,
                 rht_block=0, kappa: float = 1.0, dequant: str = "none", scale_in: bool = False,
                 esc_cap: Optional[int] = None, ovf_cap: Optional[int] = None, device=None, core_only: bool = False,
                 shape_gain: bool = False):
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        blocks = rht_block if isinstance(rht_block, (list, tuple)) else [rht_block] * len(self.shapes)
        self.blocks = [int(b) for b in blocks]
        self.signs = list(signs)
        for s in self.signs:
            _require_cuda(s, "signs")
        self.in_dtype = in_dtype
        self.kappa = float(kappa)
        self.dq = DEQUANT[dequant]
        self.scale_in = bool(scale_in)
        groups = [r * (c // 8) for r, c in self.shapes]
        total_groups = sum(groups)
        self.total_rows = sum(r for r, _ in self.shapes)
        self.esc_cap = int(esc_cap) if esc_cap is not None else max(64, total_groups // 2)
        self.ovf_cap = int(ovf_cap) if ovf_cap is not None else max(64, total_groups // 8)
        dev = self.device
        self.idx = [torch.empty((r, c // 8), dtype=torch.int16, device=dev) for r, c in self.shapes]
        self.scale = [torch.zeros(r, dtype=torch.float32, device=dev) for r, _ in self.shapes]
        self.dequant = [torch.empty((r, c), dtype=torch.bfloat16, device=dev) if self.dq else None
                        for r, c in self.shapes]
        self.esc = torch.empty(8 * self.esc_cap, dtype=torch.uint8, device=dev)
        self.ovf = torch.empty(20 * self.ovf_cap, dtype=torch.uint8, device=dev)
        self.esc_row_ptr = torch.empty(self.total_rows + 1, dtype=torch.int64, device=dev)
        self.ovf_row_ptr = torch.empty(self.total_rows + 1, dtype=torch.int64, device=dev)
        self.counters = torch.zeros(6, dtype=torch.int64, device=dev)
        self.group_base, self.row_base = [], []
        gb = rb = 0
        for (r, c), g in zip(self.shapes, groups):
            self.group_base.append(gb)
            self.row_base.append(rb)
            gb += g
            rb += r
        self._mats = (Matrix * len(self.shapes))()
        for i, ((r, c), b) in enumerate(zip(self.shapes, self.blocks)):
            m = self._mats[i]
            m.rows, m.cols, m.rht_block = r, c, b
            m.in_dtype = E8Q_BF16 if in_dtype == torch.bfloat16 else E8Q_F32
            m.signs = self.signs[i].data_ptr()
            m.idx = self.idx[i].data_ptr()
            m.scale = self.scale[i].data_ptr()
            m.dequant = self.dequant[i].data_ptr() if self.dequant[i] is not None else None
        ws_bytes = lib().e8q_encode_workspace_bytes(self._mats, len(self.shapes))
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        self.core_only = bool(core_only)
        self.shape_gain = bool(shape_gain)
        self._args = EncodeArgs(self.kappa, self.dq, 1 if self.scale_in else 0, self.esc.data_ptr(), self.esc_cap,
                                self.ovf.data_ptr(), self.ovf_cap, self.esc_row_ptr.data_ptr(),
                                self.ovf_row_ptr.data_ptr(), self.counters.data_ptr(),
                                (ENCODE_CORE_ONLY if self.core_only else 0) | (ENCODE_SHAPE_GAIN if self.shape_gain else 0), 0)

    def __call__(self, weights: Sequence[torch.Tensor], scales: Optional[Sequence[torch.Tensor]] = None,
                 stream=None) -> EncodeResult:
        if len(weights) != len(self.shapes):
            raise E8qError("number of weights does not match the encoder")
        for i, w in enumerate(weights):
            _require_cuda(w, "weight")
            if tuple(w.shape) != self.shapes[i] or w.dtype != self.in_dtype:
                raise E8qError(f"weight {i}: expected {self.shapes[i]} {self.in_dtype}, got {tuple(w.shape)} {w.dtype}")
            self._mats[i].w = w.data_ptr()
        self._load_scales(scales)
        rc = lib().e8q_project_encode(self._mats, len(self.shapes), ctypes.byref(self._args),
                                      ctypes.c_void_p(self.workspace.data_ptr()), self.workspace.numel(),
                                      _stream_handle(stream))
        _check(rc, "e8q_project_encode")
        return self.result()

    def _load_scales(self, scales):
        """Given scales go to the scale buffers the kernels read; an encoder
        built with scale_in must be given them on every call."""
        if not self.scale_in:
            if scales is not None:
                raise E8qError("scales given to an encoder built without scale_in")
            return
        if scales is None:
            raise E8qError("scale_in encoder needs scales")
        if len(scales) != len(self.shapes):
            raise E8qError("number of scale vectors does not match the encoder")
        for i, s in enumerate(scales):
            if s.numel() != self.shapes[i][0]:
                raise E8qError(f"scales {i}: expected {self.shapes[i][0]} values, got {s.numel()}")
            self.scale[i].copy_(s.reshape(-1))

    def run_noalloc(self, weights: Sequence[torch.Tensor], scales: Optional[Sequence[torch.Tensor]] = None,
                    stream=None) -> EncodeResult:
        """Same encode through e8q_project_encode_noalloc: the library's
        built-in scratch instead of this encoder's workspace (for callers
        that cannot allocate; calls on one device must not overlap).  An
        encoder built with scale_in takes its scales here as in __call__."""
        if len(weights) != len(self.shapes):
            raise E8qError("number of weights does not match the encoder")
        for i, w in enumerate(weights):
            _require_cuda(w, "weight")
            if tuple(w.shape) != self.shapes[i] or w.dtype != self.in_dtype:
                raise E8qError(f"weight {i}: expected {self.shapes[i]} {self.in_dtype}, got {tuple(w.shape)} {w.dtype}")
            self._mats[i].w = w.data_ptr()
        self._load_scales(scales)
        rc = lib().e8q_project_encode_noalloc(self._mats, len(self.shapes), ctypes.byref(self._args),
                                              _stream_handle(stream))
        _check(rc, "e8q_project_encode_noalloc")
        return self.result()

    def result(self) -> EncodeResult:
        enc = []
        for i, (r, c) in enumerate(self.shapes):
            rb = self.row_base[i]
            enc.append(Encoded(self.idx[i], self.scale[i], self.signs[i], self.esc,
                               self.esc_row_ptr[rb: rb + r + 1], self.ovf, self.ovf_row_ptr[rb: rb + r + 1],
                               r, c, self.group_base[i], self.blocks[i], self.esc_cap, self.ovf_cap))
        return EncodeResult(self.idx, self.scale, self.dequant, self.esc, self.ovf, self.esc_row_ptr,
                            self.ovf_row_ptr, self.counters, enc, self.group_base, self.row_base, self.esc_cap,
                            self.ovf_cap, self.workspace)


def e8q_project_encode(weights: Sequence[torch.Tensor], signs: Sequence[torch.Tensor], rht_block=0,
                       kappa: float = 1.0, dequant: str = "none", scales=None, esc_cap=None, ovf_cap=None,
                       stream=None) -> EncodeResult:
    """One-shot project+encode of a batch of matrices (allocates outputs)."""
    if isinstance(weights, torch.Tensor):
        weights, signs = [weights], [signs]
    enc = Encoder([tuple(w.shape) for w in weights], signs, weights[0].dtype, rht_block, kappa, dequant,
                  scales is not None, esc_cap, ovf_cap, device=weights[0].device)
    return enc(weights, scales, stream)


def e8q_decode(m: Encoded, basis: str = "rotated", out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((m.rows, m.cols), dtype=torch.bfloat16, device=m.idx.device)
    _require_cuda(out, "out")
    mc = m.c()
    _check(lib().e8q_decode(ctypes.byref(mc), DEQUANT[basis], _ptr(out), _stream_handle(stream)), "e8q_decode")
    return out


def e8q_ste_backward(grad_dequant: torch.Tensor, grad_latent: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Identity-STE backward: the latents' gradient is the dequantised
    weights' gradient.  With grad_latent None (or the same tensor) the result
    is grad_dequant itself and nothing runs; otherwise the library copies it
    into grad_latent (bf16, same number of elements)."""
    _require_cuda(grad_dequant, "grad_dequant")
    if grad_dequant.dtype != torch.bfloat16:
        raise E8qError("grad_dequant must be bf16")
    out = grad_dequant if grad_latent is None else grad_latent
    _require_cuda(out, "grad_latent")
    if out.dtype != torch.bfloat16 or out.numel() != grad_dequant.numel():
        raise E8qError("grad_latent must be bf16 with as many elements as grad_dequant")
    _check(lib().e8q_ste_backward(_ptr(grad_dequant), _ptr(out), grad_dequant.numel(), _stream_handle(stream)),
           "e8q_ste_backward")
    return out


class Gemv:
    """Pre-allocated workspace and output for y = W~ x from the 2-bit form."""

    def __init__(self, m: Encoded, batch: int):
        self.m, self.batch = m, int(batch)
        self._mc = m.c()
        ws = lib().e8q_gemv_workspace_bytes(ctypes.byref(self._mc), self.batch)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=m.idx.device)
        self.y = torch.empty((self.batch, m.rows), dtype=torch.bfloat16, device=m.idx.device)

    def __call__(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        _require_cuda(x, "x")
        if x.dtype != torch.bfloat16 or tuple(x.shape) != (self.batch, self.m.cols):
            raise E8qError(f"x must be bf16 [{self.batch}][{self.m.cols}]")
        y = self.y if out is None else out
        rc = lib().e8q_dequant_gemv(ctypes.byref(self._mc), _ptr(x), self.batch, _ptr(y),
                                    ctypes.c_void_p(self.workspace.data_ptr()), self.workspace.numel(),
                                    _stream_handle(stream))
        _check(rc, "e8q_dequant_gemv")
        return y


def e8q_dequant_gemv(m: Encoded, x: torch.Tensor, stream=None) -> torch.Tensor:
    return Gemv(m, x.shape[0])(x, stream=stream).clone()


class Gemm:
    """Pre-allocated workspace and output for Y = X W~^T from the 2-bit form
    (many activation rows; the fused tensor-core dequant-GEMM)."""

    def __init__(self, m: Encoded, batch: int):
        self.m, self.batch = m, int(batch)
        self._mc = m.c()
        ws = lib().e8q_gemm_workspace_bytes(ctypes.byref(self._mc), self.batch)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=m.idx.device)
        self.y = torch.empty((self.batch, m.rows), dtype=torch.bfloat16, device=m.idx.device)

    def __call__(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        _require_cuda(x, "x")
        if x.dtype != torch.bfloat16 or tuple(x.shape) != (self.batch, self.m.cols):
            raise E8qError(f"x must be bf16 [{self.batch}][{self.m.cols}]")
        y = self.y if out is None else out
        rc = lib().e8q_dequant_gemm(ctypes.byref(self._mc), _ptr(x), self.batch, _ptr(y),
                                    ctypes.c_void_p(self.workspace.data_ptr()), self.workspace.numel(),
                                    _stream_handle(stream))
        _check(rc, "e8q_dequant_gemm")
        return y

    def error_word(self) -> int:
        """The last call's error word (0: every bounded wait completed)."""
        return int(self.workspace[:8].cpu().numpy().view(np.uint64)[0])


def e8q_dequant_gemm(m: Encoded, x: torch.Tensor, stream=None) -> torch.Tensor:
    return Gemm(m, x.shape[0])(x, stream=stream).clone()
