"""Plain fp64 CPU oracle for the E8 quantize path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA library and never imports it.

The heavy primitives live in ``e8_oracle.c`` (plain C, fp64, single thread);
this module is argument marshalling plus the few steps that are clearer in
numpy.  Each function names the passage it follows:

* "E8-QAT: Efficient 2-Bit Quantization-Aware Training with Implicit Lattice
  Codebooks" -- abstract (implicit E8 codebook, arithmetic projection, 2-bit
  core encoding + sparse extension that keeps lattice points exactly);
  Figure 2 caption (fixed core, identity STE, escape records, Hadamard
  transforms and reconstruction scales); appendix Table 3 (65,536 core
  codewords, single-root residuals); Table 9 (escape fraction rho);
  Table 10 (payload b = 2 + 20 rho with 20-byte records).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, brute force, library routines or values printed on the pages.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "e8_oracle.c")
_SO = os.path.join(_HERE, "libe8oracle.so")

CORE_SIZE = 65536
N_ROOTS = 240

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no vectorisation flags)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        i64, i32, f64, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p
        L.eo_init.restype = ctypes.c_int
        L.eo_num_points.restype = i64
        L.eo_points.argtypes = [vp, vp]
        L.eo_roots.argtypes = [vp]
        L.eo_rank.argtypes = [vp]
        L.eo_rank.restype = i64
        L.eo_nearest.argtypes = [vp, vp]
        L.eo_margin.argtypes = [vp, vp]
        L.eo_margin.restype = f64
        L.eo_encode_point.argtypes = [vp, vp, vp]
        L.eo_encode_point.restype = ctypes.c_int
        L.eo_core_point.argtypes = [i32, vp]
        L.eo_hadamard_dense.argtypes = [vp, i64, vp]
        L.eo_fwht.argtypes = [vp, i64]
        L.eo_bf16_bits.argtypes = [f64]
        L.eo_bf16_bits.restype = ctypes.c_uint16
        L.eo_project_encode_rows.argtypes = [vp, i64, i64, vp, i64, f64, vp, vp, vp, vp, vp, vp, vp]
        L.eo_project_encode_rows.restype = i64
        L.eo_project_encode_vectors.argtypes = [vp, i64, vp, vp, vp, vp, vp]
        L.eo_nearest_core.argtypes = [vp, vp]
        L.eo_nearest_core.restype = i32
        L.eo_project_core_rows.argtypes = [vp, i64, i64, vp, i64, f64, vp, vp, vp, vp]
        L.eo_project_core_rows.restype = i64
        L.eo_dequant_rows.argtypes = [vp, vp, i64, i64, vp, i64, ctypes.c_int, vp, vp]
        L.eo_rht_vectors.argtypes = [vp, i64, i64, vp, i64, vp]
        rc = L.eo_init()
        if rc != 0:
            raise RuntimeError(f"oracle enumeration failed ({rc})")
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# Lattice tables (Table 3: 65,536 core codewords; 240-element root set R)
# --------------------------------------------------------------------------
def all_points():
    """Every E8 point with |p|^2 <= 12, doubled, in (|p|^2, lex) order."""
    L = lib()
    n = L.eo_num_points()
    c = np.zeros((n, 8), np.int8)
    n2 = np.zeros(n, np.int32)
    L.eo_points(_p(c), _p(n2))
    return c, n2


def core_points() -> np.ndarray:
    """The 65,536 core codewords (doubled coordinates); row k is index k."""
    return all_points()[0][:CORE_SIZE].copy()


def roots() -> np.ndarray:
    """The 240 roots of E8 (doubled), numbered in lexicographic order."""
    r = np.zeros((N_ROOTS, 8), np.int8)
    lib().eo_roots(_p(r))
    return r


def rank(P) -> int:
    """Rank of a doubled point in the (norm, lex) order; -1 if outside."""
    a = np.ascontiguousarray(np.asarray(P, np.int32).reshape(8))
    return int(lib().eo_rank(_p(a)))


# --------------------------------------------------------------------------
# Projection and encoding (abstract; Figure 2 (b), (c))
# --------------------------------------------------------------------------
def project_encode_vectors(x: np.ndarray):
    """Nearest E8 point of each 8-vector (no transform, no scale)."""
    x = np.ascontiguousarray(np.asarray(x, np.float64).reshape(-1, 8))
    n = x.shape[0]
    P = np.zeros((n, 8), np.int32)
    m = np.zeros(n, np.float64)
    idx = np.zeros(n, np.int32)
    kind = np.zeros(n, np.int32)
    root = np.zeros(n, np.int32)
    lib().eo_project_encode_vectors(_p(x), n, _p(P), _p(m), _p(idx), _p(kind), _p(root))
    return dict(P=P, margin=m, idx=idx, kind=kind, root=root)


def nearest_core_vectors(x: np.ndarray):
    """Core-clipped projection (Figure 2 (a): PTQ from the fixed core): the
    nearest of the 65,536 core codewords to each 8-vector, searched
    exhaustively; ties to the smaller index.  Returns idx, P, margin."""
    x = np.ascontiguousarray(np.asarray(x, np.float64).reshape(-1, 8))
    n = x.shape[0]
    idx = np.zeros(n, np.int32)
    m = np.zeros(n, np.float64)
    L = lib()
    for k in range(n):
        mk = ctypes.c_double()
        idx[k] = L.eo_nearest_core(_p(x[k]), ctypes.byref(mk))
        m[k] = mk.value
    return dict(idx=idx, P=core_points()[idx].astype(np.int32), margin=m)


def project_core(w: np.ndarray, signs: np.ndarray, block: int, kappa: float = 1.0, want_margin: bool = True):
    """The row pipeline of project_encode with the core-clipped projection:
    every group's nearest core point (no escape or overflow records)."""
    w = np.ascontiguousarray(np.asarray(w, np.float64))
    R, C = w.shape
    d = np.ascontiguousarray(np.asarray(signs, np.int8).reshape(C))
    G = R * (C // 8)
    scale = np.zeros(R, np.float64)
    P = np.zeros((G, 8), np.int32)
    m = np.zeros(G, np.float64) if want_margin else None
    idx = np.zeros(G, np.int32)
    nf = lib().eo_project_core_rows(_p(w), R, C, _p(d), int(block), float(kappa), _p(scale), _p(P),
                                    _p(m) if m is not None else None, _p(idx))
    return dict(scale=scale, P=P, margin=m, idx=idx, nonfinite=int(nf))


def encode_points(P: np.ndarray):
    """Core index / escape / overflow decision for given doubled points."""
    P = np.ascontiguousarray(np.asarray(P, np.int32).reshape(-1, 8))
    n = P.shape[0]
    idx = np.zeros(n, np.int32)
    kind = np.zeros(n, np.int32)
    root = np.zeros(n, np.int32)
    L = lib()
    for k in range(n):
        i = ctypes.c_int32()
        r = ctypes.c_int32()
        kind[k] = L.eo_encode_point(_p(P[k]), ctypes.byref(i), ctypes.byref(r))
        idx[k] = i.value
        root[k] = r.value
    return idx, kind, root


def default_block(cols: int) -> int:
    """RHT block: the largest power of two dividing cols, capped at 2048."""
    if cols <= 0:
        return 1
    return min(2048, cols & -cols)


def project_encode(w: np.ndarray, signs: np.ndarray, block: int, kappa: float = 1.0, want_x: bool = True,
                   want_margin: bool = True):
    """Figure 2 pipeline on one matrix: sign flip, blockwise RHT, row scale,
    projection of every 8-group, encoding.  ``w`` holds the stored input
    values (f32 or bf16 widened exactly)."""
    w = np.ascontiguousarray(np.asarray(w, np.float64))
    R, C = w.shape
    d = np.ascontiguousarray(np.asarray(signs, np.int8).reshape(C))
    G = R * (C // 8)
    scale = np.zeros(R, np.float64)
    x = np.zeros((R, C), np.float64) if want_x else None
    P = np.zeros((G, 8), np.int32)
    m = np.zeros(G, np.float64) if want_margin else None
    idx = np.zeros(G, np.int32)
    kind = np.zeros(G, np.int32)
    root = np.zeros(G, np.int32)
    nf = lib().eo_project_encode_rows(_p(w), R, C, _p(d), int(block), float(kappa), _p(scale),
                                      _p(x) if x is not None else None, _p(P), _p(m) if m is not None else None,
                                      _p(idx), _p(kind), _p(root))
    return dict(scale=scale, x=x, P=P, margin=m, idx=idx, kind=kind, root=root, nonfinite=int(nf))


def records(out, group_base: int = 0):
    """Escape records (group, core, root) and overflow records (group, P),
    both in group order, from a ``project_encode`` result."""
    kind, idx, root, P = out["kind"], out["idx"], out["root"], out["P"]
    e = np.nonzero(kind == 1)[0]
    o = np.nonzero(kind == 2)[0]
    esc = np.stack([e + group_base, idx[e], root[e]], axis=1).astype(np.int64) if len(e) else np.zeros((0, 3), np.int64)
    ovf_g = (o + group_base).astype(np.int64)
    ovf_P = P[o].astype(np.int32)
    return esc, ovf_g, ovf_P


def assemble_points(idx, esc_g, esc_root, ovf_g, ovf_P, n_groups: int, group_base: int = 0) -> np.ndarray:
    """p = core[idx] (+ root for an escape; the record's coordinates for an
    overflow): the exact inverse of the encoding."""
    core = core_points().astype(np.int32)
    rt = roots().astype(np.int32)
    P = core[np.asarray(idx, np.int64).reshape(n_groups)]
    if len(esc_g):
        g = np.asarray(esc_g, np.int64) - group_base
        P[g] += rt[np.asarray(esc_root, np.int64)]
    if len(ovf_g):
        g = np.asarray(ovf_g, np.int64) - group_base
        P[g] = np.asarray(ovf_P, np.int32)
    return P


def dequant(P: np.ndarray, scale: np.ndarray, signs: np.ndarray, block: int, basis: str):
    """bf16 bits of the dequantised weights.  ``scale`` is the stored fp32
    scale.  basis 'rotated': bf16(s*p); 'original': bf16(d * H(s*p)/sqrt(B)).
    Returns (bits uint16 [R][C], unrounded float64 [R][C] or None)."""
    scale = np.ascontiguousarray(np.asarray(scale, np.float64))
    R = scale.shape[0]
    Pf = np.ascontiguousarray(np.asarray(P, np.int32).reshape(R, -1))
    C = Pf.shape[1]
    d = np.ascontiguousarray(np.asarray(signs, np.int8).reshape(C))
    bits = np.zeros((R, C), np.uint16)
    b = 1 if basis == "original" else 0
    f64 = np.zeros((R, C), np.float64) if b else None
    lib().eo_dequant_rows(_p(Pf), _p(scale), R, C, _p(d), int(block), b, _p(bits), _p(f64) if f64 is not None else None)
    return bits, f64


def rht_vectors(x: np.ndarray, signs: np.ndarray, block: int) -> np.ndarray:
    """x_rot = H_B (d * x) / sqrt(B) per row of x."""
    x = np.ascontiguousarray(np.asarray(x, np.float64))
    nb, C = x.shape
    d = np.ascontiguousarray(np.asarray(signs, np.int8).reshape(C))
    out = np.zeros_like(x)
    lib().eo_rht_vectors(_p(x), nb, C, _p(d), int(block), _p(out))
    return out


def gemv(P: np.ndarray, scale: np.ndarray, signs: np.ndarray, block: int, x: np.ndarray) -> np.ndarray:
    """y[b][r] = sum_c w~[r][c] x[b][c] with the unrounded fp64 dequantised
    weights in the original basis (the decode throughput path of the
    abstract).  A dense matmul is the library step."""
    _, w = dequant(P, scale, signs, block, "original")
    return np.asarray(x, np.float64) @ w.T


def bf16_bits(v: float) -> int:
    return int(lib().eo_bf16_bits(float(v)))


def hadamard_dense(u: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(np.asarray(u, np.float64))
    v = np.zeros_like(u)
    lib().eo_hadamard_dense(_p(u), u.shape[0], _p(v))
    return v


def fwht(u: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(np.array(u, np.float64))
    lib().eo_fwht(_p(v), v.shape[0])
    return v


# --------------------------------------------------------------------------
# Shape-gain variant (SQuAT page, "shape and scale split" section): every
# weight vector splits into a unit direction, quantised against a spherical
# E8 codebook, and a scalar gain through a low-bit scalar quantiser.  The
# page fixes neither the codebook shell nor the gain grid; the readings
# taken here: the direction codebook is the 2160-point shell |p|^2 = 4
# (the core's indices 241 .. 2400, direction index = core index - 241,
# 12 bits); the gain g = |x| of the row-normalised group goes through a
# 16-level uniform quantiser on [0, 6): level k = min(15, floor(g / D)),
# D = 6 / 16, value (k + 1/2) D; code = k << 12 | direction (16 bits a
# group, 2 bits a weight).  The reconstruction is (k + 1/2) D * c / |c|.
# --------------------------------------------------------------------------
SG_SHELL_FIRST = 241      # core index of the first |p|^2 = 4 point
SG_SHELL_SIZE = 2160
SG_LEVELS = 16
SG_GAIN_MAX = 6.0
SG_STEP = SG_GAIN_MAX / SG_LEVELS


def sg_shell() -> np.ndarray:
    """The 2160 directions: doubled points of the |p|^2 = 4 shell in core
    (lex) order."""
    return core_points()[SG_SHELL_FIRST:SG_SHELL_FIRST + SG_SHELL_SIZE].astype(np.int64)


def sg_encode_vectors(x: np.ndarray):
    """Direction = the shell point of largest inner product with x (all
    shell points have one norm, so this is the nearest direction; equal
    products go to the smaller index), found by scoring all 2160; gain
    level from |x|.  Returns code, direction, level, margin (the gap between
    the best and second-best cosine)."""
    x = np.asarray(x, np.float64).reshape(-1, 8)
    S = sg_shell().astype(np.float64)
    score = x @ S.T                              # <x, P>, |P| = 4
    d = np.argmax(score, axis=1)
    top = np.take_along_axis(score, d[:, None], 1)[:, 0]
    score[np.arange(len(d)), d] = -np.inf
    second = score.max(axis=1)
    n = np.sqrt((x * x).sum(axis=1))
    margin = np.where(n > 0, (top - second) / (4.0 * np.where(n > 0, n, 1.0)), 0.0)
    k = np.minimum(SG_LEVELS - 1, np.floor(n / SG_STEP)).astype(np.int64)
    return (k << 12) | d, d, k, margin


def sg_points(code: np.ndarray) -> np.ndarray:
    """x-hat of each code: (k + 1/2) D * P / 4 (float64 [G][8])."""
    code = np.asarray(code, np.int64).reshape(-1)
    S = sg_shell().astype(np.float64)
    k = code >> 12
    return ((k + 0.5) * SG_STEP)[:, None] * S[code & 0xFFF] / 4.0


def _bf16_rne(v: np.ndarray) -> np.ndarray:
    """Round float64 to bf16 bits once, half to even (finite values)."""
    f = np.asarray(v, np.float64)
    m, e = np.frexp(f)                       # f = m 2^e, |m| in [0.5, 1)
    q = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # 8 significant bits, ties to even
    u = q.astype(np.float32).view(np.uint32)     # exact: q has 8 bits
    return (u >> np.uint32(16)).astype(np.uint16)


def sg_dequant(xhat: np.ndarray, scale: np.ndarray, signs: np.ndarray, block: int, basis: str):
    """bf16 bits of s * x-hat (basis 'rotated') or of d * H_B(s * x-hat) / sqrt(B)
    (basis 'original', the STE forward in the weights' own basis)."""
    scale = np.asarray(scale, np.float64)
    R = scale.shape[0]
    xh = np.asarray(xhat, np.float64).reshape(R, -1)
    v = scale[:, None] * xh
    if basis == "original":
        C = xh.shape[1]
        v = rht_vectors(v, np.ones(C, np.int8), block) * np.asarray(signs, np.float64).reshape(1, C)
    return _bf16_rne(v), v


def sg_project_encode(w: np.ndarray, signs: np.ndarray, block: int, kappa: float = 1.0):
    """The shape-gain pipeline on one matrix: sign flip, blockwise RHT, row
    scale (as for the lattice projection), then the shape-gain code of every
    8-group."""
    out = project_encode(w, signs, block, kappa, want_x=True, want_margin=False)
    code, d, k, margin = sg_encode_vectors(out["x"])
    return dict(scale=out["scale"], x=out["x"], code=code, dir=d, level=k, margin=margin,
                xhat=sg_points(code))


# --------------------------------------------------------------------------
# Payload accounting (Table 10; Figure 6 (c))
# --------------------------------------------------------------------------
def payload_bits_pages(rho: float) -> float:
    """Bits per weight with 20-byte coordinate records: b = 2 + 20 rho,
    rho = escaped groups / all groups (8 weights per group)."""
    return 2.0 + 20.0 * rho


def payload_bits_actual(n_groups: int, n_escape: int, n_overflow: int, esc_bytes: int = 8, ovf_bytes: int = 20) -> float:
    """Bits per weight of this library's layout: 16-bit index per group plus
    8-byte root records and 20-byte coordinate records (scales excluded)."""
    if n_groups == 0:
        return 0.0
    return (16.0 * n_groups + 8.0 * (esc_bytes * n_escape + ovf_bytes * n_overflow)) / (8.0 * n_groups)
