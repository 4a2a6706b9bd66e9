"""Seeded synthetic inputs for the E8 quantize path.

This module only draws random numbers and stores them in the input dtype;
it holds none of the method's arithmetic.  The CUDA library, the tests and
the CPU oracle all take their inputs from here.

Recipe: NumPy PCG64 ``default_rng(seed)``; values are drawn in float64 and
rounded once (round-half-even) to the stored dtype.  Sign vectors come from
``default_rng([seed, 1, matrix])`` as +-1 int8.  Shapes are rows x cols,
row-major.  Workloads (named by what they are):

* ``small_f32``      256x256 f32, N(0, 0.02^2), seed 0; plus 4,096 free
                     8-vectors 3*N(0, I) (seed [0, 2]) for brute-force checks.
* ``attn_2048``      2048x2048 bf16, Student-t(4) scaled to std 0.02, 20 rows
                     (1%) multiplied by 8, seed 2.
* ``moe_bank``       128 experts x (gate 2048x768, up 2048x768, down
                     768x2048) bf16, N(0, 0.02^2) times a per-expert factor
                     from U(0.5, 2), seed 3.
* ``mlp_14336``      up 4096x14336 and down 14336x4096 bf16, N(0, 0.015^2),
                     seed 4; upstream gradient N(0, 1e-3^2) bf16, seed 40.
* ``latent_drift``   float32 N(0, 1) [rows][cols], seed [41, matrix]: the
                     drift of latents initialised from the E8 core (the
                     caller scales it, e.g. by 0.15 x the weights' 0.015).
* ``gemv_x``         activations [batch][cols] bf16, N(0, 1), seed 5.
"""
from __future__ import annotations

import numpy as np


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float64 to bf16 once (half to even); returns uint16 bits.
    Finite inputs of normal bf16 magnitude only (what the recipes draw)."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    u = a.view(np.uint64)
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    u2 = (u + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f = u2.view(np.float64).astype(np.float32)  # exact: 8 significant bits left
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def signs(seed: int, cols: int, matrix: int = 0) -> np.ndarray:
    rng = np.random.default_rng([seed, 1, matrix])
    return rng.choice(np.array([-1, 1], np.int8), size=cols).astype(np.int8)


def small_f32(seed: int = 0, rows: int = 256, cols: int = 256):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    return w, signs(seed, cols)


def free_vectors(seed: int = 0, n: int = 4096, scale: float = 3.0) -> np.ndarray:
    rng = np.random.default_rng([seed, 2])
    return (rng.standard_normal((n, 8)) * scale).astype(np.float32)


def attn_2048(seed: int = 2, n: int = 2048, outlier_rows: int = 20, outlier_mult: float = 8.0):
    rng = np.random.default_rng(seed)
    w = rng.standard_t(4.0, size=(n, n)) * (0.02 / np.sqrt(2.0))
    rows = rng.choice(n, size=outlier_rows, replace=False)
    w[rows] *= outlier_mult
    return f64_to_bf16_bits(w), signs(seed, n)


def moe_shapes(experts: int = 128, d_model: int = 2048, d_ff: int = 768):
    """(name, rows, cols) for every matrix of the expert bank, expert-major."""
    out = []
    for e in range(experts):
        out += [(f"e{e}.gate", d_model, d_ff), (f"e{e}.up", d_model, d_ff), (f"e{e}.down", d_ff, d_model)]
    return out


def moe_bank(seed: int = 3, experts: int = 128, d_model: int = 2048, d_ff: int = 768, only=None):
    """List of (bf16 bits [rows][cols], signs) in ``moe_shapes`` order.
    ``only``: optional set of matrix indices to materialise (others None)."""
    rng = np.random.default_rng(seed)
    factors = rng.uniform(0.5, 2.0, size=experts)
    mats = []
    for m, (_, r, c) in enumerate(moe_shapes(experts, d_model, d_ff)):
        mrng = np.random.default_rng([seed, 0, m])
        if only is not None and m not in only:
            mats.append((None, signs(seed, c, m)))
            continue
        w = mrng.standard_normal((r, c)) * (0.02 * factors[m // 3])
        mats.append((f64_to_bf16_bits(w), signs(seed, c, m)))
    return mats


def mlp_14336(seed: int = 4, d_model: int = 4096, d_ff: int = 14336):
    """(up bits [d_model][d_ff], up signs), (down bits [d_ff][d_model], down signs)."""
    rng_u = np.random.default_rng([seed, 0, 0])
    rng_d = np.random.default_rng([seed, 0, 1])
    up = f64_to_bf16_bits(rng_u.standard_normal((d_model, d_ff)) * 0.015)
    down = f64_to_bf16_bits(rng_d.standard_normal((d_ff, d_model)) * 0.015)
    return (up, signs(seed, d_ff, 0)), (down, signs(seed, d_model, 1))


def mlp_grad(shape, seed: int = 40, matrix: int = 0) -> np.ndarray:
    rng = np.random.default_rng([seed, matrix])
    return f64_to_bf16_bits(rng.standard_normal(shape) * 1e-3)


def latent_drift(shape, seed: int = 41, matrix: int = 0) -> np.ndarray:
    """Unit-variance drift directions for the latents of a core-initialised
    model: float32 N(0, 1), scaled by the caller."""
    rng = np.random.default_rng([seed, matrix])
    return rng.standard_normal(shape, dtype=np.float32)


def gemv_x(batch: int, cols: int, seed: int = 5) -> np.ndarray:
    rng = np.random.default_rng([seed, batch])
    return f64_to_bf16_bits(rng.standard_normal((batch, cols)))
