"""GPU-vs-oracle comparison helpers shared by the GPU tests.

Tolerances (derived in the design notes):
* lattice points, core indices, escape/overflow records: bit-exact on every
  group whose oracle margin (nearest vs second-nearest squared distance)
  exceeds 1e-4; near-tie groups are counted and must hold a valid E8 point
  no further from x than the oracle's point plus the margin bound;
* scales: relative 1e-5 (fp32 transform and sum against fp64);
* rotated-domain dequant: bit-exact given the GPU's indices, records, scale;
* original-basis dequant: <= 1 bf16 ulp of the fp64 value, plus 2^-20 s_r;
* GEMV: ||y - y_ref|| / ||y_ref|| <= 1e-2, and each output within its bf16
  rounding (2^-8 |y_ref|) plus 1e-3 rms(y_ref) of its batch row.
"""
import os

import numpy as np

import oracle
from bit_e8_lattice_b200 import synth

MARGIN = 1e-4


def gpu_points(idx, esc_rec, ovf_rec, n_groups, group_base=0):
    """Lattice points the GPU encoded (oracle's exact inverse of the encoding)."""
    # records come in group order (checked by check_encode): the matrix's slice by binary search
    eg, og = esc_rec["group"], ovf_rec["group"]
    lo, hi = np.uint32(group_base), np.uint32(min(group_base + n_groups, 2 ** 32 - 1))
    e = esc_rec[np.searchsorted(eg, lo):np.searchsorted(eg, hi)]
    o = ovf_rec[np.searchsorted(og, lo):np.searchsorted(og, hi)]
    P = oracle.assemble_points(idx.astype(np.int64) & 0xFFFF, e["group"].astype(np.int64), e["root"].astype(np.int64),
                               o["group"].astype(np.int64), o["coord2"].astype(np.int32), n_groups, group_base)
    kind = np.zeros(n_groups, np.int32)
    kind[e["group"].astype(np.int64) - group_base] = 1
    kind[o["group"].astype(np.int64) - group_base] = 2
    root = np.full(n_groups, -1, np.int32)
    root[e["group"].astype(np.int64) - group_base] = e["root"]
    return P, kind, root, e, o


def check_encode(out, idx_gpu, scale_gpu, esc_rec, ovf_rec, group_base=0, rows_sel=None, gpr=None, label=""):
    """Compare one matrix's GPU encoding with the oracle result ``out``
    (computed on the same rows).  ``rows_sel``: the rows ``out`` covers
    (None = all).  Returns a dict of statistics."""
    idx_gpu = np.asarray(idx_gpu).astype(np.int64) & 0xFFFF
    R = out["scale"].shape[0]
    gpr = gpr if gpr is not None else out["P"].shape[0] // R
    if rows_sel is None:
        rows_sel = np.arange(R)
    rows_sel = np.asarray(rows_sel)
    n_all = idx_gpu.size
    P_all, kind_all, root_all, e, o = gpu_points(idx_gpu.reshape(-1), esc_rec, ovf_rec, n_all, group_base)
    gsel = (rows_sel[:, None] * gpr + np.arange(gpr)[None, :]).reshape(-1)
    P, kind, root = P_all[gsel], kind_all[gsel], root_all[gsel]
    idx = idx_gpu.reshape(-1)[gsel]
    np.testing.assert_allclose(np.asarray(scale_gpu)[rows_sel], out["scale"], rtol=1e-5, atol=0,
                               err_msg=f"{label}: scale")
    m = out["margin"]
    near = m <= MARGIN
    far = ~near
    bad = far & (P != out["P"]).any(1)
    assert not bad.any(), f"{label}: {bad.sum()} lattice points differ above the margin, e.g. group {np.nonzero(bad)[0][:5]}"
    assert (idx[far] == out["idx"][far]).all(), f"{label}: core index differs above the margin"
    assert (kind[far] == out["kind"][far]).all(), f"{label}: record kind differs above the margin"
    esc_far = far & (out["kind"] == 1)
    assert (root[esc_far] == out["root"][esc_far]).all(), f"{label}: escape root differs"
    # record fields agree with the index array
    if len(e):
        assert (e["core"].astype(np.int64) == idx_gpu.reshape(-1)[e["group"].astype(np.int64) - group_base]).all()
        assert (np.diff(e["group"].astype(np.int64)) > 0).all(), f"{label}: escape records not in group order"
    if len(o):
        assert (np.diff(o["group"].astype(np.int64)) > 0).all(), f"{label}: overflow records not in group order"
        assert (idx_gpu.reshape(-1)[o["group"].astype(np.int64) - group_base] == 0).all()
    # near ties: a valid lattice point as close as the oracle's, within the bound
    if near.any():
        x = out["x"].reshape(-1, 8)[near]
        Pn = P[near]
        par = Pn[:, :1] & 1
        assert ((Pn & 1) == par).all() and (Pn.sum(1) % 4 == 0).all(), f"{label}: near-tie output not in E8"
        dg = ((x - Pn / 2.0) ** 2).sum(1)
        do = ((x - out["P"][near] / 2.0) ** 2).sum(1)
        assert (dg <= do + MARGIN + 1e-6).all(), f"{label}: near-tie output too far"
    return dict(groups=int(len(m)), near_ties=int(near.sum()), rho=float((kind > 0).mean()),
                overflow=float((kind == 2).mean()), points=P, kind=kind)


def check_rotated_dequant(bits_gpu, P_gpu, scale_gpu, signs, block, label=""):
    ref, _ = oracle.dequant(P_gpu, np.asarray(scale_gpu, np.float64), signs, block, "rotated")
    got = np.asarray(bits_gpu).view(np.uint16).reshape(ref.shape)
    diff = got != ref
    assert not diff.any(), f"{label}: {diff.sum()} rotated dequant values differ"


def check_original_dequant(bits_gpu, P_gpu, scale_gpu, signs, block, label=""):
    s = np.asarray(scale_gpu, np.float64)
    _, f64 = oracle.dequant(P_gpu, s, signs, block, "original")
    got = synth.bf16_bits_to_f64(np.asarray(bits_gpu).view(np.uint16)).reshape(f64.shape)
    # one bf16 ulp of the exact value (8 significant bits), plus an absolute floor
    ulp = np.where(f64 != 0, 2.0 ** (np.floor(np.log2(np.abs(f64) + 1e-300)) - 7), 0.0)
    tol = ulp + 2.0 ** -20 * s[:, None]
    err = np.abs(got - f64)
    bad = err > tol
    assert not bad.any(), f"{label}: {bad.sum()} original-basis values off by more than 1 ulp (max {err.max()})"


def check_gemv(y_gpu, y_ref, label=""):
    """Normwise relative error <= 1e-2 (the stated GEMV bound), and every
    element within its bf16 output rounding (2^-8 relative) plus 1e-3 of
    the row's rms for the fp32 accumulation."""
    y = synth.bf16_bits_to_f64(np.asarray(y_gpu).view(np.uint16)).reshape(y_ref.shape)
    for b in range(y_ref.shape[0]):
        rms = np.sqrt((y_ref[b] ** 2).mean())
        excess = np.abs(y[b] - y_ref[b]) - (2.0 ** -8 * np.abs(y_ref[b]) + 1e-3 * rms)
        assert excess.max() <= 0, f"{label}: batch row {b}: {int((excess > 0).sum())} outputs beyond bf16 rounding"
    rel = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert rel <= 1e-2, f"{label}: relative error {rel:.3g}"
    return rel


def _oracle_rows(args):
    """Worker: the oracle on a block of rows (bf16 bits), for a process pool."""
    bits, signs, block, want_x = args
    out = oracle.project_encode(synth.bf16_bits_to_f64(bits), signs, block, 1.0, want_x=want_x)
    return {k: out[k] for k in ("scale", "x", "P", "margin", "idx", "kind", "root")}


def oracle_rows_parallel(jobs, procs=None):
    """The oracle over many (bits, signs, block, want_x) jobs in spawned
    processes (one pool; spawn, so that no CUDA state is forked)."""
    return list(oracle_rows_stream(jobs, procs))


def oracle_rows_stream(jobs, procs=None):
    """As oracle_rows_parallel, yielding the results in job order as they
    complete (bounded memory for many jobs)."""
    import multiprocessing as mp
    procs = procs or max(1, min(32, os.cpu_count() or 1))
    with mp.get_context("spawn").Pool(procs) as pool:
        yield from pool.imap(_oracle_rows, jobs, chunksize=1)


def merge_rows(outs):
    m = {}
    for k in ("scale", "P", "margin", "idx", "kind", "root"):
        m[k] = np.concatenate([o[k] for o in outs])
    m["x"] = np.concatenate([o["x"] for o in outs]) if outs[0]["x"] is not None else None
    return m


def check_encode_far(out, idx_gpu, scale_gpu, esc_rec, ovf_rec, group_base, label=""):
    """check_encode without the oracle's x: every group clear of a tie must
    agree in point, index, record kind and root; returns the near-tie count."""
    idx_gpu = np.asarray(idx_gpu).astype(np.int64).reshape(-1) & 0xFFFF
    P, kind, root, e, o = gpu_points(idx_gpu, esc_rec, ovf_rec, idx_gpu.size, group_base)
    np.testing.assert_allclose(np.asarray(scale_gpu), out["scale"], rtol=1e-5, atol=0, err_msg=f"{label}: scale")
    far = out["margin"] > MARGIN
    assert not (far & (P != out["P"]).any(1)).any(), f"{label}: lattice points differ above the margin"
    assert (idx_gpu[far] == out["idx"][far]).all(), f"{label}: core index differs above the margin"
    assert (kind[far] == out["kind"][far]).all(), f"{label}: record kind differs above the margin"
    ef = far & (out["kind"] == 1)
    assert (root[ef] == out["root"][ef]).all(), f"{label}: escape root differs"
    return int((~far).sum())
