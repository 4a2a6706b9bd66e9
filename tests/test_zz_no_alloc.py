"""The no-allocation encode entry point, e8q_project_encode_noalloc.

Some callers cannot allocate device memory at all (code that runs inside a
memory pool or a host framework that owns every allocation, or a path that
must never allocate).  For them the library offers an encode entry point
whose scratch is compiled into the library.  These tests call it through
the C ABI and check it against e8q_project_encode on two calls in a row.
This file is collected last on purpose: if it fails, a run that stops at
the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_e8_lattice_b200 import synth
from parity import MARGIN, check_original_dequant, gpu_points


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _snapshot(res):
    return dict(idx=[t.cpu().numpy().view(np.uint16).copy() for t in res.idx],
                scale=[t.cpu().numpy().copy() for t in res.scale],
                dq=[t.cpu().view(torch.int16).numpy().copy() for t in res.dequant if t is not None],
                esc=res.escape_records().copy(), ovf=res.overflow_records().copy(),
                erp=res.esc_row_ptr.cpu().numpy().copy(), orp=res.ovf_row_ptr.cpu().numpy().copy(),
                ctr=res.read_counters())


def _scrub(res):
    for t in res.idx:
        t.fill_(-1)
    for t in res.scale:
        t.fill_(float("nan"))
    for t in res.dequant:
        if t is not None:
            t.fill_(float("nan"))
    res.esc.fill_(0xFF)
    res.ovf.fill_(0xFF)
    res.esc_row_ptr.fill_(-1)
    res.ovf_row_ptr.fill_(-1)
    torch.cuda.synchronize()


@pytest.mark.gpu
def test_noalloc_equals_workspace_entry_point_f32_batch():
    """f32 matrices of two shapes in one call: both entry points run the same
    kernel, so every output must agree bit for bit, call after call."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_e8_lattice_b200 import e8q

    e8q.init()
    rng = np.random.default_rng(31)
    mats = [(rng.standard_normal((40, 256)) * 0.02).astype(np.float32),
            (rng.standard_normal((9, 2048)) * 0.02).astype(np.float32)]
    signs = [torch.from_numpy(synth.signs(31, m.shape[1], i)).cuda() for i, m in enumerate(mats)]
    W = [torch.from_numpy(m).cuda() for m in mats]
    enc = e8q.Encoder([m.shape for m in mats], signs, torch.float32, 0, 1.0, "original", esc_cap=20000,
                      ovf_cap=20000)
    ref = _snapshot(enc(W))
    assert ref["ctr"]["n_escape"] > 0
    for _ in range(2):
        _scrub(enc.result())
        got = _snapshot(enc.run_noalloc(W))
        for k in ("idx", "scale", "dq"):
            for a, b in zip(ref[k], got[k]):
                np.testing.assert_array_equal(a, b, err_msg=k)
        for k in ("esc", "ovf"):
            assert ref[k].tobytes() == got[k].tobytes(), k
        np.testing.assert_array_equal(ref["erp"], got["erp"])
        np.testing.assert_array_equal(ref["orp"], got["orp"])
        assert ref["ctr"] == got["ctr"]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_bf16():
    """bf16 2048x2048: the workspace entry point takes its fast kernel, the
    no-allocation one the general kernel; they agree exactly on every group
    clear of a near tie (oracle margin > 1e-4), on two calls in a row."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_e8_lattice_b200 import e8q

    e8q.init()
    w, d = synth.attn_2048()
    W = [_dev_bf16(w)]
    enc = e8q.Encoder([w.shape], [torch.from_numpy(d).cuda()], torch.bfloat16, 0, 1.0, "original",
                      esc_cap=w.size // 8, ovf_cap=w.size // 8)
    ref = _snapshot(enc(W))
    out = oracle.project_encode(synth.bf16_bits_to_f64(w), d, 2048, want_x=False)
    far = out["margin"] > MARGIN
    P_ref, k_ref, r_ref, _, _ = gpu_points(ref["idx"][0].reshape(-1), ref["esc"], ref["ovf"], far.size)
    for _ in range(2):
        _scrub(enc.result())
        got = _snapshot(enc.run_noalloc(W))
        assert got["ctr"]["err"] == 0 and got["ctr"]["n_dropped"] == 0
        np.testing.assert_allclose(got["scale"][0], ref["scale"][0], rtol=1e-5)
        P, k, r, _, _ = gpu_points(got["idx"][0].reshape(-1), got["esc"], got["ovf"], far.size)
        np.testing.assert_array_equal(got["idx"][0].reshape(-1)[far], ref["idx"][0].reshape(-1)[far])
        np.testing.assert_array_equal(P[far], P_ref[far])
        np.testing.assert_array_equal(k[far], k_ref[far])
        np.testing.assert_array_equal(r[far], r_ref[far])
        check_original_dequant(got["dq"][0], P, got["scale"][0], d, 2048, "noalloc original")


def _run_pair(e8q, shapes, mats, signs, dtype, dequant, scales=None, block=0):
    """The workspace entry point once, then the no-allocation one twice on
    scrubbed outputs; returns the three snapshots."""
    W = [torch.from_numpy(m).cuda() if dtype == torch.float32 else _dev_bf16(m) for m in mats]
    S = [torch.from_numpy(d).cuda() for d in signs]
    sc = None if scales is None else [torch.from_numpy(s).cuda() for s in scales]
    enc = e8q.Encoder(shapes, S, dtype, block, 1.0, dequant, scales is not None, esc_cap=4096, ovf_cap=4096)
    ref = _snapshot(enc(W, sc))
    got = []
    for _ in range(2):
        _scrub(enc.result())
        got.append(_snapshot(enc.run_noalloc(W, sc)))
    return ref, got


def _assert_same(ref, got):
    for k in ("idx", "scale", "dq"):
        for a, b in zip(ref[k], got[k]):
            np.testing.assert_array_equal(a, b, err_msg=k)
    for k in ("esc", "ovf"):
        assert ref[k].tobytes() == got[k].tobytes(), k
    np.testing.assert_array_equal(ref["erp"], got["erp"])
    np.testing.assert_array_equal(ref["orp"], got["orp"])
    assert ref["ctr"] == got["ctr"]


@pytest.mark.gpu
def test_noalloc_empty_call_writes_csr_terminators():
    """A call whose only matrix has no rows launches no kernel: the entry
    point still clears the counters and writes the CSR terminators."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_e8_lattice_b200 import e8q

    e8q.init()
    d = synth.signs(32, 256)
    ref, got = _run_pair(e8q, [(0, 256)], [np.zeros((0, 256), np.float32)], [d], torch.float32, "none")
    for g in got:
        _assert_same(ref, g)
        np.testing.assert_array_equal(g["erp"], [0])
        np.testing.assert_array_equal(g["orp"], [0])
        assert all(v == 0 for v in g["ctr"].values()), g["ctr"]


@pytest.mark.gpu
def test_noalloc_given_scales_no_dequant():
    """scale_in = 1 (fixed reconstruction scales, including a zero and a
    non-finite one) with no dequant output: the scales the caller passes are
    the ones used, and both entry points agree bit for bit."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_e8_lattice_b200 import e8q

    e8q.init()
    rng = np.random.default_rng(33)
    m = (rng.standard_normal((24, 512)) * 0.02).astype(np.float32)
    s = (np.sqrt((m.astype(np.float64) ** 2).mean(1)) * rng.uniform(0.5, 1.5, 24)).astype(np.float32)
    s[3], s[7] = 0.0, np.inf
    d = synth.signs(33, 512)
    ref, got = _run_pair(e8q, [m.shape], [m], [d], torch.float32, "none", scales=[s])
    np.testing.assert_array_equal(ref["scale"][0], s)
    assert (ref["idx"][0][3] == 0).all() and (ref["idx"][0][7] == 0).all()
    for g in got:
        _assert_same(ref, g)


@pytest.mark.gpu
def test_noalloc_rotated_dequant_bf16_narrow():
    """bf16 rows 96 wide (both entry points take the general kernel) with the
    rotated-basis dequant: outputs agree bit for bit, and the dequant is the
    exact bf16 product of the encoded points."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_e8_lattice_b200 import e8q

    e8q.init()
    rng = np.random.default_rng(34)
    w = synth.f64_to_bf16_bits(rng.standard_normal((50, 96)) * 0.02)
    d = synth.signs(34, 96)
    ref, got = _run_pair(e8q, [w.shape], [w], [d], torch.bfloat16, "rotated")
    for g in got:
        _assert_same(ref, g)
    P, _, _, _, _ = gpu_points(got[1]["idx"][0].reshape(-1), got[1]["esc"], got[1]["ovf"], 50 * 12)
    want, _ = oracle.dequant(P, got[1]["scale"][0].astype(np.float64), d, 32, "rotated")
    np.testing.assert_array_equal(got[1]["dq"][0].view(np.uint16).reshape(want.shape), want)


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Host-side check, no device work: 300,000 one-row tiles need 2.4 MB of
    tile status, more than the built-in 2 MiB."""
    from bit_e8_lattice_b200 import build, e8q

    build.build()
    L = e8q.lib()
    m = e8q.Matrix()
    m.w = m.signs = m.idx = m.scale = 0x100000
    m.dequant = None
    m.rows, m.cols, m.rht_block, m.in_dtype = 300000, 8192, 0, 1
    a = e8q.EncodeArgs()
    a.kappa, a.dequant, a.scale_in, a.counters = 1.0, 0, 0, 0x100000
    mats = (e8q.Matrix * 1)(m)
    assert L.e8q_project_encode_noalloc(mats, 1, ctypes.byref(a), None) == 5
    assert L.e8q_status_string(5).startswith(b"problem too large")
