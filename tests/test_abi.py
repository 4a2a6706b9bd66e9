"""CPU-side checks of the C ABI: the library loads, exports every function
that include/e8q.h declares, rejects bad arguments before touching a
device, and its host-built core table agrees with the oracle's
(Table 3, core decoding agreement).  No compute call is made here."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "e8q.h")


@pytest.fixture(scope="module")
def lib():
    from bit_e8_lattice_b200 import build, e8q

    build.build()
    return e8q.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(e8q_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_function_is_exported(lib):
    names = declared_functions()
    assert {"e8q_project_encode", "e8q_decode", "e8q_dequant_gemv"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_struct_sizes_match_header():
    from bit_e8_lattice_b200 import e8q

    assert ctypes.sizeof(e8q.Matrix) == 64
    assert ctypes.sizeof(e8q.EncodedC) == 104
    assert e8q.ESC_DTYPE.itemsize == 8
    assert e8q.OVF_DTYPE.itemsize == 20


def test_status_strings(lib):
    assert lib.e8q_status_string(0) == b"ok"
    assert lib.e8q_status_string(1) == b"invalid argument"
    assert lib.e8q_status_string(4) == b"workspace too small"


def test_core_table_matches_oracle(lib):
    import oracle
    from bit_e8_lattice_b200 import e8q

    np.testing.assert_array_equal(e8q.core_table(), oracle.core_points())


def _mat(rows=4, cols=64, block=0, dtype=1):
    from bit_e8_lattice_b200 import e8q

    m = e8q.Matrix()
    m.w = m.signs = m.idx = m.scale = 0x100000  # never dereferenced: the call fails before any device work
    m.dequant = None
    m.rows, m.cols, m.rht_block, m.in_dtype = rows, cols, block, dtype
    return m


def _args(**kw):
    from bit_e8_lattice_b200 import e8q

    a = e8q.EncodeArgs()
    a.kappa = kw.get("kappa", 1.0)
    a.dequant = kw.get("dequant", 0)
    a.scale_in = 0
    a.counters = 0x100000
    return a


@pytest.mark.parametrize("kw,expect", [
    (dict(cols=12), 1),            # not a multiple of 8
    (dict(cols=16392), 2),         # wider than the library handles
    (dict(block=3), 1),            # not a power of two
    (dict(block=4096), 1),         # larger than 2048
    (dict(cols=96, block=64), 1),  # does not divide cols
    (dict(dtype=7), 1),
    (dict(rows=-1), 1),
])
def test_encode_rejects_bad_matrices(lib, kw, expect):
    from bit_e8_lattice_b200 import e8q

    mats = (e8q.Matrix * 1)(_mat(**kw))
    rc = lib.e8q_project_encode(mats, 1, ctypes.byref(_args()), ctypes.c_void_p(0x100000), 1 << 20, None)
    assert rc == expect


def test_encode_rejects_bad_args(lib):
    from bit_e8_lattice_b200 import e8q

    mats = (e8q.Matrix * 1)(_mat())
    assert lib.e8q_project_encode(mats, 0, ctypes.byref(_args()), ctypes.c_void_p(0x100000), 1 << 20, None) == 1
    assert lib.e8q_project_encode(mats, 1, ctypes.byref(_args(kappa=0.0)), ctypes.c_void_p(0x100000), 1 << 20, None) == 1
    assert lib.e8q_project_encode(mats, 1, ctypes.byref(_args(dequant=5)), ctypes.c_void_p(0x100000), 1 << 20, None) == 1
    # dequant requested without an output buffer
    assert lib.e8q_project_encode(mats, 1, ctypes.byref(_args(dequant=2)), ctypes.c_void_p(0x100000), 1 << 20, None) == 1
    # workspace too small
    need = lib.e8q_encode_workspace_bytes(mats, 1)
    assert need >= 16
    assert lib.e8q_project_encode(mats, 1, ctypes.byref(_args()), ctypes.c_void_p(0x100000), need - 1, None) == 4
    assert lib.e8q_project_encode(mats, 449, ctypes.byref(_args()), ctypes.c_void_p(0x100000), 1 << 20, None) == 2


def test_workspace_bytes_counts_tiles(lib):
    from bit_e8_lattice_b200 import e8q

    # 37 rows of 256 columns: one tile of the bf16 path (up to 64 rows of
    # 28,672 elements); 3 rows of 14336: 2 rows per tile -> 2 tiles; the
    # status words need 16 + 8 * 3 bytes, and the bf16 path adds a per-CTA
    # scratch of 4 x 3584 x 16 bytes
    mats = (e8q.Matrix * 2)(_mat(rows=37, cols=256), _mat(rows=3, cols=14336))
    n = lib.e8q_encode_workspace_bytes(mats, 2)
    assert n % 256 == 0 and n >= 16 + 8 * 3
    assert n <= 256 + 3 * 4 * 3584 * 16
    mats = (e8q.Matrix * 1)(_mat(rows=4096, cols=14336))
    n = lib.e8q_encode_workspace_bytes(mats, 1)
    # status words for the general kernel's 4096 one-row tiles (either path may run)
    assert n >= 16 + 8 * 4096 and n <= (16 + 8 * 4096 + 255) // 256 * 256 + 160 * 4 * 3584 * 16


def test_decode_and_gemv_reject_bad_args(lib):
    from bit_e8_lattice_b200 import e8q

    m = e8q.EncodedC(0x100000, 0x100000, 0x100000, None, None, None, None, 0, 0, 4, 12, 0, 0, 0)
    assert lib.e8q_decode(ctypes.byref(m), 1, ctypes.c_void_p(0x100000), None) == 1  # cols % 8
    m.cols = 64
    assert lib.e8q_decode(ctypes.byref(m), 9, ctypes.c_void_p(0x100000), None) == 1  # basis
    assert lib.e8q_dequant_gemv(ctypes.byref(m), ctypes.c_void_p(0x100000), 0, ctypes.c_void_p(0x100000),
                                ctypes.c_void_p(0x100000), 1 << 20, None) == 1  # batch 0
    need = lib.e8q_gemv_workspace_bytes(ctypes.byref(m), 4)
    # fp32 and fp16 rotated activations, scale exponents, chunk offsets, partial sums
    assert need % 256 == 0 and need >= 4 * 64 * 4 + 4 * 64 * 2
    assert lib.e8q_gemv_workspace_bytes(ctypes.byref(m), 257) == 256
    assert lib.e8q_dequant_gemv(ctypes.byref(m), ctypes.c_void_p(0x100000), 4, ctypes.c_void_p(0x100000),
                                ctypes.c_void_p(0x100000), need - 1, None) == 4


def test_ste_backward_argument_checks(lib):
    """The identity-STE backward rejects bad arguments, returns at once for
    an aliased or empty call (nothing to launch, so no device is needed),
    and refuses partially overlapping buffers."""
    vp = ctypes.c_void_p
    assert lib.e8q_ste_backward(vp(0x100000), vp(0x200000), -1, None) == 1
    assert lib.e8q_ste_backward(None, vp(0x200000), 8, None) == 1
    assert lib.e8q_ste_backward(vp(0x100001), vp(0x200000), 8, None) == 1  # odd address
    assert lib.e8q_ste_backward(vp(0x100000), vp(0x100000), 1 << 20, None) == 0  # aliased: the identity
    assert lib.e8q_ste_backward(None, None, 0, None) == 0
    assert lib.e8q_ste_backward(vp(0x100000), vp(0x100010), 64, None) == 1  # overlap by 112 bytes


def test_gemv_workspace_holds_its_parts(lib):
    """The GEMV workspace holds the fp32 and fp16 rotated activations, the
    root map (one byte a group) and the main kernel's partial-sum slots."""
    from bit_e8_lattice_b200 import e8q

    m = e8q.EncodedC(0x100000, 0x100000, 0x100000, None, None, None, None, 0, 0, 4096, 14336, 0, 0, 0)
    need = lib.e8q_gemv_workspace_bytes(ctypes.byref(m), 64)
    assert need >= 64 * 14336 * 4 + 64 * 14336 * 2 + 4096 * 1792
    assert lib.e8q_gemv_workspace_bytes(ctypes.byref(m), 0) == 256
    assert lib.e8q_gemv_workspace_bytes(ctypes.byref(m), 257) == 256


def test_gemm_argument_checks_and_workspace(lib):
    """The fused GEMM rejects bad batches, misaligned activations and short
    workspaces before touching a device, and its workspace holds the fp16
    activation image (whole 256-token tiles x 32-column K tiles), the row
    map and the per-split cursor headers; the plan depends on the shapes
    only, so the size is exact."""
    from bit_e8_lattice_b200 import e8q

    vp = ctypes.c_void_p
    m = e8q.EncodedC(0x100000, 0x100000, 0x100000, None, None, None, None, 0, 0, 4096, 14336, 0, 0, 0)
    for bad in (0, -1, 65537):
        assert lib.e8q_gemm_workspace_bytes(ctypes.byref(m), bad) == 256
        assert lib.e8q_dequant_gemm(ctypes.byref(m), vp(0x100000), bad, vp(0x100000), vp(0x100000), 1 << 40,
                                    None) == 1
    for batch in (64, 256, 1000, 4096):
        need = lib.e8q_gemm_workspace_bytes(ctypes.byref(m), batch)
        tiles = (batch + 255) // 256
        assert need % 256 == 0
        assert need >= tiles * 256 * 14336 * 2 + 4096 * 14336 // 8 + 4096 * 32
        assert need == lib.e8q_gemm_workspace_bytes(ctypes.byref(m), batch)
        assert lib.e8q_dequant_gemm(ctypes.byref(m), vp(0x100008), batch, vp(0x100000), vp(0x100000), need,
                                    None) == 1  # x not 16-byte aligned
        assert lib.e8q_dequant_gemm(ctypes.byref(m), vp(0x100000), batch, vp(0x100000), vp(0x100000), need - 1,
                                    None) == 4
        assert lib.e8q_dequant_gemm(ctypes.byref(m), vp(0x100000), batch, vp(0x100000), vp(0x100080), need,
                                    None) == 4  # workspace not 256-byte aligned
    m.cols = 12
    assert lib.e8q_gemm_workspace_bytes(ctypes.byref(m), 64) == 256  # cols % 8


def test_gemm_plan_splits_k_where_tiles_are_few(lib):
    """The GEMM's K split (read off its exact workspace: fp32 partial sums
    exist only with several splits): a 4096-row matrix at 64 activation rows
    has 32 row tiles for 148 SMs and is split; a 14336-row matrix at 4096
    rows has 1,792 units and is not."""
    from bit_e8_lattice_b200 import e8q

    def rnd(x):
        return (x + 255) // 256 * 256

    def unsplit(rows, cols, batch):
        nkt = (cols + 31) // 32
        ntt = (batch + 255) // 256
        mstride = (4 * nkt + 7) // 8 * 8
        return 256 + rnd(ntt * nkt * 16384) + rnd(ntt * 256 * 4) + rnd(rows * mstride * 2) + rnd(rows)

    for rows, cols, batch, split in ((4096, 14336, 64, True), (4096, 14336, 256, True),
                                     (14336, 4096, 4096, False), (14336, 4096, 64, False)):
        m = e8q.EncodedC(0x100000, 0x100000, 0x100000, None, None, None, None, 0, 0, rows, cols, 0, 0, 0)
        need = lib.e8q_gemm_workspace_bytes(ctypes.byref(m), batch)
        base = unsplit(rows, cols, batch)
        if split:
            parts = (need - base) // (batch * rows * 4)
            assert need > base and 2 <= parts <= 32, (rows, cols, batch, need, base)
        else:
            assert need == base, (rows, cols, batch, need, base)


def test_escape_table_matches_oracle(lib):
    """Every E8 point with |p|^2 <= 22 (1,113,841 points), plus a shell
    beyond: the kernels' lookup table gives the oracle's encoding (core
    index; escape core index and root; overflow).  E8-QAT appendix Table 3,
    single-root membership."""
    import lattice_np
    import oracle
    from bit_e8_lattice_b200 import e8q

    P, n2 = lattice_np.e8_points(88)
    assert len(P) == 1113841
    far, _ = lattice_np.e8_points(96, 96)
    P = np.concatenate([P, far[::7]], 0)
    words = e8q.escape_lookup(P)
    out = oracle.project_encode_vectors(P / 2.0)
    kind, idx, root = out["kind"], out["idx"], out["root"]
    assert (out["P"] == P).all()
    expect = np.where(kind == 0, idx, np.where(kind == 1, idx | (root << 16) | (1 << 24), 2 << 24)).astype(np.uint32)
    bad = np.nonzero(words != expect)[0]
    assert len(bad) == 0, (len(bad), P[bad[:3]], words[bad[:3]], expect[bad[:3]])
    assert (kind[-len(far[::7]):] == 2).all()


def test_bench_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    """bench.py matches a committed ncu summary to the kernels by a hash of
    the kernel sources without comments and blank space: a comment edit keeps
    the hash, a code edit changes it."""
    import shutil
    import sys

    sys.path.insert(0, ROOT)
    import bench

    src = os.path.join(ROOT, "bit_e8_lattice_b200", "csrc")
    dst = tmp_path / "bit_e8_lattice_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.source_sha()
    f = dst / "ptx.cuh"
    f.write_text(f.read_text() + "\n// a comment\n/* and\n another */\n\n")
    assert bench.source_sha() == base
    f.write_text(f.read_text() + "\nnamespace e8q { constexpr int kProbe = 1; }\n")
    assert bench.source_sha() != base
    # a kernel's own hash follows only the files it is built from
    enc = bench.source_sha("k_encode_fast")
    g = dst / "gemm_tc.cuh"
    g.write_text(g.read_text() + "\nnamespace e8q { constexpr int kProbe2 = 2; }\n")
    assert bench.source_sha("k_encode_fast") == enc and bench.source_sha() != base
    f.write_text(f.read_text() + "\nnamespace e8q { constexpr int kProbe3 = 3; }\n")
    assert bench.source_sha("k_encode_fast") != enc
