"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Inputs come from ``bit_e8_lattice_b200.synth``; expected values from
``oracle`` only.  Tolerances are stated in ``tests/parity.py``.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_e8_lattice_b200 import synth
from parity import (MARGIN, check_encode, check_encode_far, check_gemv, check_original_dequant, check_rotated_dequant,
                    gpu_points, merge_rows, oracle_rows_parallel, oracle_rows_stream)
import lattice_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def e8q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_e8_lattice_b200 import e8q as m

    m.init()
    return m


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_idx(t):
    return t.cpu().numpy().view(np.uint16)


def run_encode(e8q, mats, signs, blocks=0, kappa=1.0, dequant="none", scales=None, dtype=torch.bfloat16,
               esc_cap=None, ovf_cap=None, allow_drop=False):
    ws = [dev_bf16(m) if dtype == torch.bfloat16 else dev(m.astype(np.float32)) for m in mats]
    ss = [dev(s) for s in signs]
    sc = [dev(s.astype(np.float32)) for s in scales] if scales is not None else None
    groups = sum(m.shape[0] * (m.shape[1] // 8) for m in mats)
    esc_cap = max(64, groups) if esc_cap is None else esc_cap
    ovf_cap = max(64, groups) if ovf_cap is None else ovf_cap
    enc = e8q.Encoder([w.shape for w in ws], ss, dtype, blocks, kappa, dequant, scales is not None, esc_cap, ovf_cap)
    res = enc(ws, sc)
    torch.cuda.synchronize()
    ctr = res.read_counters()
    assert ctr["err"] == 0, ctr
    assert allow_drop or ctr["n_dropped"] == 0, ctr
    return enc, res


def values(m, dtype):
    return synth.bf16_bits_to_f64(m) if dtype == torch.bfloat16 else m.astype(np.float64)


def compare_all(e8q, res, mats, signs, blocks, kappa=1.0, dtype=torch.bfloat16, label="", rows=None):
    ctr = res.read_counters()
    assert ctr["err"] == 0 and ctr["n_dropped"] == 0, ctr
    esc, ovf = res.escape_records(), res.overflow_records()
    stats = []
    for i, m in enumerate(mats):
        C = m.shape[1]
        B = blocks[i] if isinstance(blocks, (list, tuple)) else blocks
        B = oracle.default_block(C) if B == 0 else B
        rsel = np.arange(m.shape[0]) if rows is None else rows[i]
        out = oracle.project_encode(values(m, dtype)[rsel], signs[i], B, kappa)
        st = check_encode(out, host_idx(res.idx[i]), res.scale[i].cpu().numpy(), esc, ovf, res.group_base[i], rsel,
                          C // 8, label=f"{label}[{i}]")
        stats.append(st)
    return stats


# ----------------------------------------------------------------------
def test_core_decoding_agreement_decode_and_gemv(e8q):
    """Table 3: all 65,536 core codewords decode to the same coordinates
    through the decode kernel and through the GEMV kernel."""
    core = oracle.core_points().astype(np.int32)
    idx = torch.arange(65536, dtype=torch.int32).to(torch.int16).reshape(65536, 1).cuda()
    scale = torch.full((65536,), 2.0, dtype=torch.float32, device="cuda")
    signs = torch.ones(8, dtype=torch.int8, device="cuda")
    m = e8q.Encoded(idx, scale, signs, None, None, None, None, 65536, 8, 0, 1)
    out = e8q.e8q_decode(m, "rotated")
    got = synth.bf16_bits_to_f64(out.cpu().view(torch.int16).numpy().view(np.uint16))
    np.testing.assert_array_equal(got, core.astype(np.float64))  # 2 * P/2 = P, exact in bf16
    x = dev_bf16(synth.f64_to_bf16_bits(np.eye(8)))
    y = e8q.Gemv(m, 8)(x)
    got = synth.bf16_bits_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16)).T
    np.testing.assert_array_equal(got, core.astype(np.float64))


def test_small_f32_encode_decode(e8q):
    w, d = synth.small_f32()
    enc, res = run_encode(e8q, [w], [d], 256, dtype=torch.float32, dequant="rotated")
    st = compare_all(e8q, res, [w], [d], 256, dtype=torch.float32, label="small_f32")[0]
    assert st["near_ties"] <= 4 and 0.1 < st["rho"] < 0.4
    P = st["points"]
    scale = res.scale[0].cpu().numpy()
    dq = res.dequant[0].cpu().view(torch.int16).numpy()
    check_rotated_dequant(dq, P, scale, d, 256, "encode dequant rotated")
    enc_m = res.encoded[0]
    out = e8q.e8q_decode(enc_m, "rotated").cpu().view(torch.int16).numpy()
    check_rotated_dequant(out, P, scale, d, 256, "decode rotated")
    out = e8q.e8q_decode(enc_m, "original").cpu().view(torch.int16).numpy()
    check_original_dequant(out, P, scale, d, 256, "decode original")


def test_free_vectors_exact_projection(e8q):
    """4,096 vectors 3*N(0, I), no transform, scale 1: the projection sees
    exactly the oracle's x."""
    x = synth.free_vectors()
    ones = np.ones(8, np.int8)
    enc, res = run_encode(e8q, [x], [ones], 1, dtype=torch.float32, scales=[np.ones(len(x))])
    out = oracle.project_encode_vectors(x.astype(np.float64))
    out["scale"] = np.ones(len(x))
    out["x"] = x.astype(np.float64)
    st = check_encode(out, host_idx(res.idx[0]), res.scale[0].cpu().numpy(), res.escape_records(),
                      res.overflow_records(), 0, None, 1, "free_vectors")
    assert st["overflow"] > 0


@pytest.mark.parametrize("lo,hi", [(0, 48), (56, 56), (64, 64)])
def test_escape_rule_on_whole_shells(e8q, lo, hi):
    """Every E8 point of |p|^2 <= 12, = 14 and = 16 given exactly: core
    index, escape root and overflow decision agree with the oracle's
    brute-force search over the 240 roots."""
    P, _ = lattice_np.e8_points(hi, lo)
    x = (P / 2.0).astype(np.float32)
    enc, res = run_encode(e8q, [x], [np.ones(8, np.int8)], 1, dtype=torch.float32, scales=[np.ones(len(x))],
                          esc_cap=len(x), ovf_cap=len(x))
    out = oracle.project_encode_vectors(x.astype(np.float64))
    np.testing.assert_array_equal(out["P"], P)
    Pg, kind, root, _, _ = gpu_points(host_idx(res.idx[0]).reshape(-1), res.escape_records(), res.overflow_records(),
                                      len(x))
    np.testing.assert_array_equal(Pg, P)
    np.testing.assert_array_equal(host_idx(res.idx[0]).reshape(-1).astype(np.int64), out["idx"])
    np.testing.assert_array_equal(kind, out["kind"])
    np.testing.assert_array_equal(root[kind == 1], out["root"][kind == 1])


def test_attn_2048_full(e8q):
    w, d = synth.attn_2048()
    enc, res = run_encode(e8q, [w], [d], 0, dequant="original")
    st = compare_all(e8q, res, [w], [d], [2048], label="attn_2048")[0]
    assert st["near_ties"] < 200
    P = st["points"]
    scale = res.scale[0].cpu().numpy()
    check_original_dequant(res.dequant[0].cpu().view(torch.int16).numpy(), P, scale, d, 2048, "attn original")
    out = e8q.e8q_decode(res.encoded[0], "rotated").cpu().view(torch.int16).numpy()
    check_rotated_dequant(out, P, scale, d, 2048, "attn decode rotated")


def test_moe_batched_two_experts_full(e8q):
    mats = synth.moe_bank(experts=2)
    W = [m for m, _ in mats]
    S = [s for _, s in mats]
    enc, res = run_encode(e8q, W, S, 0)
    stats = compare_all(e8q, res, W, S, 0, label="moe2")
    for st in stats:
        assert st["groups"] > 0


@pytest.mark.parametrize("rows,cols,block", [(37, 256, 0), (5, 8, 0), (9, 24, 0), (3, 40, 0), (6, 96, 0),
                                             (70, 64, 0), (4, 16384, 0), (3, 768, 256), (2, 4096, 512), (129, 8, 1)])
def test_shapes_and_ragged_tiles(e8q, rows, cols, block):
    rng = np.random.default_rng(rows * 1000 + cols)
    w = synth.f64_to_bf16_bits(rng.standard_normal((rows, cols)) * 0.03)
    d = synth.signs(rows, cols)
    enc, res = run_encode(e8q, [w], [d], block, dequant="original")
    B = oracle.default_block(cols) if block == 0 else block
    st = compare_all(e8q, res, [w], [d], [B], label=f"{rows}x{cols}")[0]
    check_original_dequant(res.dequant[0].cpu().view(torch.int16).numpy(), st["points"], res.scale[0].cpu().numpy(),
                           d, B, "original")
    rp = res.esc_row_ptr.cpu().numpy()
    assert rp[0] == 0 and (np.diff(rp) >= 0).all() and rp[-1] == res.read_counters()["n_escape"]


def test_f32_input_block_2048(e8q):
    rng = np.random.default_rng(77)
    w = (rng.standard_normal((40, 4096)) * 0.02).astype(np.float32)
    d = synth.signs(77, 4096)
    enc, res = run_encode(e8q, [w], [d], 0, dtype=torch.float32)
    compare_all(e8q, res, [w], [d], [2048], dtype=torch.float32, label="f32_4096")


@pytest.mark.parametrize("kappa", [0.6, 2.5])
def test_kappa(e8q, kappa):
    w, d = synth.small_f32()
    enc, res = run_encode(e8q, [w], [d], 0, kappa=kappa, dtype=torch.float32)
    compare_all(e8q, res, [w], [d], [256], kappa=kappa, dtype=torch.float32, label=f"kappa{kappa}")


def test_nonfinite_and_zero_rows(e8q):
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((6, 64)) * 0.02).astype(np.float32)
    w[1, 3] = np.nan
    w[2, 10] = np.inf
    w[2, 11] = -np.inf
    w[3] = 0.0
    d = synth.signs(5, 64)
    enc, res = run_encode(e8q, [w], [d], 0, dtype=torch.float32)
    ctr = res.read_counters()
    assert ctr["n_nonfinite"] == 3
    out = oracle.project_encode(w.astype(np.float64), d, 64)
    assert out["nonfinite"] == 3
    check_encode(out, host_idx(res.idx[0]), res.scale[0].cpu().numpy(), res.escape_records(), res.overflow_records(),
                 0, None, 8, "nonfinite")
    assert res.scale[0].cpu().numpy()[3] == 0.0 and (host_idx(res.idx[0])[3] == 0).all()


def test_bf16_tiles_dequant_both_bases(e8q):
    """256-wide bf16 rows (64 rows per tile) with both dequant outputs."""
    rng = np.random.default_rng(21)
    w = synth.f64_to_bf16_bits(rng.standard_normal((200, 256)) * 0.02)
    d = synth.signs(21, 256)
    for mode in ("rotated", "original"):
        enc, res = run_encode(e8q, [w], [d], 0, dequant=mode)
        st = compare_all(e8q, res, [w], [d], [256], label=f"bf16 256 {mode}")[0]
        dq = res.dequant[0].cpu().view(torch.int16).numpy()
        scale = res.scale[0].cpu().numpy()
        if mode == "rotated":
            check_rotated_dequant(dq, st["points"], scale, d, 256, "rotated")
        else:
            check_original_dequant(dq, st["points"], scale, d, 256, "original")
        out = e8q.e8q_decode(res.encoded[0], mode).cpu().view(torch.int16).numpy()
        np.testing.assert_array_equal(out, dq)  # decode reproduces the encode-time output bit for bit


def test_bf16_nonfinite_inputs(e8q):
    rng = np.random.default_rng(22)
    w = synth.f64_to_bf16_bits(rng.standard_normal((8, 2048)) * 0.02)
    w[1, 5] = 0x7FC0   # NaN
    w[3, 100] = 0x7F80  # +Inf
    w[3, 2000] = 0xFF80  # -Inf
    w[6] = 0           # zero row
    d = synth.signs(22, 2048)
    enc, res = run_encode(e8q, [w], [d], 0, dequant="original")
    assert res.read_counters()["n_nonfinite"] == 3
    vals = synth.bf16_bits_to_f64(w)
    out = oracle.project_encode(vals, d, 2048)
    assert out["nonfinite"] == 3
    st = check_encode(out, host_idx(res.idx[0]), res.scale[0].cpu().numpy(), res.escape_records(),
                      res.overflow_records(), 0, None, 256, "bf16 nonfinite")
    check_original_dequant(res.dequant[0].cpu().view(torch.int16).numpy(), st["points"], res.scale[0].cpu().numpy(),
                           d, 2048, "nonfinite original")


@pytest.mark.parametrize("kappa", [0.45, 1.0, 1.5, 200.0])
def test_decode_record_heavy_tiles(e8q, kappa):
    """Decode of 2048-wide rows (7 rows a tile, ragged last tile) at scales
    whose tiles hold no records, or hundreds to thousands of them:
    bit-identical to the encode's own dequant in both bases, and the rotated
    one equal to the oracle's s * p."""
    rng = np.random.default_rng(int(kappa * 100) + 9)
    w = synth.f64_to_bf16_bits(rng.standard_normal((50, 2048)) * 0.02)
    d = synth.signs(31, 2048)
    for mode in ("rotated", "original"):
        enc, res = run_encode(e8q, [w], [d], 0, kappa=kappa, dequant=mode)
        st = compare_all(e8q, res, [w], [d], [2048], kappa=kappa, label=f"kappa{kappa} {mode}")[0]
        dq = res.dequant[0].cpu().view(torch.int16).numpy()
        out = e8q.e8q_decode(res.encoded[0], mode).cpu().view(torch.int16).numpy()
        np.testing.assert_array_equal(out, dq)
        if mode == "rotated":
            check_rotated_dequant(out, st["points"], res.scale[0].cpu().numpy(), d, 2048, f"kappa{kappa} decode")
    ctr = res.read_counters()
    per_tile = 7 * 2048 // 8
    if kappa == 200.0:
        assert ctr["n_overflow"] > 2 * per_tile  # every tile past the staging warp's first round
    if kappa == 1.5:
        assert ctr["n_escape"] > 8 * 512 and ctr["n_overflow"] > 8 * 64


def test_large_points_small_scale(e8q):
    """kappa = 200: |x| in the hundreds, lattice points far outside the core
    (overflow records with large coordinates) and the original-basis dequant
    of large |P|."""
    rng = np.random.default_rng(23)
    w = synth.f64_to_bf16_bits(rng.standard_normal((4, 2048)) * 0.02)
    d = synth.signs(23, 2048)
    enc, res = run_encode(e8q, [w], [d], 0, kappa=200.0, dequant="original")
    st = compare_all(e8q, res, [w], [d], [2048], kappa=200.0, label="kappa200")[0]
    assert np.abs(st["points"]).max() > 255
    check_original_dequant(res.dequant[0].cpu().view(torch.int16).numpy(), st["points"], res.scale[0].cpu().numpy(),
                           d, 2048, "kappa200 original")


def test_bf16_capacity_and_scale_in(e8q):
    w, d = synth.attn_2048()
    _, full = run_encode(e8q, [w], [d], 0)
    tot = full.read_counters()
    ref_e, ref_o = full.escape_records().copy(), full.overflow_records().copy()
    ref_rp = full.esc_row_ptr.cpu().numpy().copy()
    _, res = run_encode(e8q, [w], [d], 0, esc_cap=1000, ovf_cap=10, allow_drop=True)
    ctr = res.read_counters()
    assert ctr["n_dropped"] == (tot["n_escape"] - 1000) + (tot["n_overflow"] - 10)
    np.testing.assert_array_equal(res.escape_records()[:1000], ref_e[:1000])
    np.testing.assert_array_equal(res.overflow_records()[:10], ref_o[:10])
    np.testing.assert_array_equal(res.esc_row_ptr.cpu().numpy(), ref_rp)
    s = full.scale[0].cpu().numpy()
    _, given = run_encode(e8q, [w], [d], 0, scales=[s])
    np.testing.assert_array_equal(host_idx(given.idx[0]), host_idx(full.idx[0]))
    assert given.escape_records().tobytes() == ref_e.tobytes()


def test_empty_matrix(e8q):
    d = synth.signs(1, 64)
    enc, res = run_encode(e8q, [np.zeros((0, 64), np.uint16)], [d], 0)
    ctr = res.read_counters()
    assert ctr["n_escape"] == 0 and ctr["n_overflow"] == 0
    assert res.esc_row_ptr.cpu().numpy().tolist() == [0]


def test_capacity_shortfall_is_reported(e8q):
    w, d = synth.small_f32()
    _, full = run_encode(e8q, [w], [d], 0, dtype=torch.float32)
    ref_e = full.escape_records().copy()
    ref_rp = full.esc_row_ptr.cpu().numpy().copy()
    tot = full.read_counters()
    _, res = run_encode(e8q, [w], [d], 0, dtype=torch.float32, esc_cap=5, ovf_cap=0, allow_drop=True)
    ctr = res.read_counters()
    assert ctr["n_escape"] == tot["n_escape"] and ctr["n_overflow"] == tot["n_overflow"]
    assert ctr["n_dropped"] == (tot["n_escape"] - 5) + tot["n_overflow"]
    np.testing.assert_array_equal(res.escape_records()[:5], ref_e[:5])
    np.testing.assert_array_equal(res.esc_row_ptr.cpu().numpy(), ref_rp)


def test_scale_in(e8q):
    w, d = synth.small_f32()
    s = np.sqrt((w.astype(np.float64) ** 2).mean(1)) * 0.75
    enc, res = run_encode(e8q, [w], [d], 0, dtype=torch.float32, scales=[s.astype(np.float32)])
    # the oracle with a fixed scale: kappa chosen so that rms / kappa == s
    s32 = s.astype(np.float32).astype(np.float64)
    out = oracle.project_encode(w.astype(np.float64), d, 256, kappa=1.0 / 0.75)
    np.testing.assert_allclose(res.scale[0].cpu().numpy(), s32, rtol=0)
    np.testing.assert_allclose(out["scale"], s32, rtol=1e-6)
    check_encode(out, host_idx(res.idx[0]), out["scale"], res.escape_records(), res.overflow_records(), 0, None, 32,
                 "scale_in")


def test_deterministic_outputs(e8q):
    w, d = synth.attn_2048()
    _, a = run_encode(e8q, [w], [d], 0)
    ia, ea, oa = host_idx(a.idx[0]).copy(), a.escape_records().copy(), a.overflow_records().copy()
    sa = a.scale[0].cpu().numpy().copy()
    _, b = run_encode(e8q, [w], [d], 0)
    np.testing.assert_array_equal(ia, host_idx(b.idx[0]))
    np.testing.assert_array_equal(sa, b.scale[0].cpu().numpy())
    assert ea.tobytes() == b.escape_records().tobytes() and oa.tobytes() == b.overflow_records().tobytes()



@pytest.mark.parametrize("batch", [1, 4, 16, 64])
def test_gemv_small(e8q, batch):
    rng = np.random.default_rng(batch)
    w = synth.f64_to_bf16_bits(rng.standard_normal((512, 2048)) * 0.015)
    d = synth.signs(batch, 2048)
    enc, res = run_encode(e8q, [w], [d], 0)
    st = compare_all(e8q, res, [w], [d], [2048], label="gemv_w")[0]
    xb = synth.gemv_x(batch, 2048)
    y = e8q.Gemv(res.encoded[0], batch)(dev_bf16(xb))
    torch.cuda.synchronize()
    y_ref = oracle.gemv(st["points"], res.scale[0].cpu().numpy().astype(np.float64), d, 2048,
                        synth.bf16_bits_to_f64(xb))
    check_gemv(y.cpu().view(torch.int16).numpy(), y_ref, f"gemv b={batch}")


@pytest.mark.parametrize("rows,cols,batch,kappa", [
    (37, 264, 3, 1.0),      # one partial 256-column chunk + RHT block 8, rows not a multiple of 32
    (129, 8, 1, 1.0),       # one group per row
    (70, 64, 9, 1.0),       # two batch tiles, ragged second tile
    (5, 768, 100, 1.0),     # two passes over batch tiles (8 + 5)
    (33, 2056, 256, 1.0),   # largest batch, 9 chunks, block 8
    (300, 1536, 17, 2.5),   # many escapes and overflow records
    (128, 128, 16, 1.0),    # one 128-row tile, one 128-column K tile
    (257, 4096, 64, 1.0),   # three row tiles (the last of one row), several K splits
])
def test_gemv_shapes(e8q, rows, cols, batch, kappa):
    rng = np.random.default_rng(rows * 7 + cols)
    w = synth.f64_to_bf16_bits(rng.standard_normal((rows, cols)) * 0.02)
    d = synth.signs(rows, cols)
    B = oracle.default_block(cols)
    enc, res = run_encode(e8q, [w], [d], 0, kappa=kappa)
    st = compare_all(e8q, res, [w], [d], [B], kappa=kappa, label="gemv_shape")[0]
    if kappa > 2:
        ctr = res.read_counters()
        assert ctr["n_escape"] > rows and ctr["n_overflow"] > 0, ctr
    xb = synth.gemv_x(batch, cols)
    y = e8q.Gemv(res.encoded[0], batch)(dev_bf16(xb))
    torch.cuda.synchronize()
    y_ref = oracle.gemv(st["points"], res.scale[0].cpu().numpy().astype(np.float64), d, B,
                        synth.bf16_bits_to_f64(xb))
    check_gemv(y.cpu().view(torch.int16).numpy(), y_ref, f"gemv {rows}x{cols} b={batch}")


def test_gemv_large_activations(e8q):
    """Activations near the bf16 range limit: the per-row power-of-two
    scaling keeps the fp16 operand finite."""
    rng = np.random.default_rng(11)
    w = synth.f64_to_bf16_bits(rng.standard_normal((64, 2048)) * 0.02)
    d = synth.signs(3, 2048)
    enc, res = run_encode(e8q, [w], [d], 0)
    st = compare_all(e8q, res, [w], [d], [2048], label="gemv_big_x")[0]
    x = rng.standard_normal((4, 2048))
    x[0] *= 1e30
    x[1] *= 1e-30
    x[2, 5] = 3e33  # one outlier
    xb = synth.f64_to_bf16_bits(x)
    y = e8q.Gemv(res.encoded[0], 4)(dev_bf16(xb))
    torch.cuda.synchronize()
    y_ref = oracle.gemv(st["points"], res.scale[0].cpu().numpy().astype(np.float64), d, 2048,
                        synth.bf16_bits_to_f64(xb))
    got = synth.bf16_bits_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    assert np.isfinite(got).all()
    for b in (0, 1, 3):
        check_gemv(y.cpu().view(torch.int16).numpy()[b:b + 1], y_ref[b:b + 1], f"gemv big x row {b}")
    # row 2: one huge entry dominates; compare normwise only
    rel = np.linalg.norm(got[2] - y_ref[2]) / np.linalg.norm(y_ref[2])
    assert rel < 1e-2, rel


def test_gemv_repeatable(e8q):
    """The partial sums are added in a fixed order: two calls on the same
    inputs give the same bits."""
    rng = np.random.default_rng(21)
    w = synth.f64_to_bf16_bits(rng.standard_normal((700, 4096)) * 0.02)
    d = synth.signs(21, 4096)
    enc, res = run_encode(e8q, [w], [d], 0)
    xb = synth.gemv_x(5, 4096)
    g = e8q.Gemv(res.encoded[0], 5)
    y1 = g(dev_bf16(xb)).clone()
    y2 = g(dev_bf16(xb)).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_gemv_far_overflow_points(e8q):
    """A scale far below the rows' rms (s = rms / kappa, kappa 50) makes
    every group an overflow record, most with doubled coordinates beyond
    +-127; the GEMV applies those records from their 16-bit coordinates."""
    rng = np.random.default_rng(31)
    w = synth.f64_to_bf16_bits(rng.standard_normal((160, 1024)) * 0.02)
    d = synth.signs(31, 1024)
    B = oracle.default_block(1024)
    enc, res = run_encode(e8q, [w], [d], 0, kappa=50.0, esc_cap=160 * 128, ovf_cap=160 * 128)
    st = compare_all(e8q, res, [w], [d], [B], kappa=50.0, label="gemv_farP")[0]
    P = st["points"]
    assert (np.abs(P) > 127).any(axis=1).sum() > 10000
    for batch in (3, 70):
        xb = synth.gemv_x(batch, 1024)
        y = e8q.Gemv(res.encoded[0], batch)(dev_bf16(xb))
        torch.cuda.synchronize()
        y_ref = oracle.gemv(P, res.scale[0].cpu().numpy().astype(np.float64), d, B, synth.bf16_bits_to_f64(xb))
        check_gemv(y.cpu().view(torch.int16).numpy(), y_ref, f"gemv far points b={batch}")


# ----------------------------------------------------------------------
# fused dequant-GEMM (tensor cores, many activation rows)
# ----------------------------------------------------------------------
def run_gemm(e8q, m, xb):
    g = e8q.Gemm(m, xb.shape[0])
    y = g(dev_bf16(xb))
    torch.cuda.synchronize()
    assert g.error_word() == 0, "a bounded wait of the GEMM gave up"
    return y.cpu().view(torch.int16).numpy()


@pytest.mark.parametrize("rows,cols,batch,kappa", [
    (256, 2048, 64, 1.0),     # two row tiles, one token tile of 64, K splits
    (300, 1536, 100, 2.5),    # many escapes and overflow records, ragged rows and tokens
    (129, 264, 257, 1.0),     # last K tile past the row end (33 groups), block 8, a second token tile of 1
    (37, 4096, 512, 1.0),     # one partial row tile, two full token tiles, many K splits (finalize)
    (1000, 256, 300, 1.0),    # eight row tiles, no K split (direct epilogue), ragged second token tile
    (64, 8, 70, 1.0),         # one group per row: three zero groups in the only K tile
    (513, 4096, 1024, 1.0),   # five row tiles, four token tiles
])
def test_gemm_matches_oracle(e8q, rows, cols, batch, kappa):
    rng = np.random.default_rng(rows * 11 + cols + batch)
    w = synth.f64_to_bf16_bits(rng.standard_normal((rows, cols)) * 0.02)
    d = synth.signs(rows + 5, cols)
    B = oracle.default_block(cols)
    enc, res = run_encode(e8q, [w], [d], 0, kappa=kappa)
    st = compare_all(e8q, res, [w], [d], [B], kappa=kappa, label="gemm_shape")[0]
    if kappa > 2:
        ctr = res.read_counters()
        assert ctr["n_escape"] > rows and ctr["n_overflow"] > rows, ctr
    xb = synth.gemv_x(batch, cols)
    y = run_gemm(e8q, res.encoded[0], xb)
    y_ref = oracle.gemv(st["points"], res.scale[0].cpu().numpy().astype(np.float64), d, B,
                        synth.bf16_bits_to_f64(xb))
    check_gemv(y, y_ref, f"gemm {rows}x{cols} b={batch}")


@pytest.mark.parametrize("rows,cols", [(160, 1024), (2048, 256)])
def test_gemm_far_overflow_points(e8q, rows, cols):
    """kappa 1000 (s = rms / 1000): every group an overflow record, most with
    doubled coordinates beyond fp16's exact integers (+-2048), which the GEMM
    adds on CUDA cores -- in the finalize (K splits, 160 x 1024) and in the
    epilogue (one split, 2048 x 256) -- while the rest go through the tensor
    cores."""
    rng = np.random.default_rng(rows + cols)
    w = synth.f64_to_bf16_bits(rng.standard_normal((rows, cols)) * 0.02)
    d = synth.signs(rows, cols)
    B = oracle.default_block(cols)
    n = rows * cols // 8
    enc, res = run_encode(e8q, [w], [d], 0, kappa=1000.0, esc_cap=n, ovf_cap=n)
    assert res.read_counters()["n_clamped"] == 0
    # the GEMM's reference is the product with the points it was given (at
    # this scale the fp32 projection's near ties are not the fp64 oracle's)
    idx = host_idx(res.idx[0]).reshape(-1)
    P, _, _, _, _ = gpu_points(idx, res.escape_records(), res.overflow_records(), idx.size, 0)
    far_groups = (np.abs(P) > 2048).any(axis=1).sum()
    assert far_groups > 100 and (np.abs(P) <= 2048).all(axis=1).sum() > 100, far_groups
    for batch in (70, 300):
        xb = synth.gemv_x(batch, cols)
        y = run_gemm(e8q, res.encoded[0], xb)
        y_ref = oracle.gemv(P, res.scale[0].cpu().numpy().astype(np.float64), d, B, synth.bf16_bits_to_f64(xb))
        check_gemv(y, y_ref, f"gemm far points {rows}x{cols} b={batch}")


def test_gemm_large_activations_and_repeatable(e8q):
    """Activation rows near the bf16 range limit stay finite (per-row
    power-of-two scaling), and two calls give the same bits."""
    rng = np.random.default_rng(12)
    w = synth.f64_to_bf16_bits(rng.standard_normal((200, 2048)) * 0.02)
    d = synth.signs(4, 2048)
    enc, res = run_encode(e8q, [w], [d], 0)
    st = compare_all(e8q, res, [w], [d], [2048], label="gemm_big_x")[0]
    x = rng.standard_normal((96, 2048))
    x[0] *= 1e30
    x[1] *= 1e-30
    xb = synth.f64_to_bf16_bits(x)
    y = run_gemm(e8q, res.encoded[0], xb)
    y_ref = oracle.gemv(st["points"], res.scale[0].cpu().numpy().astype(np.float64), d, 2048,
                        synth.bf16_bits_to_f64(xb))
    assert np.isfinite(synth.bf16_bits_to_f64(y.view(np.uint16))).all()
    check_gemv(y, y_ref, "gemm big x")
    assert (run_gemm(e8q, res.encoded[0], xb) == y).all()


def test_gemm_equals_gemv_up_to_rounding(e8q):
    """At batch 64 both routes compute the same product; their outputs differ
    by at most the bf16 rounding of each plus the fp16 activation rounding."""
    rng = np.random.default_rng(13)
    w = synth.f64_to_bf16_bits(rng.standard_normal((384, 2048)) * 0.02)
    d = synth.signs(13, 2048)
    enc, res = run_encode(e8q, [w], [d], 0, kappa=2.0)
    xb = synth.gemv_x(64, 2048)
    a = synth.bf16_bits_to_f64(run_gemm(e8q, res.encoded[0], xb).view(np.uint16))
    b = synth.bf16_bits_to_f64(e8q.Gemv(res.encoded[0], 64)(dev_bf16(xb)).cpu().view(torch.int16).numpy().view(np.uint16))
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel < 5e-3, rel


# ----------------------------------------------------------------------
# full-size workloads, in the launch configuration bench.py times
# ----------------------------------------------------------------------
@pytest.fixture(scope="module")
def mlp_full(e8q):
    (up, d_up), (down, d_dn) = synth.mlp_14336()
    G = 4096 * (14336 // 8) + 14336 * (4096 // 8)
    W = [dev_bf16(up), dev_bf16(down)]
    S = [dev(d_up), dev(d_dn)]
    enc = e8q.Encoder([(4096, 14336), (14336, 4096)], S, torch.bfloat16, 0, 1.0, "original", esc_cap=G // 2,
                      ovf_cap=G // 16)
    res = enc(W)
    torch.cuda.synchronize()
    return dict(up=up, down=down, d_up=d_up, d_dn=d_dn, res=res, enc=enc, W=W)


def test_mlp_full_size_sampled_rows(e8q, mlp_full):
    res = mlp_full["res"]
    ctr = res.read_counters()
    assert ctr["err"] == 0 and ctr["n_dropped"] == 0
    rng = np.random.default_rng(123)
    rows = [np.sort(rng.choice(4096, 6, replace=False)), np.sort(rng.choice(14336, 6, replace=False))]
    mats = [mlp_full["up"], mlp_full["down"]]
    signs = [mlp_full["d_up"], mlp_full["d_dn"]]
    stats = compare_all(e8q, res, mats, signs, [2048, 2048], rows=rows, label="mlp")
    for i, st in enumerate(stats):
        dq = res.dequant[i].cpu().view(torch.int16).numpy()[rows[i]]
        check_original_dequant(dq, st["points"], res.scale[i].cpu().numpy()[rows[i]], signs[i], 2048,
                               f"mlp[{i}] original")
    rp = res.esc_row_ptr.cpu().numpy()
    assert rp[0] == 0 and (np.diff(rp) >= 0).all() and rp[-1] == ctr["n_escape"]


def test_mlp_full_matrices_match_oracle(e8q, mlp_full):
    """Every row of both full-size matrices (14.7 M groups) against the
    oracle, run over the host's cores: points, indices, record kinds and
    roots of every group clear of a tie, every near tie a valid E8 point as
    close as the oracle's, scales, and the records' order and fields."""
    res = mlp_full["res"]
    esc, ovf = res.escape_records(), res.overflow_records()
    mats = [(mlp_full["up"], mlp_full["d_up"]), (mlp_full["down"], mlp_full["d_dn"])]
    ties = 0
    for i, (w, d) in enumerate(mats):
        blocks = np.array_split(np.arange(w.shape[0]), 64)
        out = merge_rows(oracle_rows_parallel([(w[b], d, 2048, True) for b in blocks]))
        st = check_encode(out, host_idx(res.idx[i]), res.scale[i].cpu().numpy(), esc, ovf, res.group_base[i],
                          None, w.shape[1] // 8, f"mlp full [{i}]")
        ties += st["near_ties"]
        del out, st
    assert ties < 1e-3 * (4096 * 1792 + 14336 * 512), ties  # about 4e-4 of the groups lie within the margin


def test_moe_bank_every_matrix_matches_oracle(e8q):
    """All 384 expert matrices (75.5 M groups, one launch) against the
    oracle in full: every group clear of a tie identical, scales within
    1e-5."""
    mats = synth.moe_bank()
    W = [m for m, _ in mats]
    S = [s for _, s in mats]
    G = sum(m.shape[0] * (m.shape[1] // 8) for m in W)
    enc, res = run_encode(e8q, W, S, 0, esc_cap=G // 2, ovf_cap=G // 16)
    esc, ovf = res.escape_records(), res.overflow_records()
    idx = [host_idx(t) for t in res.idx]
    scales = [t.cpu().numpy() for t in res.scale]
    del enc
    ties = 0
    jobs = ((W[i], S[i], oracle.default_block(W[i].shape[1]), False) for i in range(len(W)))
    for i, out in enumerate(oracle_rows_stream(jobs)):
        ties += check_encode_far(out, idx[i], scales[i], esc, ovf, res.group_base[i], f"expert matrix {i}")
    assert ties < 0.001 * G, ties


def test_decode_full_size(e8q, mlp_full):
    """Decode of both full-size matrices: the original basis equals the
    encode's own original-basis output bit for bit (same points, scales and
    arithmetic); the rotated basis matches the oracle on sampled rows."""
    res = mlp_full["res"]
    rng = np.random.default_rng(321)
    signs = [mlp_full["d_up"], mlp_full["d_dn"]]
    for i in range(2):
        m = res.encoded[i]
        out = e8q.e8q_decode(m, "original")
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), res.dequant[i].view(torch.int16)), f"matrix {i}: decode != encode dequant"
        rot = e8q.e8q_decode(m, "rotated").cpu().view(torch.int16).numpy()
        rows = np.sort(rng.choice(m.rows, 5, replace=False))
        idx = host_idx(res.idx[i])
        gpr = m.cols // 8
        P_all, _, _, _, _ = gpu_points(idx.reshape(-1), res.escape_records(), res.overflow_records(), idx.size,
                                       res.group_base[i])
        P = P_all.reshape(m.rows, gpr, 8)[rows].reshape(-1, 8)
        check_rotated_dequant(rot[rows], P, res.scale[i].cpu().numpy()[rows], signs[i], 2048, f"decode rotated [{i}]")


@pytest.mark.parametrize("batch", [1, 4, 16, 64])
def test_gemv_full_size(e8q, mlp_full, batch):
    res = mlp_full["res"]
    m = res.encoded[0]
    idx = host_idx(res.idx[0]).reshape(-1)
    P, _, _, _, _ = gpu_points(idx, res.escape_records(), res.overflow_records(), idx.size, 0)
    xb = synth.gemv_x(batch, 14336)
    y = e8q.Gemv(m, batch)(dev_bf16(xb))
    torch.cuda.synchronize()
    y_ref = oracle.gemv(P, res.scale[0].cpu().numpy().astype(np.float64), mlp_full["d_up"], 2048,
                        synth.bf16_bits_to_f64(xb))
    check_gemv(y.cpu().view(torch.int16).numpy(), y_ref, f"gemv full b={batch}")


@pytest.mark.parametrize("batch", [256, 1024])
def test_gemm_full_size(e8q, mlp_full, batch):
    """The fused GEMM on the encoded up matrix at the benchmark's token
    counts, every output against the oracle."""
    res = mlp_full["res"]
    m = res.encoded[0]
    idx = host_idx(res.idx[0]).reshape(-1)
    P, _, _, _, _ = gpu_points(idx, res.escape_records(), res.overflow_records(), idx.size, 0)
    xb = synth.gemv_x(batch, 14336)
    y = run_gemm(e8q, m, xb)
    y_ref = oracle.gemv(P, res.scale[0].cpu().numpy().astype(np.float64), mlp_full["d_up"], 2048,
                        synth.bf16_bits_to_f64(xb))
    check_gemv(y, y_ref, f"gemm full b={batch}")


def test_moe_bank_full_size_sampled(e8q):
    """All 384 expert matrices (604M weights) in one launch; two rows of
    every eighth matrix checked against the oracle."""
    mats = synth.moe_bank()
    W = [m for m, _ in mats]
    S = [s for _, s in mats]
    G = sum(m.shape[0] * (m.shape[1] // 8) for m in W)
    enc, res = run_encode(e8q, W, S, 0, esc_cap=G // 2, ovf_cap=G // 16)
    esc, ovf = res.escape_records(), res.overflow_records()
    rng = np.random.default_rng(7)
    for i in range(0, len(W), 8):
        C = W[i].shape[1]
        rsel = np.sort(rng.choice(W[i].shape[0], 2, replace=False))
        out = oracle.project_encode(synth.bf16_bits_to_f64(W[i][rsel]), S[i], oracle.default_block(C))
        check_encode(out, host_idx(res.idx[i]), res.scale[i].cpu().numpy(), esc, ovf, res.group_base[i], rsel, C // 8,
                     label=f"moe[{i}]")


# ----------------------------------------------------------------------
# core-clipped projection (Figure 2 (a): PTQ from the fixed core)
# ----------------------------------------------------------------------
def run_core(e8q, mats, signs, blocks=0, kappa=1.0, dequant="none", dtype=torch.bfloat16, scales=None):
    ws = [dev_bf16(m) if dtype == torch.bfloat16 else dev(m.astype(np.float32)) for m in mats]
    ss = [dev(s) for s in signs]
    sc = [dev(s.astype(np.float32)) for s in scales] if scales is not None else None
    enc = e8q.Encoder([w.shape for w in ws], ss, dtype, blocks, kappa, dequant, scales is not None, 64, 64,
                      core_only=True)
    res = enc(ws, sc)
    torch.cuda.synchronize()
    ctr = res.read_counters()
    assert ctr["err"] == 0 and ctr["n_escape"] == 0 and ctr["n_overflow"] == 0 and ctr["n_dropped"] == 0, ctr
    assert (res.esc_row_ptr.cpu().numpy() == 0).all() and (res.ovf_row_ptr.cpu().numpy() == 0).all()
    return res


def check_core(out, idx_gpu, label):
    idx = np.asarray(idx_gpu).astype(np.int64).reshape(-1) & 0xFFFF
    far = out["margin"] > MARGIN
    bad = far & (idx != out["idx"])
    assert not bad.any(), f"{label}: {bad.sum()} core indices differ above the margin, e.g. {np.nonzero(bad)[0][:5]}"
    return int((~far).sum())


@pytest.mark.parametrize("kappa", [1.0, 0.5, 3.0])
def test_core_only_f32_matches_oracle(e8q, kappa):
    """f32 256x256 (general kernel), kappa 1 (a quarter of the groups outside
    the core), 0.5 (far outside: the exhaustive fallback) and 3 (almost all
    inside): the nearest core point of every group clear of a tie, and the
    scales of the unclipped projection."""
    w, d = synth.small_f32()
    res = run_core(e8q, [w], [d], 0, kappa, "rotated", torch.float32)
    out = oracle.project_core(w.astype(np.float64), d, 256, kappa)
    check_core(out, host_idx(res.idx[0]), f"core kappa {kappa}")
    np.testing.assert_allclose(res.scale[0].cpu().numpy(), out["scale"], rtol=1e-5)
    core = oracle.core_points().astype(np.int32)
    P = core[host_idx(res.idx[0]).astype(np.int64).reshape(-1)]
    check_rotated_dequant(res.dequant[0].cpu().view(torch.int16).numpy(), P, res.scale[0].cpu().numpy(), d, 256,
                          "core rotated")


def test_core_only_bf16_rows_and_original_basis(e8q):
    """bf16 2048-wide rows (the general kernel takes the core-only calls) with
    the original-basis dequant of the chosen core points."""
    w, d = synth.attn_2048()
    w = w[:96]
    res = run_core(e8q, [w], [d], 0, 1.0, "original")
    out = oracle.project_core(synth.bf16_bits_to_f64(w), d, 2048)
    ties = check_core(out, host_idx(res.idx[0]), "core bf16")
    assert ties < 50
    core = oracle.core_points().astype(np.int32)
    P = core[host_idx(res.idx[0]).astype(np.int64).reshape(-1)]
    check_original_dequant(res.dequant[0].cpu().view(torch.int16).numpy(), P, res.scale[0].cpu().numpy(), d, 2048,
                           "core original")


def test_core_only_fixes_every_core_point(e8q):
    """All 65,536 core points fed exactly (no transform, scale 1) with a
    small perturbation map to themselves: rho = 0 at PTQ init."""
    core = oracle.core_points().astype(np.float64) / 2.0
    rng = np.random.default_rng(19)
    x = (core + rng.uniform(-0.05, 0.05, core.shape)).astype(np.float32).reshape(-1, 64)
    ones = np.ones(64, np.int8)
    res = run_core(e8q, [x], [ones], 1, 1.0, "none", torch.float32, scales=[np.ones(x.shape[0])])
    np.testing.assert_array_equal(host_idx(res.idx[0]).astype(np.int64).reshape(-1), np.arange(65536))


def test_ste_backward_identity_on_mlp_gradient(e8q):
    """Identity STE (Figure 2 (b)): the dense-MLP step's seeded N(0, 1e-3^2)
    bf16 gradients of both matrices reach the latents bit for bit, copied
    (vector path, and an unaligned element path with a ragged tail) or
    aliased (the same tensor, nothing launched)."""
    for i, shape in enumerate([(4096, 14336), (14336, 4096)]):
        g_bits = synth.mlp_grad(shape, matrix=i)
        g = dev_bf16(g_bits)
        out = torch.full_like(g, float("nan"))
        r = e8q.e8q_ste_backward(g, out)
        torch.cuda.synchronize()
        assert r is out
        assert np.array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16), g_bits)
        assert e8q.e8q_ste_backward(g) is g
    g = dev_bf16(synth.mlp_grad((3, 1001), matrix=2))
    buf = torch.full((3 * 1001 + 1,), float("nan"), dtype=torch.bfloat16, device="cuda")
    e8q.e8q_ste_backward(g.reshape(-1), buf[1:])  # 2-byte aligned destination
    flat = g.reshape(-1)[5:]
    dst = torch.empty(flat.numel(), dtype=torch.bfloat16, device="cuda")
    e8q.e8q_ste_backward(flat, dst)  # 2-byte aligned source, 3,998 values
    torch.cuda.synchronize()
    assert torch.equal(buf[1:].view(torch.int16), g.reshape(-1).view(torch.int16))
    assert torch.equal(dst.view(torch.int16), flat.view(torch.int16))
    assert torch.isnan(buf[:1].float()).all()


def _encoded_view(e8q, idx, scale, signs, esc, ovf, erp, orp, cols):
    """An e8q.Encoded over combined (whole-matrix) buffers."""
    return e8q.Encoded(idx, scale, signs, esc, erp, ovf, orp, idx.shape[0], cols, 0, 0,
                       max(1, esc.numel() // 8), max(1, ovf.numel() // 20))


def test_row_shards_encoded_on_gpu_equal_oracle_whole_matrix(e8q):
    """Row-sharded encoding (the multi-GPU path's local step) with the CUDA
    kernels: three uneven row shards of one matrix, each its own encode call
    (group ids from the shard's first row), joined by combine_shards, equal
    the oracle's encoding of the whole matrix (above the tie margin); the
    row-split GEMV (each shard's rows, concatenated) matches the oracle's
    whole-matrix product."""
    from bit_e8_lattice_b200 import dist as e8dist

    rng = np.random.default_rng(18)
    R, C = 300, 2048
    w = synth.f64_to_bf16_bits(rng.standard_normal((R, C)) * 0.02)
    d = synth.signs(18, C)
    x_bits = synth.gemv_x(4, C)
    x = dev_bf16(x_bits)
    parts, ys = [], []
    for a, b in [(0, 77), (77, 150), (150, 300)]:
        _, res = run_encode(e8q, [w[a:b]], [d], 0)
        ctr = res.read_counters()
        parts.append((res.idx[0], res.scale[0], res.esc.clone(), ctr["n_escape"], res.ovf.clone(), ctr["n_overflow"],
                      res.esc_row_ptr.clone(), res.ovf_row_ptr.clone(), a))
        ys.append(e8q.Gemv(res.encoded[0], 4)(x).clone())
    idx, scale, esc, ovf, erp, orp = e8dist.combine_shards(parts, C // 8)
    torch.cuda.synchronize()
    out = oracle.project_encode(synth.bf16_bits_to_f64(w), d, 2048)
    esc_np = np.frombuffer(esc.cpu().numpy().tobytes(), e8q.ESC_DTYPE)
    ovf_np = np.frombuffer(ovf.cpu().numpy().tobytes(), e8q.OVF_DTYPE)
    st = check_encode(out, host_idx(idx), scale.cpu().numpy(), esc_np, ovf_np, 0, None, C // 8, "row shards")
    assert st["rho"] > 0.1
    np.testing.assert_array_equal(erp.cpu().numpy()[-1], len(esc_np))
    # the whole-matrix GEMV from the joined form equals the shards' rows
    m = _encoded_view(e8q, idx, scale, dev(d), esc, ovf, erp, orp, C)
    y_whole = e8q.Gemv(m, 4)(x)
    y_split = torch.cat(ys, dim=1)
    P = st["points"]
    y_ref = oracle.gemv(P, scale.cpu().numpy().astype(np.float64), d, 2048, synth.bf16_bits_to_f64(x_bits))
    check_gemv(y_split.cpu().view(torch.int16).numpy(), y_ref, "row-split GEMV")
    check_gemv(y_whole.cpu().view(torch.int16).numpy(), y_ref, "joined-form GEMV")


def test_gather_encoded_nccl_one_rank(e8q):
    """gather_encoded on CUDA tensors over NCCL (one rank, its two
    collectives included): the gathered encoding of a matrix equals the
    oracle's encoding of it above the tie margin, and its record bytes and
    row pointers equal the encode call's own."""
    import socket
    from datetime import timedelta

    import torch.distributed as dist
    from bit_e8_lattice_b200 import dist as e8dist

    rng = np.random.default_rng(17)
    w = synth.f64_to_bf16_bits(rng.standard_normal((96, 2048)) * 0.02)
    d = synth.signs(17, 2048)
    enc, res = run_encode(e8q, [w], [d], 0)
    ctr = res.read_counters()
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60))
    try:
        out = e8dist.gather_encoded(res.idx[0], res.scale[0], res.esc, ctr["n_escape"], res.ovf, ctr["n_overflow"],
                                    res.esc_row_ptr, res.ovf_row_ptr, 0)
        y = e8dist.gemv_rows_allgather(e8q.Gemv(res.encoded[0], 4)(dev_bf16(synth.gemv_x(4, 2048))))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(out[0], res.idx[0]) and torch.equal(out[1], res.scale[0])
    assert torch.equal(out[2], res.esc[: 8 * ctr["n_escape"]]) and torch.equal(out[3], res.ovf[: 20 * ctr["n_overflow"]])
    assert torch.equal(out[4], res.esc_row_ptr) and torch.equal(out[5], res.ovf_row_ptr)
    ref = oracle.project_encode(synth.bf16_bits_to_f64(w), d, 2048)
    esc_np = np.frombuffer(out[2].cpu().numpy().tobytes(), e8q.ESC_DTYPE)
    ovf_np = np.frombuffer(out[3].cpu().numpy().tobytes(), e8q.OVF_DTYPE)
    st = check_encode(ref, host_idx(out[0]), out[1].cpu().numpy(), esc_np, ovf_np, 0, None, 256, "gathered")
    y_ref = oracle.gemv(st["points"], out[1].cpu().numpy().astype(np.float64), d, 2048,
                        synth.bf16_bits_to_f64(synth.gemv_x(4, 2048)))
    check_gemv(y.cpu().view(torch.int16).numpy(), y_ref, "gathered GEMV")


# ----------------------------------------------------------------------
# shape-gain code (SQuAT page, "shape and scale split")
# ----------------------------------------------------------------------
def run_shape_gain(e8q, mats, signs, blocks=0, kappa=1.0, dequant="none", dtype=torch.bfloat16):
    ws = [dev_bf16(m) if dtype == torch.bfloat16 else dev(m.astype(np.float32)) for m in mats]
    ss = [dev(s) for s in signs]
    enc = e8q.Encoder([w.shape for w in ws], ss, dtype, blocks, kappa, dequant, False, 64, 64, shape_gain=True)
    res = enc(ws)
    torch.cuda.synchronize()
    ctr = res.read_counters()
    assert ctr["err"] == 0 and ctr["n_escape"] == 0 and ctr["n_overflow"] == 0 and ctr["n_dropped"] == 0, ctr
    assert (res.esc_row_ptr.cpu().numpy() == 0).all() and (res.ovf_row_ptr.cpu().numpy() == 0).all()
    return res


def check_shape_gain(out, code_gpu, label):
    """Directions equal wherever the best shell point leads the second by
    more than the tie margin; gain levels equal wherever |x| / (6/16) is not
    within 1e-4 of a level boundary.  Returns the near-tie count."""
    code = np.asarray(code_gpu).astype(np.int64).reshape(-1) & 0xFFFF
    far = out["margin"] > MARGIN
    bad = far & ((code & 0xFFF) != out["dir"])
    assert not bad.any(), f"{label}: {bad.sum()} directions differ above the margin, e.g. {np.nonzero(bad)[0][:5]}"
    assert ((code & 0xFFF) < 2160).all()
    n = np.sqrt((out["x"].reshape(-1, 8) ** 2).sum(1)) / oracle.SG_STEP
    clear = np.abs(n - np.rint(n)) > 1e-4
    bad = clear & ((code >> 12) != out["level"])
    assert not bad.any(), f"{label}: {bad.sum()} gain levels differ away from a boundary"
    return int((~far).sum())


@pytest.mark.parametrize("kappa", [1.0, 3.0])
def test_shape_gain_f32_matches_oracle(e8q, kappa):
    """f32 256x256 (block 256): every direction clear of a tie and every
    gain level clear of a boundary as the oracle's; kappa 3 puts many gains
    past the grid (level 15); rotated dequant of the chosen codes exact."""
    w, d = synth.small_f32()
    res = run_shape_gain(e8q, [w], [d], 0, kappa, "rotated", torch.float32)
    out = oracle.sg_project_encode(w.astype(np.float64), d, 256, kappa)
    ties = check_shape_gain(out, host_idx(res.idx[0]), f"shape-gain kappa {kappa}")
    assert ties < 50
    np.testing.assert_allclose(res.scale[0].cpu().numpy(), out["scale"], rtol=1e-5)
    if kappa > 2:
        assert ((host_idx(res.idx[0]).astype(np.int64) & 0xFFFF) >> 12 == 15).mean() > 0.2
    s32 = res.scale[0].cpu().numpy().astype(np.float64)
    xh = oracle.sg_points(host_idx(res.idx[0]).astype(np.int64).reshape(-1) & 0xFFFF)
    bits, _ = oracle.sg_dequant(xh, s32, d, 256, "rotated")
    got = res.dequant[0].cpu().view(torch.int16).numpy().view(np.uint16)
    assert (got == bits).all()


@pytest.mark.parametrize("rows,cols", [(96, 2048), (37, 264), (5, 16384)])
def test_shape_gain_bf16_original_basis(e8q, rows, cols):
    """bf16 rows of several widths and RHT blocks (2048, 8, 2048), original-
    basis dequant of the chosen codes within one bf16 ulp of the fp64
    inverse transform."""
    rng = np.random.default_rng(rows + cols)
    w = synth.f64_to_bf16_bits(rng.standard_normal((rows, cols)) * 0.015)
    d = synth.signs(rows, cols)
    B = oracle.default_block(cols)
    res = run_shape_gain(e8q, [w], [d], 0, 1.0, "original")
    out = oracle.sg_project_encode(synth.bf16_bits_to_f64(w), d, B)
    check_shape_gain(out, host_idx(res.idx[0]), f"shape-gain {rows}x{cols}")
    s = res.scale[0].cpu().numpy().astype(np.float64)
    xh = oracle.sg_points(host_idx(res.idx[0]).astype(np.int64).reshape(-1) & 0xFFFF)
    _, f64 = oracle.sg_dequant(xh, s, d, B, "original")
    got = synth.bf16_bits_to_f64(res.dequant[0].cpu().view(torch.int16).numpy().view(np.uint16)).reshape(f64.shape)
    ulp = np.where(f64 != 0, 2.0 ** (np.floor(np.log2(np.abs(f64) + 1e-300)) - 7), 0.0)
    bad = np.abs(got - f64) > ulp + 2.0 ** -20 * s[:, None]
    assert not bad.any(), f"{bad.sum()} original-basis values off by more than 1 ulp"


def test_shape_gain_shell_points_are_fixed(e8q):
    """Rows made of shell points (doubled / 2, times a per-row factor) map to
    themselves: direction = the point's own index, for all 2160 points."""
    S = oracle.sg_shell().astype(np.float64)
    rows = (S / 2.0).reshape(270, 64)  # 8 points a row, rows of 64
    w = rows * np.linspace(0.5, 2.0, 270)[:, None]
    d = np.ones(64, np.int8)
    res = run_shape_gain(e8q, [w.astype(np.float32)], [d], 1, 1.0, "none", torch.float32)
    code = host_idx(res.idx[0]).astype(np.int64).reshape(-1) & 0xFFFF
    assert ((code & 0xFFF) == np.arange(2160)).all()


def test_shape_gain_flag_rules(e8q):
    """The two flags together are rejected."""
    w, d = synth.small_f32()
    with pytest.raises(e8q.E8qError):
        e8q.Encoder([w.shape], [dev(d)], torch.float32, 0, 1.0, "none", False, 64, 64, core_only=True,
                    shape_gain=True)([dev(w)])
