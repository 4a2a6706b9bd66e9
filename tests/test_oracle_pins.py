"""Pins for the CPU oracle: each check ties it to something other than itself
(closed forms, brute force, library routines, numbers printed on the pages).

Page cited throughout: "E8-QAT: Efficient 2-Bit Quantization-Aware Training
with Implicit Lattice Codebooks" (abstract; Figure 2 caption; appendix
Tables 3, 4, 9, 10).
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.linalg

from bit_e8_lattice_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------
# independent helpers (numpy; none of the oracle's code)
# ----------------------------------------------------------------------
def np_e8_points(max_n2=48):
    """All doubled E8 points of |P|^2 <= max_n2 by direct numpy filtering."""
    pts = []
    for vals in (np.arange(-6, 7, 2), np.arange(-5, 6, 2)):
        grid = np.array(list(itertools.product(vals, repeat=4)), np.int32)  # half the coordinates
        n2h = (grid * grid).sum(1)
        sh = grid.sum(1)
        ok = n2h <= max_n2
        grid, n2h, sh = grid[ok], n2h[ok], sh[ok]
        for i in range(len(grid)):
            rem = max_n2 - n2h[i]
            sel = (n2h <= rem) & (((sh[i] + sh) % 4) == 0)
            if sel.any():
                pts.append(np.concatenate([np.repeat(grid[i:i + 1], sel.sum(), 0), grid[sel]], 1))
    P = np.concatenate(pts, 0)
    n2 = (P * P).sum(1)
    order = np.lexsort(tuple(P[:, k] for k in range(7, -1, -1)) + (n2,))
    return P[order], n2[order]


def sigma3(m):
    return sum(d ** 3 for d in range(1, m + 1) if m % d == 0)


def brute_nearest(x, width=1):
    """Nearest E8 point by exhaustive search of a box around x (doubled
    output), plus the sorted squared distances of the candidates."""
    off = np.array(list(itertools.product(range(-width, width + 1), repeat=8)), np.float64)
    out, d1, d2 = [], [], []
    for v in x:
        cands = []
        base_i = np.round(v)
        ci = base_i + off
        ci = ci[(ci.sum(1) % 2) == 0]
        base_h = np.floor(v) + 0.5
        ch = base_h + off
        ch = ch[(np.round(ch.sum(1)) % 2) == 0]
        c = np.concatenate([ci, ch], 0)
        dist = ((c - v) ** 2).sum(1)
        order = np.argsort(dist, kind="stable")
        out.append(np.round(2 * c[order[0]]).astype(np.int32))
        d1.append(dist[order[0]])
        d2.append(dist[order[1]])
    return np.array(out), np.array(d1), np.array(d2)


def bf16_value(bits):
    return synth.bf16_bits_to_f64(np.asarray(bits, np.uint16))


def bf16_neighbours_ok(v, bits):
    """bits must be the bf16 nearest to v, ties to an even significand."""
    r = float(bf16_value(np.array([bits]))[0])
    b = int(bits)
    up = float(bf16_value(np.array([(b + 1) & 0xFFFF]))[0]) if (b & 0x7FFF) != 0x7F7F else math.inf
    dn = float(bf16_value(np.array([(b - 1) & 0xFFFF]))[0]) if (b & 0x7FFF) != 0 else -r
    err = abs(v - r)
    if err > abs(v - up) or err > abs(v - dn):
        return False
    if err == abs(v - up) or err == abs(v - dn):  # a tie must land on even
        return (b & 1) == 0
    return True


# ----------------------------------------------------------------------
# lattice enumeration, core and roots (Table 3: 65,536 core codewords)
# ----------------------------------------------------------------------
def test_shell_counts_match_theta_series(orc):
    _, n2 = orc.all_points()
    norms = n2 // 4  # |p|^2
    assert (n2 % 4 == 0).all()
    counts = {int(k): int(v) for k, v in zip(*np.unique(norms, return_counts=True))}
    assert counts[0] == 1
    for m in range(1, 7):  # theta_E8 = 1 + 240 sum sigma_3(m) q^(2m)
        assert counts[2 * m] == 240 * sigma3(m), m
    assert set(counts) == {0, 2, 4, 6, 8, 10, 12}


def test_enumeration_and_order_match_numpy(orc):
    c, n2 = orc.all_points()
    P, pn2 = np_e8_points()
    assert c.shape == P.shape
    np.testing.assert_array_equal(c.astype(np.int32), P)
    np.testing.assert_array_equal(n2, pn2)


def test_core_size_and_composition(orc):
    core = orc.core_points().astype(np.int32)
    assert core.shape == (65536, 8)  # Table 3
    n2 = (core * core).sum(1)
    assert (n2 <= 48).all()
    assert (n2 <= 40).sum() == 1 + 240 * sum(sigma3(m) for m in range(1, 6))  # 56,881
    assert (n2 == 48).sum() == 65536 - 56881
    # the norm-12 members are the lexicographically smallest of their shell
    P, pn2 = np_e8_points()
    shell = P[pn2 == 48]
    np.testing.assert_array_equal(core[n2 == 48], shell[: 65536 - 56881])
    assert len({tuple(r) for r in core}) == 65536


def test_roots_structure(orc):
    r = orc.roots().astype(np.int32)
    assert r.shape == (240, 8)
    assert ((r * r).sum(1) == 8).all()
    integer = (r % 2 == 0).all(1)
    assert integer.sum() == 112 and (~integer).sum() == 128
    assert ((np.abs(r[integer]) == 2).sum(1) == 2).all()
    assert ((np.abs(r[~integer]) == 1).all(1)).all()
    assert ((r[~integer] < 0).sum(1) % 2 == 0).all()
    order = np.lexsort(tuple(r[:, k] for k in range(7, -1, -1)))
    np.testing.assert_array_equal(order, np.arange(240))
    core = orc.core_points().astype(np.int32)
    np.testing.assert_array_equal(core[1:241], r)  # root k is core index k + 1
    np.testing.assert_array_equal(core[0], np.zeros(8))


def test_rank_is_position(orc):
    core = orc.core_points().astype(np.int32)
    rng = np.random.default_rng(11)
    for k in rng.choice(65536, 300, replace=False):
        assert orc.rank(core[k]) == k
    assert orc.rank([1, 0, 0, 0, 0, 0, 0, 0]) == -1  # mixed parity
    assert orc.rank([2, 0, 0, 0, 0, 0, 0, 0]) == -1  # sum not divisible by 4
    assert orc.rank([8, 0, 0, 0, 0, 0, 0, 0]) == -1  # beyond |p|^2 = 12


# ----------------------------------------------------------------------
# projection (abstract: arithmetic projection onto E8)
# ----------------------------------------------------------------------
def test_projection_matches_brute_force_on_free_vectors(orc):
    x = synth.free_vectors().astype(np.float64)
    out = orc.project_encode_vectors(x)
    bp, d1, d2 = brute_nearest(x, width=1)
    near_tie = (d2 - d1) <= 1e-9
    assert near_tie.sum() == 0
    np.testing.assert_array_equal(out["P"], bp)


def test_margin_matches_brute_second_nearest(orc):
    x = synth.free_vectors(seed=7, n=24).astype(np.float64)
    out = orc.project_encode_vectors(x)
    bp, d1, d2 = brute_nearest(x, width=2)
    np.testing.assert_array_equal(out["P"], bp)
    np.testing.assert_allclose(out["margin"], d2 - d1, atol=1e-9)


def test_projection_fixes_lattice_points_and_small_noise(orc):
    c, _ = orc.all_points()
    rng = np.random.default_rng(3)
    P = c[rng.choice(len(c), 2000)].astype(np.int32)
    out = orc.project_encode_vectors(P / 2.0)
    np.testing.assert_array_equal(out["P"], P)
    noise = rng.standard_normal(P.shape)
    noise *= (0.6 * rng.random((len(P), 1))) / np.linalg.norm(noise, axis=1, keepdims=True)  # |n| < 1/sqrt(2)
    out = orc.project_encode_vectors(P / 2.0 + noise)
    np.testing.assert_array_equal(out["P"], P)
    # membership of every output
    Q = out["P"]
    par = Q[:, :1] & 1
    assert ((Q & 1) == par).all() and (Q.sum(1) % 4 == 0).all()


def test_projection_hand_cases(orc):
    # D8 half: round (0.6,0.2,0..) -> (1,0,..) has odd sum; the worst-rounded
    # coordinate (0.6 -> 1, error 0.4) moves back to 0; the D8+1/2 candidate
    # D8+1/2 answer (.5,.5,...,.5) is at distance 1.6.
    x = np.array([[0.6, 0.2, 0, 0, 0, 0, 0, 0]])
    assert orc.project_encode_vectors(x)["P"].tolist() == [[0] * 8]
    # all coordinates 0.45: D8 gives 0 (distance 1.62); D8+1/2 gives all 0.5
    # (sum 4, even; distance 0.02).
    x = np.full((1, 8), 0.45)
    assert orc.project_encode_vectors(x)["P"].tolist() == [[1] * 8]
    # (0.9, 0.9, 0, ...): rounds to (1,1,0,...), sum even, distance 0.02.
    x = np.array([[0.9, 0.9, 0, 0, 0, 0, 0, 0]])
    assert orc.project_encode_vectors(x)["P"].tolist() == [[2, 2, 0, 0, 0, 0, 0, 0]]
    # (1.2, 0, ..., 0): rounds to (1,0,...), odd sum; the only nonzero error
    # is on coordinate 0, which moves towards x: (2,0,...,0), distance 0.64.
    # The D8+1/2 side ends at (1.5,-.5,.5,...,.5), distance 1.84; the next
    # D8 points (0,...) and (1,+-1,0,...) are at 1.44 and 1.04.
    x = np.array([[1.2, 0, 0, 0, 0, 0, 0, 0]])
    assert orc.project_encode_vectors(x)["P"].tolist() == [[4, 0, 0, 0, 0, 0, 0, 0]]


def test_projection_tie_conventions(orc):
    # Parity-fix tie: (0.6, 0.6, 1, 0, ...) rounds to (1,1,1,0,...), odd sum,
    # and coordinates 0 and 1 share the largest error 0.4.  The lowest index
    # moves: (0,1,1,0,...) at distance 0.52 (the D8+1/2 side is at 1.52).
    x = np.array([[0.6, 0.6, 1, 0, 0, 0, 0, 0]])
    assert orc.project_encode_vectors(x)["P"].tolist() == [[0, 2, 2, 0, 0, 0, 0, 0]]
    # Coset tie: (1/4, ..., 1/4) is at distance 0.5 from both 0 (D8) and
    # (1/2, ..., 1/2) (D8+1/2); the tie keeps the D8 point.
    x = np.full((1, 8), 0.25)
    out = orc.project_encode_vectors(x)
    assert out["P"].tolist() == [[0] * 8]
    assert abs(out["margin"][0]) < 1e-12


def test_tie_has_zero_margin(orc):
    # midpoint of 0 and the root (1,1,0,...): both at distance 0.5
    x = np.array([[0.5, 0.5, 0, 0, 0, 0, 0, 0]])
    out = orc.project_encode_vectors(x)
    assert abs(out["margin"][0]) < 1e-12


# ----------------------------------------------------------------------
# encoding (abstract, Figure 2 (c), Table 3)
# ----------------------------------------------------------------------
def test_core_points_encode_to_themselves(orc):
    """Table 9: points initialised in the core give no escapes (rho = 0)."""
    core = orc.core_points().astype(np.int32)
    out = orc.project_encode_vectors(core / 2.0)
    np.testing.assert_array_equal(out["P"], core)
    assert (out["kind"] == 0).all()
    np.testing.assert_array_equal(out["idx"], np.arange(65536))


def _roundtrip_and_rule_checks(orc, out):
    core = orc.core_points().astype(np.int32)
    rt = orc.roots().astype(np.int32)
    P, kind, idx, root = out["P"], out["kind"], out["idx"], out["root"]
    esc, ovf_g, ovf_P = orc.records(out)
    Q = orc.assemble_points(idx, esc[:, 0], esc[:, 2], ovf_g, ovf_P, len(P))
    np.testing.assert_array_equal(Q, P)  # decode(encode(p)) == p
    e = kind == 1
    # Table 3: every escape residual is one root
    np.testing.assert_array_equal(P[e] - core[idx[e]], rt[root[e]])
    # the chosen core point is the (norm, lex)-smallest of all P - r: the
    # smallest core index among the valid ones
    for g in np.nonzero(kind > 0)[0][:400]:
        cand = P[g] - rt
        n2 = (cand * cand).sum(1)
        order = np.lexsort(tuple(cand[:, k] for k in range(7, -1, -1)) + (n2,))
        best = cand[order[0]]
        if kind[g] == 1:
            np.testing.assert_array_equal(core[idx[g]], best)
        else:
            assert orc.rank(best) < 0 or orc.rank(best) >= 65536
    return e.mean(), (kind == 2).mean()


def test_encode_roundtrip_small_f32(orc):
    w, d = synth.small_f32()
    out = orc.project_encode(w.astype(np.float64), d, orc.default_block(256))
    rho, ovf = _roundtrip_and_rule_checks(orc, out)
    assert 0.1 < rho < 0.4 and 0 < ovf < 0.05


def test_encode_roundtrip_free_vectors(orc):
    x = synth.free_vectors().astype(np.float64)
    out = orc.project_encode_vectors(x)
    rho, ovf = _roundtrip_and_rule_checks(orc, out)
    assert ovf > 0  # 3*N(0, I) reaches far past the core


# ----------------------------------------------------------------------
# randomized Hadamard transform and scales (Figure 2)
# ----------------------------------------------------------------------
@pytest.mark.parametrize("n", [1, 2, 4, 8, 64, 256, 1024])
def test_fwht_and_dense_match_scipy_hadamard(orc, n):
    rng = np.random.default_rng(n)
    u = rng.standard_normal(n)
    H = scipy.linalg.hadamard(n).astype(np.float64)  # Sylvester construction
    np.testing.assert_allclose(orc.fwht(u), H @ u, rtol=1e-12, atol=1e-12)
    if n <= 256:
        np.testing.assert_allclose(orc.hadamard_dense(u), H @ u, rtol=1e-12, atol=1e-12)


def test_hadamard_involution_and_norm(orc):
    rng = np.random.default_rng(5)
    u = rng.standard_normal(2048)
    v = orc.fwht(u) / math.sqrt(2048)
    np.testing.assert_allclose(np.linalg.norm(v), np.linalg.norm(u), rtol=1e-12)
    np.testing.assert_allclose(orc.fwht(v) / math.sqrt(2048), u, atol=1e-12)  # H^2 = B I


def test_scale_is_rms_of_raw_row_and_x_matches_scipy(orc):
    w, d = synth.small_f32()
    w = w.astype(np.float64)
    out = orc.project_encode(w, d, 256)
    np.testing.assert_allclose(out["scale"], np.sqrt((w * w).mean(1)), rtol=1e-12)
    H = scipy.linalg.hadamard(256) / 16.0
    v = (w * d) @ H.T
    np.testing.assert_allclose(out["x"], v / out["scale"][:, None], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose((out["x"] ** 2).mean(1), 1.0, rtol=1e-12)
    out2 = orc.project_encode(w, d, 256, kappa=2.0)
    np.testing.assert_allclose(out2["scale"], out["scale"] / 2, rtol=1e-15)


def test_blockwise_rht_three_blocks(orc):
    rng = np.random.default_rng(9)
    w = rng.standard_normal((3, 768))
    d = synth.signs(9, 768)
    out = orc.project_encode(w, d, 256)
    H = scipy.linalg.hadamard(256) / 16.0
    v = np.concatenate([(w[:, k * 256:(k + 1) * 256] * d[k * 256:(k + 1) * 256]) @ H.T for k in range(3)], 1)
    np.testing.assert_allclose(out["x"], v / out["scale"][:, None], rtol=1e-10, atol=1e-12)


def test_nonfinite_and_zero_rows(orc):
    w = np.zeros((3, 16))
    w[1] = np.linspace(-1, 1, 16)
    w[1, 3] = np.nan
    w[2, 5] = np.inf
    d = np.ones(16, np.int8)
    out = orc.project_encode(w, d, 16)
    assert out["nonfinite"] == 2
    assert out["scale"][0] == 0.0 and (out["idx"][:2] == 0).all() and (out["kind"][:2] == 0).all()
    assert np.isfinite(out["scale"]).all()


def test_default_block_rule(orc):
    assert orc.default_block(256) == 256
    assert orc.default_block(768) == 256
    assert orc.default_block(2048) == 2048
    assert orc.default_block(14336) == 2048
    assert orc.default_block(4096) == 2048
    assert orc.default_block(24) == 8


# ----------------------------------------------------------------------
# dequantisation (abstract: lattice points kept exactly; bf16 latents)
# ----------------------------------------------------------------------
def test_bf16_rounding_matches_torch_on_f32_values(orc):
    import torch

    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000),
                        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0, -0.0, 2.0 ** -130]])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.bf16_bits(float(t)) for t in v32], np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_bf16_rounding_is_single_rounding_from_double(orc):
    rng = np.random.default_rng(2)
    # values with more significant bits than f32 near bf16 midpoints
    base = rng.integers(128, 256, 500).astype(np.float64)
    v = (base + 0.5 + rng.choice([-1, 1], 500) * 2.0 ** -30) * 2.0 ** rng.integers(-20, 20, 500)
    for t in v:
        assert bf16_neighbours_ok(t, orc.bf16_bits(t)), t


def test_dequant_rotated_is_nearest_bf16_of_exact_product(orc):
    w, d = synth.small_f32()
    out = orc.project_encode(w.astype(np.float64), d, 256)
    s32 = out["scale"].astype(np.float32).astype(np.float64)
    bits, _ = orc.dequant(out["P"], s32, d, 256, "rotated")
    exact = s32[:, None] * (out["P"].reshape(256, 256) / 2.0)
    flat_b, flat_v = bits.reshape(-1), exact.reshape(-1)
    for k in np.random.default_rng(0).choice(flat_b.size, 3000, replace=False):
        assert bf16_neighbours_ok(flat_v[k], flat_b[k])


def test_dequant_original_inverts_rotation(orc):
    w, d = synth.small_f32()
    out = orc.project_encode(w.astype(np.float64), d, 256)
    s = out["scale"]
    _, f64 = orc.dequant(out["P"], s, d, 256, "original")
    H = scipy.linalg.hadamard(256) / 16.0
    rot = s[:, None] * out["P"].reshape(256, 256) / 2.0
    np.testing.assert_allclose(f64, (rot @ H.T) * d, rtol=1e-10, atol=1e-14)


def test_gemv_two_routes_agree(orc):
    w, d = synth.small_f32()
    out = orc.project_encode(w.astype(np.float64), d, 256)
    x = synth.bf16_bits_to_f64(synth.gemv_x(4, 256))
    y = orc.gemv(out["P"], out["scale"], d, 256, x)
    H = scipy.linalg.hadamard(256) / 16.0
    xrot = (x * d) @ H.T
    y2 = (out["scale"][None, :] / 2.0) * (xrot @ out["P"].reshape(256, 256).T)
    np.testing.assert_allclose(y, y2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(orc.rht_vectors(x, d, 256), xrot, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------
# payload accounting (Tables 3, 4, 9, 10)
# ----------------------------------------------------------------------
def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_payload_formula_reproduces_table10(orc):
    for r in _golden_rows("table10_payload.txt"):
        rho, db, b = float(r[-3]), float(r[-2]), float(r[-1])
        assert abs(orc.payload_bits_pages(rho) - 2.0 - db) <= 0.5e-3 * db
        assert round(orc.payload_bits_pages(rho), 6) == b
        # 20-byte records: delta_b = 20 * rho
        assert abs(orc.payload_bits_actual(10 ** 9, 0, round(rho * 10 ** 9), ovf_bytes=20) - b) < 1e-6


def test_escape_fraction_counts_groups(orc):
    kv = {r[0]: float(r[1]) for r in _golden_rows("table3_escape_count.txt")}
    rho = kv["escaped_groups"] / (kv["quantized_params"] / kv["group_size"])
    assert round(rho, 9) == kv["rho_step375"]
    assert kv["core_codewords"] == len(orc.core_points())


# ----------------------------------------------------------------------
# Core-clipped projection (E8-QAT Figure 2 (a): PTQ from the fixed core)
# ----------------------------------------------------------------------
def _independent_core():
    """The 65,536 first points in (norm, lex) order, enumerated by numpy
    (not the oracle's table), as undoubled coordinates."""
    P, _ = np_e8_points(48)
    return P[:65536].astype(np.float64) / 2.0


def test_nearest_core_matches_kdtree_search(orc):
    """A KD-tree nearest-neighbour query over an independently enumerated core
    gives the oracle's nearest core point on every vector clear of a tie;
    vectors span the core's inside, its boundary and far outside it."""
    from scipy.spatial import cKDTree

    core = _independent_core()
    tree = cKDTree(core)
    rng = np.random.default_rng(77)
    x = np.concatenate([rng.standard_normal((600, 8)) * s for s in (0.7, 1.2, 1.8, 3.0)])
    out = orc.nearest_core_vectors(x)
    dist, k = tree.query(x)
    clear = out["margin"] > 1e-9
    assert clear.mean() > 0.99
    np.testing.assert_array_equal(out["idx"][clear], k[clear])
    np.testing.assert_allclose(((x - out["P"] / 2.0) ** 2).sum(1), dist ** 2, rtol=1e-12, atol=1e-12)


def test_nearest_core_fixes_core_points_and_agrees_inside(orc):
    """Every core point maps to itself (rho = 0 at PTQ init, Table 9, step
    100); a vector whose nearest E8 point is in the core gets that point."""
    core = orc.core_points().astype(np.float64) / 2.0
    sel = np.arange(0, 65536, 97)
    out = orc.nearest_core_vectors(core[sel] + 1e-3)
    np.testing.assert_array_equal(out["idx"], sel)
    rng = np.random.default_rng(78)
    x = rng.standard_normal((800, 8)) * 1.1
    free = orc.project_encode_vectors(x)
    inside = (free["kind"] == 0) & (free["margin"] > 1e-9)
    assert inside.mean() > 0.5
    out = orc.nearest_core_vectors(x[inside])
    np.testing.assert_array_equal(out["idx"], free["idx"][inside])


def test_nearest_core_of_far_vectors_lies_on_the_boundary(orc):
    """Far outside the core the nearest core point has |p|^2 >= 10 (the core
    holds the whole ball |p|^2 <= 10 and part of the next shell) and points
    the way of x."""
    rng = np.random.default_rng(79)
    x = rng.standard_normal((300, 8))
    x = x / np.linalg.norm(x, axis=1, keepdims=True) * 6.0
    out = orc.nearest_core_vectors(x)
    p = out["P"] / 2.0
    assert ((p ** 2).sum(1) >= 10 - 1e-9).all()
    cos = (p * x).sum(1) / (np.linalg.norm(p, axis=1) * 6.0)
    assert (cos > 0.8).all()


def test_project_core_rows_scale_and_no_records(orc):
    """The row pipeline with the core-clipped projection: the same scales as
    the unclipped pipeline, every group a core point, each as close as any
    core point can be (checked against the KD-tree on the oracle's x)."""
    from scipy.spatial import cKDTree

    w, d = synth.small_f32(rows=24)
    full = orc.project_encode(w.astype(np.float64), d, 256)
    core = orc.project_core(w.astype(np.float64), d, 256)
    np.testing.assert_array_equal(core["scale"], full["scale"])
    tree = cKDTree(_independent_core())
    dist, k = tree.query(full["x"].reshape(-1, 8))
    clear = core["margin"] > 1e-9
    np.testing.assert_array_equal(core["idx"][clear], k[clear])
    kept = full["kind"] == 0
    np.testing.assert_array_equal(core["idx"][kept & clear], full["idx"][kept & clear])


# ----------------------------------------------------------------------
# shape-gain variant (SQuAT page, "shape and scale split")
# ----------------------------------------------------------------------
def structured_direction(x):
    """Best |p|^2 = 4 shell point for one vector by the shell's three
    families (doubled coordinates): +-4 e_i; +-2 on four coordinates; odd
    coordinates with one +-3 and a coordinate sum divisible by 4.  Written
    from the shell's structure, independent of the oracle's scoring."""
    ax = np.abs(x)
    sg = np.where(x < 0, -1, 1)
    best = []
    i = int(np.argmax(ax))
    P = np.zeros(8, np.int64)
    P[i] = 4 * sg[i]
    best.append(P)
    top = np.argsort(-ax, kind="stable")[:4]
    P = np.zeros(8, np.int64)
    P[top] = 2 * sg[top]
    best.append(P)
    for j in range(8):  # position of the +-3
        for flip in range(-1, 8):  # no flip, or the coordinate whose sign is reversed
            P = sg.astype(np.int64).copy()
            P[j] *= 3
            if flip >= 0:
                P[flip] = -P[flip]
            if P.sum() % 4 == 0:
                best.append(P)
    scores = [float(x @ P) for P in best]
    return best[int(np.argmax(scores))], max(scores)


def test_sg_shell_is_the_norm4_shell(orc):
    S = orc.sg_shell()
    P, n2 = np_e8_points(16)
    ref = P[n2 == 16]
    assert S.shape == (2160, 8) and (S == ref).all()
    assert orc.rank(S[0]) == orc.SG_SHELL_FIRST and orc.rank(S[-1]) == orc.SG_SHELL_FIRST + 2159
    # the shell's families: 16 of type +-4 e_i, 1120 of type (+-2)^4, 1024 odd
    a = np.abs(S)
    assert ((a == 4).sum(1) == 1).sum() == 16
    assert ((a == 2).sum(1) == 4).sum() == 1120
    assert ((a % 2 == 1).all(1)).sum() == 1024


def test_sg_direction_matches_structured_search(orc):
    rng = np.random.default_rng(77)
    x = rng.standard_normal((3000, 8)) * rng.uniform(0.2, 4.0, (3000, 1))
    code, d, k, margin = orc.sg_encode_vectors(x)
    S = orc.sg_shell()
    checked = 0
    for i in range(len(x)):
        P, sc = structured_direction(x[i])
        assert abs(sc - float(x[i] @ S[d[i]])) <= 1e-9 * (1 + abs(sc))
        if margin[i] > 1e-9:
            assert (P == S[d[i]]).all()
            checked += 1
    assert checked > 2900


def test_sg_direction_fixed_points_symmetry_and_scale(orc):
    S = orc.sg_shell()
    code, d, k, m = orc.sg_encode_vectors(S / 2.0)
    assert (d == np.arange(2160)).all() and (k == 5).all()  # |p| = 2 -> floor(2 / 0.375) = 5
    rng = np.random.default_rng(5)
    x = rng.standard_normal((500, 8))
    _, d1, _, m1 = orc.sg_encode_vectors(x)
    _, d2, _, _ = orc.sg_encode_vectors(3.7 * x)
    _, d3, _, _ = orc.sg_encode_vectors(-x)
    ok = m1 > 1e-9
    assert (d1[ok] == d2[ok]).all()
    # -x picks -P
    assert (S[d3[ok]] == -S[d1[ok]]).all()


def test_sg_gain_levels_and_reconstruction(orc):
    D = orc.SG_STEP
    assert D == 0.375 and orc.SG_LEVELS == 16
    u = np.zeros((20, 8))
    u[:, 0] = 1.0
    g = np.array([0.0, 0.1, 0.374, 0.376, 1.0, 2.9, 5.99, 6.0, 7.5, 100.0] + [0.375 * j + 0.1 for j in range(10)])
    code, d, k, _ = orc.sg_encode_vectors(u * g[:, None])
    want = np.minimum(15, np.floor(g / D)).astype(np.int64)
    assert (k == want).all() and ((code >> 12) == want).all()
    xh = orc.sg_points(code)
    assert np.allclose(np.sqrt((xh * xh).sum(1)), (want + 0.5) * D)  # |P| / 4 = 1
    # the direction of x-hat is the chosen shell point
    S = orc.sg_shell().astype(np.float64)
    assert np.allclose(xh, ((want + 0.5) * D)[:, None] * S[code & 0xFFF] / 4)


def test_sg_dequant_bases(orc):
    rng = np.random.default_rng(9)
    R, C, B = 3, 64, 16
    w = rng.standard_normal((R, C)) * 0.02
    d = np.where(rng.random(C) < 0.5, -1, 1).astype(np.int8)
    out = orc.sg_project_encode(w, d, B)
    s32 = out["scale"].astype(np.float32).astype(np.float64)
    rot_bits, rot = orc.sg_dequant(out["xhat"], s32, d, B, "rotated")
    assert np.array_equal(rot, s32[:, None] * out["xhat"].reshape(R, C))
    assert all(bf16_neighbours_ok(v, b) for v, b in zip(rot.ravel(), rot_bits.ravel()))
    orig_bits, orig = orc.sg_dequant(out["xhat"], s32, d, B, "original")
    H = scipy.linalg.hadamard(B) / math.sqrt(B)
    ref = (s32[:, None] * out["xhat"].reshape(R, C)).reshape(R, C // B, B) @ H.T
    assert np.allclose(orig, ref.reshape(R, C) * d[None, :], rtol=0, atol=1e-15)
    assert all(bf16_neighbours_ok(v, b) for v, b in zip(orig.ravel(), orig_bits.ravel()))
    # the round trip: rotating the original-basis reconstruction back gives s * x-hat
    back = orc.rht_vectors(orig, d, B)
    assert np.allclose(back, s32[:, None] * out["xhat"].reshape(R, C), atol=1e-15)
