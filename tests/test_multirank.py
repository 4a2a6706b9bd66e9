"""Two gloo ranks on CPU: row shards encode exactly like the whole matrix,
and the timing reduction takes the maximum over ranks."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    from datetime import timedelta

    import oracle
    from bit_e8_lattice_b200 import dist as e8dist
    from bit_e8_lattice_b200 import synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, d = synth.small_f32()
        a, b = e8dist.shard_rows(w.shape[0], world, rank)
        out = oracle.project_encode(w[a:b].astype(np.float64), d, 256, want_x=False, want_margin=False)
        shards = [None] * world
        dist.all_gather_object(shards, (a, b, out["idx"], out["kind"], out["root"], out["P"], out["scale"]))
        mx = e8dist.max_over_ranks(10.0 + rank)
        q.put((rank, shards, mx))
    finally:
        dist.destroy_process_group()


def test_row_shards_reproduce_whole_matrix_and_max_reduction():
    import oracle
    from bit_e8_lattice_b200 import synth

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, d = synth.small_f32()
    full = oracle.project_encode(w.astype(np.float64), d, 256, want_x=False, want_margin=False)
    gpr = 256 // 8
    for rank, shards, mx in results:
        assert mx == 10.0 + (world - 1)
        covered = 0
        for a, b, idx, kind, root, P, scale in shards:
            np.testing.assert_array_equal(idx, full["idx"][a * gpr:b * gpr])
            np.testing.assert_array_equal(kind, full["kind"][a * gpr:b * gpr])
            np.testing.assert_array_equal(P, full["P"][a * gpr:b * gpr])
            np.testing.assert_array_equal(scale, full["scale"][a:b])
            covered += b - a
        assert covered == w.shape[0]


def test_shard_rows_partition():
    from bit_e8_lattice_b200.dist import shard_rows

    for rows in (0, 1, 7, 256, 14336):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def _library_form(out, rows, gpr):
    """The oracle's encoding in the library's layout: int16 indices, fp32
    scales, escape / overflow record bytes (group ids from the first row),
    int64 row pointers."""
    from bit_e8_lattice_b200.e8q import ESC_DTYPE, OVF_DTYPE

    idx, kind, root, P = out["idx"], out["kind"], out["root"], out["P"]
    ge, go = np.nonzero(kind == 1)[0], np.nonzero(kind == 2)[0]
    esc = np.zeros(len(ge), ESC_DTYPE)
    esc["group"], esc["core"], esc["root"] = ge, idx[ge], root[ge]
    ovf = np.zeros(len(go), OVF_DTYPE)
    ovf["group"], ovf["coord2"] = go, P[go]
    erp = np.concatenate([[0], np.cumsum((kind == 1).reshape(rows, gpr).sum(1))]).astype(np.int64)
    orp = np.concatenate([[0], np.cumsum((kind == 2).reshape(rows, gpr).sum(1))]).astype(np.int64)
    return (idx.astype(np.uint16).view(np.int16).reshape(rows, gpr), out["scale"].astype(np.float32),
            esc.tobytes(), len(ge), ovf.tobytes(), len(go), erp, orp)


def _gather_worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import oracle
    from bit_e8_lattice_b200 import dist as e8dist
    from bit_e8_lattice_b200 import synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, d = synth.small_f32()
        a, b = e8dist.shard_rows(w.shape[0], world, rank)
        out = oracle.project_encode(w[a:b].astype(np.float64), d, 256, want_x=False, want_margin=False)
        idx, scale, esc, ne, ovf, no, erp, orp = _library_form(out, b - a, 256 // 8)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
        esc_t = torch.frombuffer(bytearray(esc + bytes(8)), dtype=torch.uint8)  # room past the records
        ovf_t = torch.frombuffer(bytearray(ovf + bytes(20)), dtype=torch.uint8)
        res = e8dist.gather_encoded(t(idx), t(scale), esc_t, ne, ovf_t, no, t(erp), t(orp), a)
        q.put((rank, [r.numpy().copy() for r in res]))
    finally:
        dist.destroy_process_group()


def test_gather_encoded_row_shards_equal_whole_matrix():
    """Three gloo ranks with uneven row shards: after gather_encoded every
    rank holds exactly the whole matrix's encoding (indices, scales, records
    with group ids from the first row, row pointers)."""
    import oracle
    from bit_e8_lattice_b200 import synth

    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, d = synth.small_f32()
    full = oracle.project_encode(w.astype(np.float64), d, 256, want_x=False, want_margin=False)
    idx, scale, esc, ne, ovf, no, erp, orp = _library_form(full, w.shape[0], 256 // 8)
    assert ne > 0 and no >= 0
    for rank, got in results:
        np.testing.assert_array_equal(got[0], idx)
        np.testing.assert_array_equal(got[1], scale)
        assert got[2].tobytes() == esc and got[3].tobytes() == ovf
        np.testing.assert_array_equal(got[4], erp)
        np.testing.assert_array_equal(got[5], orp)


def test_shift_group_ids_across_the_sign_bit():
    """Group ids are uint32 carried in int32 words: shifting them by a shard's
    first group crosses 2^31 without error and wraps at 2^32."""
    import torch
    from bit_e8_lattice_b200.dist import shift_group_ids

    ids = np.array([0, 5, 2**31 - 3, 2**31 + 7, 2**32 - 1], dtype=np.uint64)
    for off in (0, 1, 10, 2**31, 2**32 - 5):
        words = torch.from_numpy(ids.astype(np.uint32).view(np.int32))
        got = shift_group_ids(words, off).numpy().view(np.uint32).astype(np.uint64)
        np.testing.assert_array_equal(got, (ids + np.uint64(off)) % np.uint64(2**32))


def _gemv_split_worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import oracle
    from bit_e8_lattice_b200 import dist as e8dist
    from bit_e8_lattice_b200 import synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, d = synth.small_f32(rows=200)
        x = synth.bf16_bits_to_f64(synth.gemv_x(3, 256))
        a, b = e8dist.shard_rows(w.shape[0], world, rank)
        out = oracle.project_encode(w[a:b].astype(np.float64), d, 256, want_x=False, want_margin=False)
        y_local = oracle.gemv(out["P"], out["scale"], d, 256, x)  # this rank's rows of W x
        y = e8dist.gemv_rows_allgather(torch.from_numpy(y_local))
        q.put((rank, y.numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_gemv_row_split_allgather_equals_whole_matrix():
    """Two gloo ranks, uneven row shards of a 200-row matrix: each multiplies
    its own rows (oracle GEMV on its shard's encoding), gemv_rows_allgather
    gives every rank the whole y, equal to the oracle's whole-matrix product."""
    import oracle
    from bit_e8_lattice_b200 import synth

    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gemv_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, d = synth.small_f32(rows=200)
    x = synth.bf16_bits_to_f64(synth.gemv_x(3, 256))
    full = oracle.project_encode(w.astype(np.float64), d, 256, want_x=False, want_margin=False)
    y_ref = oracle.gemv(full["P"], full["scale"], d, 256, x)
    for rank, y in results:
        assert y.shape == y_ref.shape
        np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)


def test_combine_shards_without_a_process_group():
    """combine_shards alone (the step after the exchange) joins three uneven
    shards, given out of order, into the whole matrix's encoding."""
    import torch

    import oracle
    from bit_e8_lattice_b200 import dist as e8dist
    from bit_e8_lattice_b200 import synth

    w, d = synth.small_f32()
    parts = []
    for a, b in [(100, 256), (0, 37), (37, 100)]:
        out = oracle.project_encode(w[a:b].astype(np.float64), d, 256, want_x=False, want_margin=False)
        idx, scale, esc, ne, ovf, no, erp, orp = _library_form(out, b - a, 32)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
        parts.append((t(idx), t(scale), torch.frombuffer(bytearray(esc + bytes(8)), dtype=torch.uint8), ne,
                      torch.frombuffer(bytearray(ovf + bytes(20)), dtype=torch.uint8), no, t(erp), t(orp), a))
    got = [r.numpy() for r in e8dist.combine_shards(parts, 32)]
    full = oracle.project_encode(w.astype(np.float64), d, 256, want_x=False, want_margin=False)
    idx, scale, esc, ne, ovf, no, erp, orp = _library_form(full, w.shape[0], 32)
    np.testing.assert_array_equal(got[0], idx)
    np.testing.assert_array_equal(got[1], scale)
    assert got[2].tobytes() == esc and got[3].tobytes() == ovf
    np.testing.assert_array_equal(got[4], erp)
    np.testing.assert_array_equal(got[5], orp)
