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
