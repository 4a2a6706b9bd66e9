"""Process-group helpers for running the path on several GPUs.

Rows (and whole matrices) are independent -- the scale is per row and the
Hadamard transform stays inside a row -- so work is split by rows.  Two
exchanges serve row-sharded weights: gather_encoded (every rank encodes its
own rows, then all ranks hold the whole matrix in the 2-bit form) and
gemv_rows_allgather (every rank multiplies its own rows, then all ranks
hold the whole product).
"""
from __future__ import annotations

import os


def rank_info():
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_rows(rows: int, world: int, rank: int):
    """Contiguous row range [start, stop) of this rank; sizes differ by at most one."""
    base, extra = divmod(rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the default process group."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shift_group_ids(words, offset: int):
    """uint32 group ids held in an int32 tensor, plus offset, modulo 2^32 (as int32)."""
    import torch

    g = ((words.to(torch.int64) & 0xFFFFFFFF) + int(offset)) & 0xFFFFFFFF
    return torch.where(g >= (1 << 31), g - (1 << 32), g).to(torch.int32)


def combine_shards(parts, gpr: int):
    """Join row shards of one matrix's encoding, in row order, into the whole
    matrix's encoding (no communication).  Each part is (idx, scale, esc,
    n_esc, ovf, n_ovf, esc_row_ptr, ovf_row_ptr, row_start) as
    gather_encoded takes it: idx int16 [rows_r][gpr], scale float32
    [rows_r], esc / ovf record bytes (8 / 20 bytes a record, group ids
    numbered from the shard's first row; the first n_esc / n_ovf are used),
    row pointers int64 [rows_r + 1] from 0, row_start the shard's first row.
    Returns idx, scale, esc, ovf (bytes), esc_row_ptr, ovf_row_ptr of the
    whole matrix, group ids numbered from its first row."""
    import torch

    parts = sorted(parts, key=lambda t: int(t[8]))
    dev = parts[0][0].device
    idx_out, sc_out, esc_out, ovf_out, erp_out, orp_out = [], [], [], [], [], []
    e_base = o_base = 0
    for idx, scale, esc, n_esc, ovf, n_ovf, erp, orp, row_start in parts:
        n_esc, n_ovf, off = int(n_esc), int(n_ovf), int(row_start) * gpr
        e = esc.reshape(-1)[: 8 * n_esc].view(torch.int32).view(-1, 2).clone()
        o = ovf.reshape(-1)[: 20 * n_ovf].view(torch.int32).view(-1, 5).clone()
        for t in (e, o):
            if t.shape[0]:
                t[:, 0] = shift_group_ids(t[:, 0], off)
        idx_out.append(idx.reshape(-1, gpr))
        sc_out.append(scale.reshape(-1))
        esc_out.append(e)
        ovf_out.append(o)
        erp_out.append(erp.reshape(-1)[:-1] + e_base)
        orp_out.append(orp.reshape(-1)[:-1] + o_base)
        e_base += n_esc
        o_base += n_ovf
    erp_out.append(torch.tensor([e_base], dtype=torch.int64, device=dev))
    orp_out.append(torch.tensor([o_base], dtype=torch.int64, device=dev))
    return (torch.cat(idx_out), torch.cat(sc_out), torch.cat(esc_out).view(torch.uint8).reshape(-1),
            torch.cat(ovf_out).view(torch.uint8).reshape(-1), torch.cat(erp_out), torch.cat(orp_out))


def gather_encoded(idx, scale, esc, n_esc: int, ovf, n_ovf: int, esc_row_ptr, ovf_row_ptr, row_start: int,
                   group=None):
    """All-gather a row-sharded encoding so that every rank holds the whole
    matrix in the 2-bit form (E8-QAT, abstract: only indices and the sparse
    records travel, about 2 + 8 rho + 20 rho_o bytes per group instead of
    the 16 bytes of bf16 weights; the SQuAT page's distributed search
    likewise returns only discrete indices).

    Every rank passes its own shard as combine_shards describes it.  Two
    collectives: the shard sizes (one small all_gather, read on the host to
    size the next), then one all_gather of every shard packed into a single
    byte buffer (indices, scales, records, row pointers; padded to the
    largest shard).  Shards are in rank order and contiguous.  Works with
    any backend whose all_gather handles the tensors' device (NCCL for CUDA
    tensors, gloo for CPU ones); every rank makes the same collective calls.
    """
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    dev = idx.device
    gpr = idx.shape[1]
    rows = idx.shape[0]
    n_esc, n_ovf = int(n_esc), int(n_ovf)
    counts = torch.tensor([rows, n_esc, n_ovf, int(row_start)], dtype=torch.int64, device=dev)
    all_counts = [torch.empty_like(counts) for _ in range(world)]
    dist.all_gather(all_counts, counts, group=group)
    cnt = torch.stack(all_counts).cpu().tolist()  # [world][rows, n_esc, n_ovf, row_start]

    def sizes(c):  # byte lengths of the packed parts of one shard
        r, ne, no = c[0], c[1], c[2]
        return [2 * r * gpr, 4 * r, 8 * ne, 20 * no, 8 * (r + 1), 8 * (r + 1)]

    def pad16(n):  # every part starts on a 16-byte boundary, so that it can be viewed as its type
        return (n + 15) // 16 * 16

    cap = max(sum(pad16(n) for n in sizes(c)) for c in cnt)
    mine = [idx.contiguous().view(torch.uint8).reshape(-1), scale.contiguous().view(torch.uint8).reshape(-1),
            esc.reshape(-1)[: 8 * n_esc], ovf.reshape(-1)[: 20 * n_ovf],
            esc_row_ptr.contiguous().view(torch.uint8).reshape(-1), ovf_row_ptr.contiguous().view(torch.uint8).reshape(-1)]
    buf = torch.zeros(cap, dtype=torch.uint8, device=dev)
    o = 0
    for t in mine:
        buf[o: o + t.numel()] = t
        o += pad16(t.numel())
    bufs = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(bufs, buf, group=group)
    parts = []
    for r in range(world):
        sz, o, pieces = sizes(cnt[r]), 0, []
        for n in sz:
            pieces.append(bufs[r][o: o + n])
            o += pad16(n)
        rr = cnt[r][0]
        parts.append((pieces[0].view(torch.int16).reshape(rr, gpr), pieces[1].view(torch.float32), pieces[2],
                      cnt[r][1], pieces[3], cnt[r][2], pieces[4].view(torch.int64), pieces[5].view(torch.int64),
                      cnt[r][3]))
    return combine_shards(parts, gpr)


def gemv_rows_allgather(y_local, group=None):
    """Row-split dequant-GEMV or -GEMM, exchange step: every rank computed
    y_local = W_r x for its own row shard W_r (bf16 [batch][rows_r], from
    e8q_dequant_gemv or e8q_dequant_gemm: both write that layout); one
    all_gather (padded to the largest shard) gives every rank the whole
    y = W x, [batch][sum of rows_r] in rank order."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    dev = y_local.device
    n = torch.tensor([y_local.shape[1]], dtype=torch.int64, device=dev)
    ns = [torch.empty_like(n) for _ in range(world)]
    dist.all_gather(ns, n, group=group)
    rows = [int(t.item()) for t in ns]
    cap = max(rows)
    buf = torch.zeros((y_local.shape[0], cap), dtype=y_local.dtype, device=dev)
    buf[:, : y_local.shape[1]] = y_local
    outs = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(outs, buf, group=group)
    return torch.cat([o[:, :r] for o, r in zip(outs, rows)], dim=1)
