"""Process-group helpers for running the path on several GPUs.

Rows (and whole matrices) are independent -- the scale is per row and the
Hadamard transform stays inside a row -- so work is split by rows with no
data-path collective; the benchmark's only collective is the timing
reduction.  gather_encoded is the exchange for row-sharded weights: every
rank encodes its own rows and all ranks then hold the whole matrix in the
2-bit form.
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


def gather_encoded(idx, scale, esc, n_esc: int, ovf, n_ovf: int, esc_row_ptr, ovf_row_ptr, row_start: int,
                   group=None):
    """All-gather a row-sharded encoding so that every rank holds the whole
    matrix in the 2-bit form (E8-QAT, abstract: only indices and the sparse
    records travel, about 2 + 8 rho + 20 rho_o bytes per group instead of
    the 16 bytes of bf16 weights).

    Every rank passes its own shard, encoded with group ids numbered from the
    shard's first row (as one encode call over the shard gives them):
    idx int16 [rows_r][cols/8], scale float32 [rows_r], esc / ovf the record
    bytes (8 and 20 bytes a record; the first n_esc / n_ovf are used),
    esc_row_ptr / ovf_row_ptr int64 [rows_r + 1] (from 0), and row_start, the
    shard's first row in the whole matrix.  Shards are in rank order and
    contiguous.  Returns idx, scale, esc, ovf, esc_row_ptr, ovf_row_ptr of the
    whole matrix, with group ids numbered from its first row.  Works with any
    backend whose all_gather handles the tensors' device (NCCL for CUDA
    tensors, gloo for CPU ones); every rank makes the same collective calls.
    """
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    dev = idx.device
    gpr = idx.shape[1]
    counts = torch.tensor([idx.shape[0], int(n_esc), int(n_ovf), int(row_start)], dtype=torch.int64, device=dev)
    all_counts = [torch.empty_like(counts) for _ in range(world)]
    dist.all_gather(all_counts, counts, group=group)
    cnt = torch.stack(all_counts).cpu().tolist()  # [world][rows, n_esc, n_ovf, row_start]

    def gather_padded(t, n_items: int, item_shape, dtype, key: int):
        cap = max(1, max(c[key] for c in cnt))
        buf = torch.zeros((cap,) + tuple(item_shape), dtype=dtype, device=dev)
        if n_items:
            buf[:n_items] = t[:n_items]
        parts = [torch.empty_like(buf) for _ in range(world)]
        dist.all_gather(parts, buf, group=group)
        return [parts[r][: cnt[r][key]] for r in range(world)]

    # indices travel as their bytes (every backend gathers uint8)
    idx_parts = [t.view(idx.dtype) for t in gather_padded(idx.contiguous().view(torch.uint8), idx.shape[0], (2 * gpr,),
                                                          torch.uint8, 0)]
    scale_parts = gather_padded(scale, scale.shape[0], (), scale.dtype, 0)
    esc_parts = gather_padded(esc.view(torch.int32).view(-1, 2), int(n_esc), (2,), torch.int32, 1)
    ovf_parts = gather_padded(ovf.view(torch.int32).view(-1, 5), int(n_ovf), (5,), torch.int32, 2)
    # row pointers: all_gather of the padded [rows_r + 1] arrays
    rp_cap = max(c[0] for c in cnt) + 1

    def gather_rp(rp):
        buf = torch.zeros(rp_cap, dtype=torch.int64, device=dev)
        buf[: rp.shape[0]] = rp
        parts = [torch.empty_like(buf) for _ in range(world)]
        dist.all_gather(parts, buf, group=group)
        return [parts[r][: cnt[r][0] + 1] for r in range(world)]

    erp_parts, orp_parts = gather_rp(esc_row_ptr), gather_rp(ovf_row_ptr)
    esc_out, ovf_out, erp_out, orp_out = [], [], [], []
    e_base = o_base = 0
    for r in range(world):
        off = cnt[r][3] * gpr  # the shard's first group in the whole matrix
        e = esc_parts[r].clone()
        o = ovf_parts[r].clone()
        for t in (e, o):
            if t.shape[0]:
                t[:, 0] = shift_group_ids(t[:, 0], off)
        esc_out.append(e)
        ovf_out.append(o)
        erp_out.append(erp_parts[r][:-1] + e_base)
        orp_out.append(orp_parts[r][:-1] + o_base)
        e_base += cnt[r][1]
        o_base += cnt[r][2]
    erp_out.append(torch.tensor([e_base], dtype=torch.int64, device=dev))
    orp_out.append(torch.tensor([o_base], dtype=torch.int64, device=dev))
    return (torch.cat(idx_parts), torch.cat(scale_parts), torch.cat(esc_out).view(torch.uint8).reshape(-1),
            torch.cat(ovf_out).view(torch.uint8).reshape(-1), torch.cat(erp_out), torch.cat(orp_out))
