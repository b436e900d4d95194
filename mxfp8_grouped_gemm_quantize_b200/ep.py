"""Expert-parallel token exchange around the grouped GEMM (one process per GPU).

Each MoE layer wraps its grouped GEMMs in two all-to-alls (opensourcebeat.com,
"Enabling up to 41% faster pre-training: MXFP8 and DeepEP for DeepSeek-V3 on
B200 with TorchTitan", section "Двухсторонняя атака"): the dispatch sends every
routed (token, slot) pair's row to the rank that owns its expert, and the
return brings the expert outputs back.  The experts are split into P
contiguous ranges: rank r owns experts [r*E/P, (r+1)*E/P).

This module orders rows and exchanges them; transport is
torch.distributed.all_to_all_single (NCCL between GPUs, gloo on CPU).  Every
arithmetic step of the layer stays in the library's kernels.  On one rank:

    rows, local_e, ex = dispatch(x, idx, E)                  # rows routed here, sender by sender
    offs, perm, inv, _ = mxfp8_moe_plan(local_e[:, None], E // P)
    q, s, qT, sT = mxfp8_permute_quantize_dual(rows, perm, offs)
    ...grouped GEMMs on (q, s, qT, sT) with offs; outputs y_grouped [R, C]...
    y_rows = mxfp8_moe_combine(y_grouped, inv, ones)          # back to the received order (exact)
    y_pairs = give_back(y_rows, ex)                           # [T*k, C], row p = pair p = t*k + j
    y = mxfp8_moe_combine(y_pairs, arange(T*k).view(T, k), w)

The exchange moves bf16 rows (2 bytes per element); sending the MXFP8 codes
and scales instead (1 + 1/32 bytes) and fusing the transfer into the quantiser
over NVLink peer memory are the next steps and are not built.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Exchange:
    """Bookkeeping of one dispatch, for the return trip."""
    order: torch.Tensor      # int64 [T*k]: pair indices sorted by destination rank (stable)
    send_counts: list        # rows this rank sent to each rank
    recv_counts: list        # rows this rank received from each rank
    num_pairs: int           # T*k


def _sizes(group):
    return dist.get_world_size(group), dist.get_rank(group)


def dispatch(x: torch.Tensor, idx: torch.Tensor, num_experts: int, group=None):
    """x: [T, C] token rows; idx: integer [T, k] global expert ids in [0, E).

    Returns (rows [R, C], local_expert int32 [R], Exchange): the rows routed
    to this rank's experts, grouped by sending rank (rank 0's first) and in
    (token, slot) order within a sender, with their expert ids relative to
    this rank's range.  Raises ValueError if E is not a multiple of the group
    size or an id is out of range."""
    P, _ = _sizes(group)
    if num_experts % P != 0:
        raise ValueError(f"{num_experts} experts cannot be split evenly over {P} ranks")
    if x.dim() != 2 or idx.dim() != 2 or x.shape[0] != idx.shape[0]:
        raise ValueError("x must be [T, C] and idx [T, k] with the same T")
    epr = num_experts // P
    T, k = idx.shape
    flat = idx.reshape(-1).to(torch.int64)
    if flat.numel() and (int(flat.min()) < 0 or int(flat.max()) >= num_experts):
        raise ValueError("expert id out of range")
    dest = torch.div(flat, epr, rounding_mode="floor")
    order = torch.sort(dest, stable=True).indices
    send = torch.bincount(dest, minlength=P).to(torch.int64)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    sc, rc = send.tolist(), recv.tolist()
    rows_out = x.index_select(0, torch.div(order, k, rounding_mode="floor"))
    rows_in = x.new_empty((sum(rc), x.shape[1]))
    dist.all_to_all_single(rows_in, rows_out, output_split_sizes=rc, input_split_sizes=sc, group=group)
    le_out = torch.remainder(flat.index_select(0, order), epr).to(torch.int32)
    le_in = torch.empty(sum(rc), dtype=torch.int32, device=x.device)
    dist.all_to_all_single(le_in, le_out, output_split_sizes=rc, input_split_sizes=sc, group=group)
    return rows_in, le_in, Exchange(order, sc, rc, T * k)


def give_back(y_rows: torch.Tensor, ex: Exchange, group=None) -> torch.Tensor:
    """y_rows: [R, C], one output row per row received by dispatch, in the
    same order.  Returns [T*k, C] on the token's home rank: row p is the
    output for pair p = token * k + slot."""
    if y_rows.shape[0] != sum(ex.recv_counts):
        raise ValueError("one output row per received row is needed")
    back = y_rows.new_empty((sum(ex.send_counts), y_rows.shape[1]))
    dist.all_to_all_single(back, y_rows.contiguous(), output_split_sizes=ex.send_counts,
                           input_split_sizes=ex.recv_counts, group=group)
    out = torch.empty_like(back)
    out.index_copy_(0, ex.order, back)
    return out
