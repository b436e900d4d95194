"""Expert-parallel token exchange around the grouped GEMM (one process per GPU).

Outside the single-GPU hot path: the layer's timed step runs on one GPU's
experts; this module is the exchange that feeds them when the experts are
spread over P ranks.

Each MoE layer wraps its grouped GEMMs in two all-to-alls (opensourcebeat.com,
"Enabling up to 41% faster pre-training: MXFP8 and DeepEP for DeepSeek-V3 on
B200 with TorchTitan", section "Двухсторонняя атака"): the dispatch sends the
tokens to the ranks that own their experts, the return brings the expert
outputs back.  A token needed by several experts of one rank crosses once and
is copied there (iitak.ru, "NVIDIA в 10 раз ускорила обучение
моделей-«смесей экспертов» на JAX", paragraph on NCCL EP).  Rank r owns
experts [r*E/P, (r+1)*E/P).

What travels (formats in include/mxfp8.h, "expert-parallel dispatch"):
  - one record per (token, destination rank): the token row in rowwise MXFP8,
    codes + scale bytes, 1 + 1/32 bytes per element instead of bf16's 2;
  - one pair entry per routed (token, slot): local expert id and record index;
  - on the way back, one bf16 output row per pair.
The plan, the quantise-and-pack, the unpack into the grouped GEMM's layout and
the return gather run in the library's kernels; this module only moves their
buffers with torch.distributed.all_to_all_single (NCCL between GPUs, gloo on
CPU) along the plan's counts.  On one rank:

    d = dispatch(x, idx, E)                           # plan + pack, exchange
    offs, perm, inv, q, s = receive(d, E // P)        # grouped rowwise MXFP8 of the received rows
    y_grouped = mxfp8_grouped_gemm_fwd(q, s, wq, ws, offs, N)
    y_back = give_back(y_grouped, inv, d)             # [pairs sent, N], row ret_pos[t, j] = slot (t, j)
    y = mxfp8_moe_combine(y_back, d.ret_pos, w)

`exchange` and `return_rows` are the transport alone and take buffers made
anywhere (the CPU tests build them with the oracle and move them over gloo).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Dispatch:
    """What arrived at this rank, and the bookkeeping of the return trip."""
    records: torch.Tensor       # uint8 [R_in, record bytes]: rowwise MXFP8 token rows, by source rank
    pair_expert: torch.Tensor   # int32 [S_in]: local expert of each received pair
    pair_rec: torch.Tensor      # int32 [S_in]: record of each pair, within its source's records
    recv_counts: list           # [2P]: records from each source, then pairs from each source
    send_counts: list           # [2P]: records to each rank, then pairs to each rank
    cols: int                   # elements per token row
    ret_pos: torch.Tensor | None = None   # int32 [T, k]: row of each slot's output on the way back (-1: none)


def _sizes(group):
    return dist.get_world_size(group), dist.get_rank(group)


def source_bases(recv_counts) -> list:
    """[2P] counts -> [2(P+1)]: first pair of each source (and the total), then
    first record of each source (and the total)."""
    P = len(recv_counts) // 2
    rec, pairs = recv_counts[:P], recv_counts[P:]
    out = [0]
    for c in pairs:
        out.append(out[-1] + int(c))
    out.append(0)
    for c in rec:
        out.append(out[-1] + int(c))
    return out


def exchange(records: torch.Tensor, pair_expert: torch.Tensor, pair_rec: torch.Tensor, send_counts, group=None):
    """Transport of one dispatch.  records [R, B] uint8, pair_expert / pair_rec
    int32 [S], send_counts [2P] (records, then pairs, to each rank; host ints),
    all in send order.  Returns (records_in, pair_expert_in, pair_rec_in,
    recv_counts), sources in rank order."""
    P, _ = _sizes(group)
    sc = [int(c) for c in send_counts]
    if len(sc) != 2 * P:
        raise ValueError(f"send_counts needs {2 * P} entries")
    if records.shape[0] != sum(sc[:P]) or pair_expert.numel() != sum(sc[P:]) or pair_rec.numel() != sum(sc[P:]):
        raise ValueError("buffers do not match the counts")
    dev = records.device
    cnt_out = torch.tensor(sc, dtype=torch.int64, device=dev).view(2, P).t().contiguous()   # [P, 2]
    cnt_in = torch.empty_like(cnt_out)
    dist.all_to_all_single(cnt_in, cnt_out, group=group)
    rc = cnt_in.t().reshape(-1).tolist()
    rec_in = records.new_empty((sum(rc[:P]), records.shape[1]))
    dist.all_to_all_single(rec_in, records.contiguous(), output_split_sizes=rc[:P], input_split_sizes=sc[:P],
                           group=group)
    pe_in = pair_expert.new_empty(sum(rc[P:]))
    pr_in = pair_rec.new_empty(sum(rc[P:]))
    dist.all_to_all_single(pe_in, pair_expert.contiguous(), output_split_sizes=rc[P:], input_split_sizes=sc[P:],
                           group=group)
    dist.all_to_all_single(pr_in, pair_rec.contiguous(), output_split_sizes=rc[P:], input_split_sizes=sc[P:],
                           group=group)
    return rec_in, pe_in, pr_in, rc


def return_rows(y_ret: torch.Tensor, recv_counts, send_counts, group=None) -> torch.Tensor:
    """Transport of the return trip: y_ret holds one row per received pair in
    arrival order; returns one row per sent pair, in send order."""
    P, _ = _sizes(group)
    rc, sc = [int(c) for c in recv_counts[P:]], [int(c) for c in send_counts[P:]]
    if y_ret.shape[0] != sum(rc):
        raise ValueError("one row per received pair is needed")
    back = y_ret.new_empty((sum(sc),) + tuple(y_ret.shape[1:]))
    dist.all_to_all_single(back, y_ret.contiguous(), output_split_sizes=sc, input_split_sizes=rc, group=group)
    return back


def dispatch(x: torch.Tensor, idx: torch.Tensor, num_experts: int, group=None) -> Dispatch:
    """x: bf16 [T, C] token rows on this rank's GPU; idx: int32 [T, k] global
    expert ids.  Plans and packs with the library's kernels, then exchanges.
    Raises ValueError if E is not a multiple of the group size, and the
    library's error if an id is outside [0, E)."""
    from . import mxfp8_ep_pack, mxfp8_ep_plan, mxfp8_get_status, MXFP8Error
    P, _ = _sizes(group)
    if num_experts % P != 0:
        raise ValueError(f"{num_experts} experts cannot be split evenly over {P} ranks")
    if x.dim() != 2 or idx.dim() != 2 or x.shape[0] != idx.shape[0]:
        raise ValueError("x must be [T, C] and idx [T, k] with the same T")
    counts, rec_token, pair_expert, pair_rec, ret_pos, work = mxfp8_ep_plan(idx.to(torch.int32).contiguous(),
                                                                            num_experts, P)
    st = mxfp8_get_status(work)            # synchronises: NCCL needs the counts on the host
    if st != 0:
        raise MXFP8Error(st, "mxfp8_ep_plan")
    sc = counts.tolist()
    R, S = sum(sc[:P]), sum(sc[P:])
    records = mxfp8_ep_pack(x.contiguous(), rec_token[:R])
    rec_in, pe_in, pr_in, rc = exchange(records, pair_expert[:S], pair_rec[:S], sc, group)
    return Dispatch(rec_in, pe_in, pr_in, rc, sc, x.shape[1], ret_pos)


def receive(d: Dispatch, num_local_experts: int):
    """Groups the received pairs by local expert and writes their rows as the
    grouped GEMM's rowwise MXFP8 operand.  Returns (offs, perm, inv, q, scales):
    offs int32 [E_loc + 1], perm int32 [S_in] (pair of each grouped row),
    inv int32 [S_in, 1] (grouped row of each pair)."""
    from . import mxfp8_ep_unpack, mxfp8_get_status, mxfp8_moe_plan, MXFP8Error
    dev = d.records.device
    offs, perm, inv, work = mxfp8_moe_plan(d.pair_expert.view(-1, 1), num_local_experts)
    src_base = torch.tensor(source_bases(d.recv_counts), dtype=torch.int32).to(dev, non_blocking=True)
    q, scales = mxfp8_ep_unpack(d.records, d.cols, d.pair_rec, src_base, perm, offs)
    st = mxfp8_get_status(work)
    if st != 0:
        raise MXFP8Error(st, "mxfp8_moe_plan")
    return offs, perm, inv, q, scales


def give_back(y_grouped: torch.Tensor, inv: torch.Tensor, d: Dispatch, group=None) -> torch.Tensor:
    """y_grouped [S_in, N]: expert outputs of the grouped rows.  Sends each
    received pair's row back to its source; returns [pairs sent, N] whose row
    d.ret_pos[t, j] is slot (t, j)'s output (mxfp8_moe_combine's yp and inv)."""
    from . import mxfp8_gather_rows
    y_ret = mxfp8_gather_rows(y_grouped, inv.reshape(-1).contiguous())
    return return_rows(y_ret, d.recv_counts, d.send_counts, group)
