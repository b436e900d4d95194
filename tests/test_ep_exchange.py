"""The expert-parallel exchange on CPU with two and three gloo ranks: every
routed pair's row reaches the rank owning its expert, grouped by sender in
(token, slot) order with its local expert id, and the return trip puts each
expert output back at its pair's position on the token's home rank."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(rank, T, k, E, C, dtype):
    g = torch.Generator().manual_seed(1000 + rank)
    logits = torch.randn((T, E), generator=g)
    idx = torch.topk(logits, k, dim=1).indices.to(torch.int32)      # distinct experts per token
    x = torch.randn((T, C), generator=g).to(dtype)
    return x, idx


def _rank(rank, world, port, q, T, k, E, C, dtype):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        from mxfp8_grouped_gemm_quantize_b200 import ep
        x, idx = _inputs(rank, T, k, E, C, dtype)
        rows, le, ex = ep.dispatch(x, idx, E)
        epr = E // world
        # expected: senders in rank order, each sender's pairs routed here in (token, slot) order
        exp_rows, exp_le = [], []
        for s in range(world):
            xs, idxs = _inputs(s, T, k, E, C, dtype)
            flat = idxs.reshape(-1).long()
            for p in range(T * k):
                if int(flat[p]) // epr == rank:
                    exp_rows.append(xs[p // k])
                    exp_le.append(int(flat[p]) % epr)
        ok = len(exp_rows) == rows.shape[0] and torch.equal(torch.stack(exp_rows) if exp_rows else rows, rows) \
            and le.tolist() == exp_le
        # "experts": scale each received row by (local expert + 1), exactly representable
        y_rows = rows * (le.to(rows.dtype) + 1)[:, None]
        back = ep.give_back(y_rows, ex)
        flat = idx.reshape(-1).long()
        exp_back = x.index_select(0, torch.arange(T * k) // k) * (flat % epr + 1).to(x.dtype)[:, None]
        ok = ok and torch.equal(back, exp_back) and back.shape == (T * k, C)
        q.put((rank, ok, rows.shape[0]))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world,T,k,E,C,dtype", [(2, 12, 3, 8, 16, torch.float32),
                                                 (2, 7, 2, 4, 8, torch.bfloat16),
                                                 (3, 10, 4, 12, 8, torch.float32)])
def test_dispatch_and_return(world, T, k, E, C, dtype):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, T, k, E, C, dtype)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok, _ in got), got
    assert sum(n for _, _, n in got) == world * T * k       # every pair landed somewhere exactly once


def _bad(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        from mxfp8_grouped_gemm_quantize_b200 import ep
        x = torch.zeros((4, 8))
        errs = []
        for E, idx in ((5, torch.zeros((4, 1), dtype=torch.int32)),          # 5 experts over 2 ranks
                       (4, torch.full((4, 1), 4, dtype=torch.int32))):        # id out of range
            try:
                ep.dispatch(x, idx, E)
                errs.append(False)
            except ValueError:
                errs.append(True)
        q.put((rank, errs))
    finally:
        torch.distributed.destroy_process_group()


def test_invalid_splits_and_ids_are_rejected_before_any_exchange():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bad, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(e == [True, True] for _, e in got)


def _edge(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        from mxfp8_grouped_gemm_quantize_b200 import ep
        E, C = 4, 8
        if rank == 0:   # no tokens at all
            x, idx = torch.zeros((0, C)), torch.zeros((0, 2), dtype=torch.int32)
        else:           # every pair goes to rank 1's own experts (2 and 3)
            x = torch.arange(5 * C, dtype=torch.float32).view(5, C)
            idx = torch.tensor([[2, 3]] * 5, dtype=torch.int32)
        rows, le, ex = ep.dispatch(x, idx, E)
        back = ep.give_back(rows * 2, ex)
        if rank == 0:
            ok = rows.shape == (0, C) and le.numel() == 0 and back.shape == (0, C)
        else:
            exp = x.repeat_interleave(2, dim=0)
            ok = torch.equal(rows, exp) and le.tolist() == [0, 1] * 5 and torch.equal(back, exp * 2)
        q.put((rank, ok))
    finally:
        torch.distributed.destroy_process_group()


def test_a_rank_without_tokens_and_a_rank_receiving_nothing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_edge, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok in got), got
