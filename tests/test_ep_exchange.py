"""The expert-parallel exchange on CPU with two and three gloo ranks, MXFP8
payloads.  Each rank plans and packs its tokens (here with the oracle, since
the library's kernels need a GPU), `ep.exchange` moves records and pair
entries, and the receiver's grouped rowwise MXFP8 equals, byte for byte, the
quantisation the local path (every rank's tokens on one device) gives the rows
of that rank's experts.  The return trip (`ep.return_rows`) and the combine
give the local layer's output bit for bit."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(rank, T, k, E, C):
    from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
    rng = np.random.default_rng(1000 + rank)
    idx = np.argsort(-rng.standard_normal((T, E)), axis=1)[:, :k].astype(np.int32)   # distinct experts
    w = rng.random((T, k)).astype(np.float32)
    x = wl.normal_bf16((T, C), 1.0, 2000 + rank)
    return x, idx, w


def _layer_rank(rank, world, port, q, T, k, E, C, N):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from mxfp8_grouped_gemm_quantize_b200 import ep, workloads as wl
        epr = E // world
        x, idx, w = _inputs(rank, T, k, E, C)
        W = wl.normal_bf16((E * N, C), 0.05, 77)

        def experts(q_rows, sf_rows, offs, e0):
            wq, wsf = oracle.quantize_rowwise(W[e0 * N:(e0 + len(offs) - 1) * N])
            y = np.zeros((q_rows.shape[0], N))
            for _, lo, hi, Ye in oracle.fwd_by_expert(q_rows, sf_rows, wq, wsf, offs, N):
                y[lo:hi] = Ye
            return oracle.bf16_from_double(y)

        # send side
        pl = oracle.ep_plan(idx, E, world)
        records = torch.from_numpy(oracle.ep_pack(x, pl.rec_token))
        rec_in, pe_in, pr_in, rc = ep.exchange(records, torch.from_numpy(pl.pair_expert),
                                               torch.from_numpy(pl.pair_rec), pl.counts.tolist())
        # receive side
        offs, perm, inv = oracle.moe_plan(pe_in.numpy()[:, None], epr)
        qr, sfr = oracle.ep_unpack(rec_in.numpy(), C, pr_in.numpy(), ep.source_bases(rc), perm, offs)
        # the local path over every rank's tokens
        ins = [_inputs(s, T, k, E, C) for s in range(world)]
        X = torch.cat([a[0] for a in ins])
        idx_all = np.concatenate([a[1] for a in ins])
        offs_g, perm_g, inv_g = oracle.moe_plan(idx_all, E)
        lo, hi = int(offs_g[rank * epr]), int(offs_g[(rank + 1) * epr])
        q_ref, sf_ref = oracle.quantize_rowwise(X[torch.from_numpy(perm_g[lo:hi].astype(np.int64))],
                                                offs_g[rank * epr:(rank + 1) * epr + 1] - lo)
        nb = oracle.rowwise_scale_bytes(hi - lo, C, epr) if hi > lo else 0
        ok_rows = bool(np.array_equal(offs, offs_g[rank * epr:(rank + 1) * epr + 1] - lo)
                       and np.array_equal(qr, q_ref) and np.array_equal(sfr[:nb], sf_ref[:nb]))
        # payload: MXFP8 records, not bf16 rows
        sent_bytes = records.numel()
        bf16_bytes = 2 * C * int(pl.counts[world:].sum())
        # return trip and combine
        y_r = experts(qr, sfr, offs, rank * epr)
        y_ret = torch.from_numpy(y_r[inv[:, 0]].view(np.int16)).view(torch.bfloat16)
        back = ep.return_rows(y_ret, rc, pl.counts.tolist()).view(torch.int16).numpy().view(np.uint16)
        y = oracle.moe_combine(back, pl.ret_pos, w)
        qg, sg = oracle.quantize_rowwise(X[torch.from_numpy(perm_g.astype(np.int64))], offs_g)
        y_local = oracle.moe_combine(experts(qg, sg, offs_g, 0), inv_g, np.concatenate([a[2] for a in ins]))
        ok_y = bool(np.array_equal(y, y_local[rank * T:(rank + 1) * T]))
        q.put((rank, ok_rows, ok_y, sent_bytes, bf16_bytes, int(pl.counts[world:].sum())))
    finally:
        torch.distributed.destroy_process_group()


def _run(target, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q) + args) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("world,T,k,E,C,N", [(2, 40, 3, 8, 64, 32), (3, 30, 4, 12, 96, 32),
                                             (2, 25, 6, 8, 1408, 32)])
def test_mxfp8_dispatch_and_return_match_the_local_layer(world, T, k, E, C, N):
    got = _run(_layer_rank, world, T, k, E, C, N)
    assert all(ok_rows for _, ok_rows, _, _, _, _ in got), got
    assert all(ok_y for _, _, ok_y, _, _, _ in got), got
    assert sum(n for *_, n in got) == world * T * k              # every routed pair was sent once
    for _, _, _, sent, bf16, _ in got:
        assert sent < 0.6 * bf16                                   # codes + scales, each token once per rank


def _bad(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        from mxfp8_grouped_gemm_quantize_b200 import ep
        recs = torch.zeros((3, 16), dtype=torch.uint8)
        pe = torch.zeros(4, dtype=torch.int32)
        errs = []
        for counts in ([1, 1, 2], [1, 1, 2, 1], [1, 2, 2, 1]):    # wrong length; 2 records, not 3; 3 pairs, not 4
            try:
                ep.exchange(recs, pe, pe, counts)
                errs.append(False)
            except ValueError:
                errs.append(True)
        try:
            ep.return_rows(torch.zeros((3, 8)), [0, 0, 1, 1], [0, 0, 1, 1])
            errs.append(False)
        except ValueError:
            errs.append(True)
        q.put((rank, errs))
    finally:
        torch.distributed.destroy_process_group()


def test_buffers_that_do_not_match_the_counts_are_rejected_before_any_exchange():
    got = _run(_bad, 2)
    assert all(e == [True, True, True, True] for _, e in got), got


def _edge(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from mxfp8_grouped_gemm_quantize_b200 import ep, workloads as wl
        E, C = 4, 64
        if rank == 0:   # no tokens at all
            x, idx = wl.normal_bf16((0, C), 1.0, 1), np.zeros((0, 2), dtype=np.int32)
        else:           # every pair goes to rank 1's own experts (2 and 3): one record per token
            x, idx = wl.normal_bf16((5, C), 1.0, 2), np.array([[2, 3]] * 5, dtype=np.int32)
        pl = oracle.ep_plan(idx, E, world)
        records = torch.from_numpy(oracle.ep_pack(x, pl.rec_token))
        rec_in, pe_in, pr_in, rc = ep.exchange(records, torch.from_numpy(pl.pair_expert),
                                               torch.from_numpy(pl.pair_rec), pl.counts.tolist())
        y_ret = torch.arange(pe_in.numel() * 8, dtype=torch.float32).view(-1, 8)
        back = ep.return_rows(y_ret, rc, pl.counts.tolist())
        if rank == 0:
            ok = rec_in.shape[0] == 0 and pe_in.numel() == 0 and back.shape == (0, 8) and rc == [0, 0, 0, 0]
        else:
            ok = (rec_in.shape[0] == 5 and rc == [0, 5, 0, 10] and pe_in.tolist() == [0, 1] * 5
                  and pr_in.tolist() == [0, 0, 1, 1, 2, 2, 3, 3, 4, 4] and torch.equal(back, y_ret)
                  and torch.equal(rec_in, records))
        q.put((rank, ok))
    finally:
        torch.distributed.destroy_process_group()


def test_a_rank_without_tokens_and_a_rank_receiving_nothing():
    got = _run(_edge, 2)
    assert all(ok for _, ok in got), got
