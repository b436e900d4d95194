"""Pins for the oracle's expert-parallel dispatch (CPU): the send plan, the
MXFP8 records a token travels in, and the receiving side's grouped layout.

- the plan equals a brute-force enumeration of (rank, token, slot) triples on
  small inputs, and keeps its invariants on larger ones; with one rank it
  reduces to the local dispatch plan (pinned against numpy's stable argsort);
- a record's codes and scale bytes equal an independent numpy block quantiser
  (np.log2 + ml_dtypes);
- records sent by several ranks and unpacked by their receivers give, byte for
  byte, the oracle's rowwise quantisation of the rows the local path (all
  tokens on one device) groups under those experts; the return trip and the
  combine give the local path's output bit for bit.
"""
import itertools

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl


def _routing(seed, T, k, E):
    rng = np.random.default_rng(seed)
    return np.argsort(-rng.standard_normal((T, E)), axis=1)[:, :k].astype(np.int32)


def brute_plan(idx, E, P):
    """Enumerates the valid (rank, token, slot) triples in sorted order."""
    T, k = idx.shape
    epr = E // P
    triples = sorted((int(e) // epr, t, j) for t in range(T) for j in range(k)
                     for e in [idx[t, j]] if 0 <= e < E)
    records = sorted({(p, t) for p, t, _ in triples})
    rec_at = {r: i for i, r in enumerate(records)}
    first_rec = {p: min((i for i, (q, _) in enumerate(records) if q == p), default=0) for p in range(P)}
    counts = [sum(1 for q, _ in records if q == p) for p in range(P)] + \
             [sum(1 for q, _, _ in triples if q == p) for p in range(P)]
    ret = -np.ones((T, k), dtype=np.int64)
    pe, prc = [], []
    for s, (p, t, j) in enumerate(triples):
        ret[t, j] = s
        pe.append(int(idx[t, j]) % epr)
        prc.append(rec_at[(p, t)] - first_rec[p])
    return counts, [t for _, t in records], pe, prc, ret


@pytest.mark.parametrize("seed,T,k,E,P", [(0, 9, 3, 8, 2), (1, 12, 4, 12, 3), (2, 7, 2, 4, 4),
                                          (3, 10, 6, 12, 1), (4, 11, 8, 16, 4)])
def test_plan_equals_brute_force(seed, T, k, E, P):
    idx = _routing(seed, T, k, E)
    pl = oracle.ep_plan(idx, E, P)
    counts, rec_token, pe, prc, ret = brute_plan(idx, E, P)
    assert pl.counts.tolist() == counts
    assert pl.rec_token.tolist() == rec_token
    assert pl.pair_expert.tolist() == pe and pl.pair_rec.tolist() == prc
    assert np.array_equal(pl.ret_pos, ret)
    assert pl.bad == 0


def test_plan_with_repeated_experts_bad_ids_and_empty_tokens():
    idx = np.array([[5, 5, 1], [9, -1, 2], [0, 3, 3], [7, 7, 7]], dtype=np.int32)
    pl = oracle.ep_plan(idx, 8, 2)
    counts, rec_token, pe, prc, ret = brute_plan(idx, 8, 2)
    assert pl.counts.tolist() == counts and pl.rec_token.tolist() == rec_token
    assert pl.pair_expert.tolist() == pe and pl.pair_rec.tolist() == prc and np.array_equal(pl.ret_pos, ret)
    assert pl.bad == 2 and pl.ret_pos[1, 0] == -1 and pl.ret_pos[1, 1] == -1
    # a token whose three slots hit one rank travels once to it
    assert pl.rec_token[pl.records_to(1)].tolist().count(3) == 1


def test_plan_invariants_at_scale():
    T, k, E, P = 4096, 8, 64, 8
    idx = _routing(7, T, k, E)
    pl = oracle.ep_plan(idx, E, P)
    S = T * k
    assert pl.counts[P:].sum() == S
    assert sorted(pl.ret_pos.reshape(-1).tolist()) == list(range(S))       # a bijection onto the pairs
    epr = E // P
    for p in range(P):
        recs = pl.rec_token[pl.records_to(p)]
        assert np.all(np.diff(recs) > 0)                                      # one record per token, ascending
        want = np.unique(np.nonzero((idx // epr) == p)[0])
        assert np.array_equal(recs, want)
    for t, j in itertools.product(range(0, T, 97), range(k)):
        s = int(pl.ret_pos[t, j])
        p = int(idx[t, j]) // epr
        assert pl.pairs_to(p).start <= s < pl.pairs_to(p).stop
        assert pl.pair_expert[s] == idx[t, j] % epr
        assert pl.rec_token[pl.records_to(p).start + pl.pair_rec[s]] == t
    # dedup: fewer records than pairs whenever a token has two experts on one rank
    assert pl.counts[:P].sum() < S


def test_one_rank_reduces_to_the_local_plan():
    T, k, E = 300, 4, 16
    idx = _routing(11, T, k, E)
    pl = oracle.ep_plan(idx, E, 1)
    assert pl.counts.tolist() == [T, T * k] and pl.rec_token.tolist() == list(range(T))
    offs_l, perm_l, inv_l = oracle.moe_plan(idx, E)
    offs_r, perm_r, inv_r = oracle.moe_plan(pl.pair_expert[:, None], E)
    assert np.array_equal(offs_l, offs_r)
    # grouped row r holds the same token on both sides
    assert np.array_equal(perm_l, pl.rec_token[pl.pair_rec[perm_r]])
    assert np.array_equal(pl.ret_pos, np.arange(T * k).reshape(T, k))


def test_plan_rejects_uneven_splits():
    with pytest.raises(ValueError):
        oracle.ep_plan(np.zeros((2, 1), dtype=np.int32), 5, 2)


def _np_record(row_f64: np.ndarray) -> np.ndarray:
    """Independent record of one row: codes via np.log2 + ml_dtypes, scale bytes, zero pad."""
    C = row_f64.size
    b = row_f64.reshape(C // 32, 32)
    amax = np.abs(b).max(axis=1)
    with np.errstate(divide="ignore"):
        s = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 8, -127)
    s = np.clip(s, -127, 127).astype(np.int64)
    v = np.clip(np.ldexp(b, -s[:, None]), -448, 448)
    codes = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8).reshape(-1)
    out = np.zeros(oracle.ep_record_bytes(C), dtype=np.uint8)
    out[:C] = codes
    out[C:C + C // 32] = (s + 127).astype(np.uint8)
    return out


@pytest.mark.parametrize("C", [64, 96, 1408])
def test_records_equal_an_independent_block_quantiser(C):
    T = 40
    x = wl.normal_bf16((T, C), 1.0, 3)
    xs = x.clone()
    xs[5, 7] = 3e4                              # an outlier block
    xs[6] = 0                                   # an all-zero row
    xs[7, :32] = -0.0                           # signed zeros
    rec_token = np.array([0, 5, 6, 7, 39, 5, 12], dtype=np.int32)
    recs = oracle.ep_pack(xs, rec_token)
    assert recs.shape == (rec_token.size, oracle.ep_record_bytes(C)) and recs.shape[1] % 16 == 0
    xf = xs.to(torch.float64).numpy()
    for i, t in enumerate(rec_token):
        assert np.array_equal(recs[i], _np_record(xf[t])), (i, t)


def test_a_token_index_out_of_range_packs_a_zero_record():
    x = wl.normal_bf16((4, 64), 1.0, 4)
    recs = oracle.ep_pack(x, np.array([1, 4, -1], dtype=np.int32))
    assert recs[1:].max() == 0 and recs[0].max() > 0


def _exchange(plans, payloads_send, P):
    """Moves each source's blocks to their destination ranks, sources in rank order."""
    recv = []
    for r in range(P):
        recs = np.concatenate([payloads_send[q][0][plans[q].records_to(r)] for q in range(P)])
        pe = np.concatenate([plans[q].pair_expert[plans[q].pairs_to(r)] for q in range(P)])
        prc = np.concatenate([plans[q].pair_rec[plans[q].pairs_to(r)] for q in range(P)])
        counts = [plans[q].counts[r] for q in range(P)] + [plans[q].counts[P + r] for q in range(P)]
        recv.append((recs, pe, prc, counts))
    return recv


@pytest.mark.parametrize("P,T,k,E,C", [(2, 60, 3, 8, 64), (3, 50, 4, 12, 96), (4, 33, 8, 16, 128)])
def test_unpacked_rows_equal_the_local_quantisation(P, T, k, E, C):
    epr = E // P
    xs = [wl.normal_bf16((T, C), 1.0, 100 + q) for q in range(P)]
    idxs = [_routing(200 + q, T, k, E) for q in range(P)]
    plans = [oracle.ep_plan(idxs[q], E, P) for q in range(P)]
    send = [(oracle.ep_pack(xs[q], plans[q].rec_token),) for q in range(P)]
    recv = _exchange(plans, send, P)
    # local path: every source's tokens in rank order on one device
    X = torch.cat(xs)
    offs_g, perm_g, _ = oracle.moe_plan(np.concatenate(idxs), E)
    for r in range(P):
        recs, pe, prc, counts = recv[r]
        offs, perm, _ = oracle.moe_plan(pe[:, None], epr)
        q, sf = oracle.ep_unpack(recs, C, prc, oracle.ep_source_bases(counts), perm, offs)
        lo, hi = int(offs_g[r * epr]), int(offs_g[(r + 1) * epr])
        assert np.array_equal(offs, offs_g[r * epr:(r + 1) * epr + 1] - lo)
        rows = X[torch.from_numpy(perm_g[lo:hi].astype(np.int64))]
        q_ref, sf_ref = oracle.quantize_rowwise(rows, offs)
        nb = oracle.rowwise_scale_bytes(hi - lo, C, epr) if hi > lo else 0
        assert np.array_equal(q, q_ref)
        assert np.array_equal(sf[:nb], sf_ref[:nb])


def test_return_and_combine_equal_the_local_layer():
    """Expert outputs (the oracle's forward GEMM on the unpacked rows) go back
    along the pairs and are combined at ret_pos: the local layer's output."""
    P, T, k, E, C, N = 2, 40, 3, 8, 64, 32
    epr = E // P
    xs = [wl.normal_bf16((T, C), 1.0, 300 + q) for q in range(P)]
    idxs = [_routing(400 + q, T, k, E) for q in range(P)]
    ws = [np.random.default_rng(500 + q).random((T, k)).astype(np.float32) for q in range(P)]
    W = wl.normal_bf16((E * N, C), 0.05, 9)

    def experts(q_rows, sf_rows, offs, e0):
        """bf16 outputs of experts e0.. on grouped rows (the oracle's forward GEMM)."""
        wq, wsf = oracle.quantize_rowwise(W[e0 * N:(e0 + len(offs) - 1) * N])
        y = np.zeros((q_rows.shape[0], N))
        for _, lo, hi, Ye in oracle.fwd_by_expert(q_rows, sf_rows, wq, wsf, offs, N):
            y[lo:hi] = Ye
        return oracle.bf16_from_double(y)

    # local layer
    X = torch.cat(xs)
    idx_all = np.concatenate(idxs)
    offs_g, perm_g, inv_g = oracle.moe_plan(idx_all, E)
    qg, sg = oracle.quantize_rowwise(X[torch.from_numpy(perm_g.astype(np.int64))], offs_g)
    yp = experts(qg, sg, offs_g, 0)
    y_local = oracle.moe_combine(yp, inv_g, np.concatenate(ws))
    # through the exchange
    plans = [oracle.ep_plan(idxs[q], E, P) for q in range(P)]
    send = [(oracle.ep_pack(xs[q], plans[q].rec_token),) for q in range(P)]
    recv = _exchange(plans, send, P)
    back_parts = {q: [] for q in range(P)}
    for r in range(P):
        recs, pe, prc, counts = recv[r]
        offs, perm, inv = oracle.moe_plan(pe[:, None], epr)
        q_r, s_r = oracle.ep_unpack(recs, C, prc, oracle.ep_source_bases(counts), perm, offs)
        y_r = experts(q_r, s_r, offs, r * epr)
        y_ret = y_r[inv[:, 0]]                   # one row per received pair, in arrival order
        base = np.concatenate([[0], np.cumsum(counts[P:])])
        for q in range(P):
            back_parts[q].append(y_ret[base[q]:base[q + 1]])
    for q in range(P):
        y_back = np.concatenate(back_parts[q])
        y_q = oracle.moe_combine(y_back, plans[q].ret_pos, ws[q])
        assert np.array_equal(y_q, y_local[q * T:(q + 1) * T]), q
