"""GPU parity of the expert-parallel dispatch kernels (through the C ABI):
the send plan, the quantise-and-pack of token rows into MXFP8 records, the
receiver's unpack into the grouped rowwise layout and the return gather.

Several ranks are emulated on one GPU: every source plans and packs its own
tokens, the blocks of its send buffers are concatenated per destination in
source order (what the all-to-all delivers), and each receiver unpacks.  All
of it is integer or byte work, so every comparison is exact: against the
oracle, and against the local path (every rank's tokens on one device)."""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.helpers import np_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert m.mxfp8_device_supported(), "GPU tests need an sm_100 device"
    return m


def _routing(seed, T, k, E):
    rng = np.random.default_rng(seed)
    return np.argsort(-rng.standard_normal((T, E)), axis=1, kind="stable")[:, :k].astype(np.int32)


class Sent:
    """One source's plan and records (library kernels), with host counts."""

    def __init__(self, mx, x, idx, E, P):
        self.counts_d, rec_token, pair_expert, pair_rec, self.ret_pos, work = mx.mxfp8_ep_plan(
            torch.from_numpy(idx).cuda(), E, P)
        self.status = mx.mxfp8_get_status(work)
        self.counts = self.counts_d.cpu().tolist()
        self.P = P
        R, S = sum(self.counts[:P]), sum(self.counts[P:])
        self.rec_token, self.pair_expert, self.pair_rec = rec_token[:R], pair_expert[:S], pair_rec[:S]
        self.records = mx.mxfp8_ep_pack(x, self.rec_token) if x is not None else None

    def records_to(self, p):
        c = self.counts[:self.P]
        return slice(sum(c[:p]), sum(c[:p + 1]))

    def pairs_to(self, p):
        c = self.counts[self.P:]
        return slice(sum(c[:p]), sum(c[:p + 1]))


def _check_plan(mx, idx, E, P, expect_status=0):
    s = Sent(mx, None, idx, E, P)
    ref = oracle.ep_plan(idx, E, P)
    assert s.status == expect_status
    assert s.counts == ref.counts.tolist()
    np.testing.assert_array_equal(s.rec_token.cpu().numpy(), ref.rec_token)
    np.testing.assert_array_equal(s.pair_expert.cpu().numpy(), ref.pair_expert)
    np.testing.assert_array_equal(s.pair_rec.cpu().numpy(), ref.pair_rec)
    np.testing.assert_array_equal(s.ret_pos.cpu().numpy(), ref.ret_pos)


@pytest.mark.parametrize("seed,T,k,E,P", [(0, 9, 3, 8, 2), (1, 300, 4, 12, 3), (2, 1000, 8, 64, 8),
                                          (3, 77, 6, 12, 1), (4, 2048, 8, 256, 8), (5, 0, 4, 8, 2),
                                          (6, 33, 32, 64, 4), (7, 100, 1, 256, 256), (8, 16384, 8, 256, 8)])
def test_plan_matches_oracle(mx, seed, T, k, E, P):
    _check_plan(mx, _routing(seed, T, k, E), E, P)


def test_plan_with_repeated_experts_and_bad_ids(mx):
    idx = np.array([[5, 5, 1], [9, -1, 2], [0, 3, 3], [7, 7, 7]] * 20, dtype=np.int32)
    _check_plan(mx, idx, 8, 2, expect_status=7)      # MXF8_ERR_BAD_ROUTING; the valid slots still planned


def test_plan_rejects_bad_arguments(mx):
    idx = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    for E, P in ((5, 2), (8, 0), (512, 512)):
        with pytest.raises(mx.MXFP8Error):
            mx.mxfp8_ep_plan(idx, E, P)
    with pytest.raises(mx.MXFP8Error):
        mx.mxfp8_ep_plan(torch.zeros((4, 33), dtype=torch.int32, device="cuda"), 64, 2)


def _specials(x: torch.Tensor) -> torch.Tensor:
    x = x.clone()
    x[1, 3] = 3e4                    # an outlier block
    x[2] = 0                         # an all-zero row
    x[3, :32] = -0.0                 # signed zeros
    x[4, 32:64] = 1e-40              # bf16 subnormals
    x[5, 5] = 448 * 2 ** 10          # saturation boundary after scaling
    return x


@pytest.mark.parametrize("C", [64, 1408, 2048, 7168])
def test_pack_matches_oracle(mx, C):
    T = 300
    x = _specials(wl.normal_bf16((T, C), 1.0, C))
    rec_token = np.concatenate([np.arange(T), [T, -1, 7, 7]]).astype(np.int32)   # out-of-range tokens pack zeros
    recs = mx.mxfp8_ep_pack(x.cuda(), torch.from_numpy(rec_token).cuda())
    assert recs.shape == (rec_token.size, mx.mxfp8_ep_record_bytes(C)) == (rec_token.size, oracle.ep_record_bytes(C))
    np.testing.assert_array_equal(np_u8(recs), oracle.ep_pack(x, rec_token))


def _emulate(mx, xs, idxs, E, P):
    """Sources plan and pack; returns their Sent objects and, per receiver,
    (records, pair_expert, pair_rec, recv_counts) as the all-to-all delivers them."""
    sent = [Sent(mx, xs[q].cuda(), idxs[q], E, P) for q in range(P)]
    recv = []
    for r in range(P):
        recs = torch.cat([sent[q].records[sent[q].records_to(r)] for q in range(P)])
        pe = torch.cat([sent[q].pair_expert[sent[q].pairs_to(r)] for q in range(P)])
        prc = torch.cat([sent[q].pair_rec[sent[q].pairs_to(r)] for q in range(P)])
        rc = [sent[q].counts[r] for q in range(P)] + [sent[q].counts[P + r] for q in range(P)]
        recv.append((recs, pe, prc, rc))
    return sent, recv


def _receive(mx, recv_r, C, epr):
    from mxfp8_grouped_gemm_quantize_b200 import ep
    recs, pe, prc, rc = recv_r
    offs, perm, inv, work = mx.mxfp8_moe_plan(pe.view(-1, 1).contiguous(), epr)
    assert mx.mxfp8_get_status(work) == 0
    src_base = torch.tensor(ep.source_bases(rc), dtype=torch.int32, device="cuda")
    q, sf = mx.mxfp8_ep_unpack(recs, C, prc, src_base, perm, offs)
    return offs, perm, inv, q, sf


@pytest.mark.parametrize("P,T,k,E,C,check", [(2, 100, 3, 8, 64, "all"), (3, 200, 4, 12, 1408, "all"),
                                             (4, 500, 8, 32, 2048, "all"), (8, 2048, 8, 256, 7168, "ends")])
def test_unpacked_rows_equal_the_local_quantisation(mx, P, T, k, E, C, check):
    epr = E // P
    xs = [wl.with_outliers(wl.normal_bf16((T, C), 1.0, 50 + q), 1e-3, 100.0, 60 + q) for q in range(P)]
    idxs = [_routing(70 + q, T, k, E) for q in range(P)]
    sent, recv = _emulate(mx, xs, idxs, E, P)
    assert all(s.status == 0 for s in sent)
    X = torch.cat(xs).cuda()
    offs_g, perm_g, _, work = mx.mxfp8_moe_plan(torch.from_numpy(np.concatenate(idxs)).cuda(), E)
    assert mx.mxfp8_get_status(work) == 0
    og = offs_g.cpu().numpy()
    for r in (range(P) if check == "all" else (0, P - 1)):
        offs, perm, _, q, sf = _receive(mx, recv[r], C, epr)
        lo, hi = int(og[r * epr]), int(og[(r + 1) * epr])
        offs_loc = offs_g[r * epr:(r + 1) * epr + 1] - lo
        assert torch.equal(offs, offs_loc)
        # the local path: the library's rowwise quantiser on the rows this rank's experts get
        q_ref, sf_ref = mx.mxfp8_quantize_rowwise(X[perm_g[lo:hi].long()].contiguous(), offs_loc.contiguous())
        # defined scale bytes: the atoms of the groups' 128-row blocks (the rest of the bound is not written)
        rb = int(np.sum((np.diff(offs_loc.cpu().numpy()) + 127) // 128))
        defined = rb * ((C + 127) // 128) * 512
        assert torch.equal(q, q_ref)
        assert torch.equal(sf[:defined], sf_ref[:defined])
        # and the oracle's unpack of the same received buffers
        recs, pe, prc, rc = recv[r]
        from mxfp8_grouped_gemm_quantize_b200 import ep
        q_o, sf_o = oracle.ep_unpack(np_u8(recs), C, prc.cpu().numpy(), ep.source_bases(rc),
                                     perm.cpu().numpy(), offs.cpu().numpy())
        np.testing.assert_array_equal(np_u8(q), q_o)
        np.testing.assert_array_equal(np_u8(sf)[:defined], sf_o[:defined])


def test_gather_rows(mx):
    src = wl.normal_bf16((300, 136), 1.0, 5).cuda()
    idx = torch.tensor([5, 0, 299, 300, -1, 17, 17], dtype=torch.int32, device="cuda")
    out = mx.mxfp8_gather_rows(src, idx)
    want = torch.zeros((7, 136), dtype=torch.bfloat16, device="cuda")
    ok = (idx >= 0) & (idx < 300)
    want[ok] = src[idx[ok].long()]
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    with pytest.raises(mx.MXFP8Error):
        mx.mxfp8_gather_rows(wl.normal_bf16((4, 4), 1.0, 1).cuda(), idx)     # 8-byte rows


@pytest.mark.parametrize("P,T,k,E,K,N", [(2, 150, 3, 8, 256, 128), (4, 300, 6, 16, 512, 256)])
def test_emulated_layer_equals_the_local_layer(mx, P, T, k, E, K, N):
    """Dispatch, grouped GEMM on each rank's experts, return and combine give
    the local layer's output bit for bit."""
    epr = E // P
    xs = [wl.normal_bf16((T, K), 1.0, 80 + q) for q in range(P)]
    idxs = [_routing(90 + q, T, k, E) for q in range(P)]
    ws = [torch.from_numpy(np.random.default_rng(95 + q).random((T, k)).astype(np.float32)).cuda() for q in range(P)]
    W = wl.normal_bf16((E * N, K), 0.05, 99).cuda()
    # local layer
    X = torch.cat(xs).cuda()
    offs_g, perm_g, inv_g, _ = mx.mxfp8_moe_plan(torch.from_numpy(np.concatenate(idxs)).cuda(), E)
    xq, xsf, _, _ = mx.mxfp8_permute_quantize_dual(X, perm_g, offs_g)
    wq, wsf = mx.mxfp8_quantize_rowwise(W)
    y_g = mx.mxfp8_grouped_gemm_fwd(xq, xsf, wq, wsf, offs_g, N, work=mx.new_workspace(E, xq.shape[0], N, K))
    y_local = mx.mxfp8_moe_combine(y_g, inv_g, torch.cat(ws))
    # through the emulated exchange
    sent, recv = _emulate(mx, xs, idxs, E, P)
    back = {q: [] for q in range(P)}
    for r in range(P):
        offs, perm, inv, q, sf = _receive(mx, recv[r], K, epr)
        wq_r, wsf_r = mx.mxfp8_quantize_rowwise(W[r * epr * N:(r + 1) * epr * N].contiguous())
        y_r = mx.mxfp8_grouped_gemm_fwd(q, sf, wq_r, wsf_r, offs, N, work=mx.new_workspace(epr, q.shape[0], N, K))
        y_ret = mx.mxfp8_gather_rows(y_r, inv.view(-1).contiguous())
        pc = recv[r][3][P:]
        base = np.concatenate([[0], np.cumsum(pc)])
        for qq in range(P):
            back[qq].append(y_ret[int(base[qq]):int(base[qq + 1])])
    for qq in range(P):
        y_back = torch.cat(back[qq])
        y = mx.mxfp8_moe_combine(y_back, sent[qq].ret_pos, ws[qq])
        assert torch.equal(y.view(torch.int16), y_local[qq * T:(qq + 1) * T].view(torch.int16)), qq
