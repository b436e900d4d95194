"""GPU parity of the MoE dispatch plan, the permute fused with dual MXFP8
quantisation, and the weighted combine (through the C ABI).

All three are exact: the plan is integer work (offsets, permutation and its
inverse equal the oracle's), the fused permute-quantise must equal the
oracle's quantisation of the gathered rows byte for byte, and the combine
is the fp64 sum rounded once to bf16, so it equals the oracle bit for bit."""
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


def _routing(rng, T, k, E, skew=0.0):
    logits = rng.standard_normal((T, E)) - skew * np.log1p(np.arange(E))[None, :]
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :k].astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    return idx, w


def _plan(mx, idx, E):
    offs, perm, inv, work = mx.mxfp8_moe_plan(torch.from_numpy(idx).cuda(), E)
    assert mx.mxfp8_get_status(work) == 0
    return offs, perm, inv


def check_plan(mx, idx, E):
    offs, perm, inv = _plan(mx, idx, E)
    ro, rp, ri = oracle.moe_plan(idx, E)
    np.testing.assert_array_equal(offs.cpu().numpy(), ro)
    np.testing.assert_array_equal(perm.cpu().numpy(), rp)
    np.testing.assert_array_equal(inv.cpu().numpy(), ri)
    return offs, perm, inv


CASES = [(1, 1, 1, 0.0), (40, 2, 5, 0.0), (1000, 6, 64, 0.0), (1500, 8, 32, 2.0), (3000, 1, 16, 0.0),
         (777, 4, 256, 1.0), (2049, 3, 7, 3.0)]


@pytest.mark.parametrize("T,k,E,skew", CASES)
def test_plan_matches_oracle(mx, T, k, E, skew):
    idx, _ = _routing(np.random.default_rng(T + 13 * k), T, k, E, skew)
    check_plan(mx, idx, E)


def test_plan_many_chunks_and_empty_experts(mx):
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 100, size=(20000, 5)).astype(np.int32)   # experts 100..199 stay empty
    check_plan(mx, idx, 200)


def test_plan_no_tokens(mx):
    offs, perm, inv = _plan(mx, np.zeros((0, 4), dtype=np.int32), 8)
    assert offs.cpu().numpy().tolist() == [0] * 9 and perm.numel() == 0


def test_plan_reports_bad_expert_ids(mx):
    idx = np.array([[0, 1], [2, 9], [1, -3]], dtype=np.int32)
    offs, perm, inv, work = mx.mxfp8_moe_plan(torch.from_numpy(idx).cuda(), 3)
    assert mx.mxfp8_get_status(work) == 7
    inv = inv.cpu().numpy()
    assert inv[1, 1] == -1 and inv[2, 1] == -1
    # the valid pairs still get a consistent plan
    o = offs.cpu().numpy()
    assert o.tolist() == [0, 1, 3, 4]
    assert sorted(inv[inv >= 0].tolist()) == [0, 1, 2, 3]


def test_plan_rejects_bad_arguments(mx):
    idx = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):
        mx.mxfp8_moe_plan(idx, 0)
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):
        mx.mxfp8_moe_plan(idx, 257)


def check_permute_quantize(mx, x, idx, E):
    offs, perm, inv = _plan(mx, idx, E)
    xd = x.cuda()
    q, s, qT, sT = mx.mxfp8_permute_quantize_dual(xd, perm, offs)
    torch.cuda.synchronize()
    o = offs.cpu().numpy()
    xp = x[torch.from_numpy(perm.cpu().numpy().astype(np.int64))]
    rq, rs = oracle.quantize_rowwise(xp, o)
    np.testing.assert_array_equal(np_u8(q), rq)
    R, C = xp.shape
    RB, PG = oracle.group_blocks(o, R)
    n = RB * oracle.rowwise_pitch(C) * 512
    np.testing.assert_array_equal(np_u8(s)[:n], rs[:n])
    cq, cs = oracle.quantize_colwise(xp, o)
    np.testing.assert_array_equal(np_u8(qT)[:, :PG], cq[:, :PG])
    pitch = oracle.colwise_pitch(R, E)
    g = np_u8(sT)
    for rb in range((C + 127) // 128):
        a = rb * pitch
        np.testing.assert_array_equal(g[a * 512:(a + RB) * 512], cs[a * 512:(a + RB) * 512])
    return offs, perm, inv, (q, s, qT, sT)


@pytest.mark.parametrize("T,k,E,C", [(40, 2, 5, 256), (300, 6, 16, 160), (1000, 8, 32, 512), (513, 1, 3, 96)])
def test_permute_quantize_matches_oracle(mx, T, k, E, C):
    rng = np.random.default_rng(T * 7 + C)
    idx, _ = _routing(rng, T, k, E, 1.0)
    x = wl.normal_bf16((T, C), 1.0, T + C)
    check_permute_quantize(mx, x, idx, E)


def test_permute_quantize_equals_dual_on_gathered_rows(mx):
    """Whole buffers, sentinel-filled: the fused kernel writes exactly what
    the dual quantiser writes for the gathered matrix."""
    r = wl.routing("tiny")
    x = wl.normal_bf16((r.T, r.K), 1.0, 5).cuda()
    offs, perm, inv = _plan(mx, r.idx, r.E)
    R, C = perm.numel(), r.K

    def bufs():
        ld = mx.mxfp8_colwise_ld(R, r.E)
        f = lambda *sh: torch.full(sh, 0xA5, dtype=torch.uint8, device="cuda")  # noqa: E731
        return (f(R, C), f(mx.mxfp8_rowwise_scale_bytes(R, C, r.E)), f(C, ld), f(mx.mxfp8_colwise_scale_bytes(R, C, r.E)))

    a, b = bufs(), bufs()
    mx.mxfp8_permute_quantize_dual(x, perm, offs, *a)
    mx.mxfp8_quantize_dual(x[perm.long()].contiguous(), offs, *b)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_permute_out_of_range_index_reads_zero_row(mx):
    x = wl.normal_bf16((10, 64), 1.0, 2).cuda()
    perm = torch.tensor([0, 99, 3, -1], dtype=torch.int32, device="cuda")
    offs = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    q, s, qT, sT = mx.mxfp8_permute_quantize_dual(x, perm, offs)
    torch.cuda.synchronize()
    qn = np_u8(q)
    assert np.all(qn[1] == 0) and np.all(qn[3] == 0)
    np.testing.assert_array_equal(qn[[0, 2]], oracle.quantize_rowwise(x.cpu()[[0, 3]])[0])


@pytest.mark.parametrize("T,k,E,C", [(40, 2, 5, 64), (500, 6, 64, 136), (1000, 8, 32, 256), (300, 1, 4, 8),
                                     (100, 10, 16, 64)])
def test_combine_matches_oracle(mx, T, k, E, C):
    rng = np.random.default_rng(T + k + C)
    idx, w = _routing(rng, T, k, E)
    offs, perm, inv = _plan(mx, idx, E)
    yp = wl.normal_bf16((T * k, C), 1.0, T + C)
    y = mx.mxfp8_moe_combine(yp.cuda(), inv, torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    ref = oracle.moe_combine(yp, inv.cpu().numpy(), w)
    np.testing.assert_array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref)


def test_combine_extreme_values_round_like_the_oracle(mx):
    """Sums near the bf16 overflow threshold, in the subnormal range and with
    exact ties exercise every branch of the rounding."""
    rng = np.random.default_rng(21)
    T, k, C = 64, 2, 64
    idx = np.stack([np.zeros(T, np.int32), np.ones(T, np.int32)], axis=1)
    w = np.ones((T, k), dtype=np.float32)
    mags = 2.0 ** rng.integers(-140, 121, size=(T * k, 1))       # finite bf16 inputs (no NaN from Inf - Inf)
    yp = torch.from_numpy(rng.standard_normal((T * k, C)) * mags).to(torch.bfloat16)
    yp[0, :] = torch.tensor(3.3e38).to(torch.bfloat16)          # two of these overflow
    yp[1, :] = torch.tensor(2.0 ** -133).to(torch.bfloat16)      # smallest subnormal
    offs, perm, inv = _plan(mx, idx, 2)
    inv[0, 1] = 0                                               # token 0 adds row 0 twice
    y = mx.mxfp8_moe_combine(yp.cuda(), inv, torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    ref = oracle.moe_combine(yp, inv.cpu().numpy(), w)
    np.testing.assert_array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref)


def test_full_size_dispatch_ds_v3_16b(mx):
    """The DeepSeek-V3-16B-like routing at full size: plan equals the
    oracle's, the fused permute-quantise equals the dual quantiser on the
    gathered rows (whole buffers), the combine equals the oracle's on a
    seeded sample of tokens."""
    r = wl.routing("ds-v3-16b")
    offs, perm, inv = check_plan(mx, r.idx, r.E)
    x = wl.normal_bf16((r.T, r.K), 1.0, 7).cuda()
    a = mx.mxfp8_permute_quantize_dual(x, perm, offs)
    b = mx.mxfp8_quantize_dual(x[perm.long()].contiguous(), offs)
    torch.cuda.synchronize()
    R, C = perm.numel(), r.K
    RB, PG = oracle.group_blocks(offs.cpu().numpy(), R)
    assert torch.equal(a[0], b[0]) and torch.equal(a[2][:, :PG], b[2][:, :PG])
    n = RB * oracle.rowwise_pitch(C) * 512
    assert torch.equal(a[1][:n], b[1][:n])
    yp = wl.normal_bf16((R, 2048), 1.0, 8)
    y = mx.mxfp8_moe_combine(yp.cuda(), inv, torch.from_numpy(r.w).cuda())
    torch.cuda.synchronize()
    toks = np.random.default_rng(4).choice(r.T, 256, replace=False)
    inv_np = inv.cpu().numpy()
    ref = oracle.moe_combine(yp, inv_np[toks], r.w[toks])
    np.testing.assert_array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16)[toks], ref)


def test_combine_nan_where_the_sum_is_undefined(mx):
    """Inf + (-Inf) and NaN inputs give a NaN output (a generated NaN's sign is
    not fixed by the definition, so only NaN-ness is compared there); every
    other element stays bit-exact."""
    T, k, C = 8, 2, 64
    idx = np.stack([np.zeros(T, np.int32), np.ones(T, np.int32)], axis=1)
    w = np.ones((T, k), dtype=np.float32)
    yp = wl.normal_bf16((T * k, C), 1.0, 31)
    offs, perm, inv = _plan(mx, idx, 2)
    inv_np = inv.cpu().numpy()
    yp[inv_np[0, 0], :8] = float("inf")
    yp[inv_np[0, 1], :8] = float("-inf")
    yp[inv_np[1, 0], 8:16] = float("nan")
    y = mx.mxfp8_moe_combine(yp.cuda(), inv, torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = oracle.moe_combine(yp, inv_np, w)
    nan = lambda a: ((a & 0x7F80) == 0x7F80) & ((a & 0x007F) != 0)  # noqa: E731
    assert nan(ref[0, :8]).all() and nan(got[0, :8]).all()
    assert nan(ref[1, 8:16]).all() and nan(got[1, 8:16]).all()
    mask = ~nan(ref)
    np.testing.assert_array_equal(got[mask], ref[mask])
