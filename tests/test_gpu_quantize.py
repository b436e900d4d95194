"""GPU parity of the MXFP8 quantisers against the CPU oracle: codes and
scale bytes bit-exact, through the C ABI (Python binding)."""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.helpers import np_u8, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert m.mxfp8_device_supported(), "GPU tests need an sm_100 device"
    return m


def _offs_dev(offs):
    return None if offs is None else torch.as_tensor(np.asarray(offs, dtype=np.int32)).cuda()


def check_rowwise(mx, x: torch.Tensor, offs=None):
    q, sf = mx.mxfp8_quantize_rowwise(x.cuda(), _offs_dev(offs))
    torch.cuda.synchronize()
    rq, rsf = oracle.quantize_rowwise(x, offs)
    np.testing.assert_array_equal(np_u8(q), rq)
    RB, _ = oracle.group_blocks(offs, x.shape[0])
    n = RB * oracle.rowwise_pitch(x.shape[1]) * 512
    np.testing.assert_array_equal(np_u8(sf)[:n], rsf[:n])


def check_colwise(mx, x: torch.Tensor, offs=None):
    R, C = x.shape
    qT, sf = mx.mxfp8_quantize_colwise(x.cuda(), _offs_dev(offs))
    torch.cuda.synchronize()
    rq, rsf = oracle.quantize_colwise(x, offs)
    RB, PG = oracle.group_blocks(offs, R)
    np.testing.assert_array_equal(np_u8(qT)[:, :PG], rq[:, :PG])
    pitch = oracle.colwise_pitch(R, 1 if offs is None else len(offs) - 1)
    gsf = np_u8(sf)
    for rb in range((C + 127) // 128):
        a = rb * pitch
        np.testing.assert_array_equal(gsf[a * 512:(a + RB) * 512], rsf[a * 512:(a + RB) * 512])


def _all_finite_bf16(order: str, seed=0) -> torch.Tensor:
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    b = b[((b >> 7) & 0xFF) != 0xFF]                    # 65280 finite patterns
    if order == "shuffled":
        b = np.random.default_rng(seed).permutation(b)
    b = b[: (b.size // 128) * 128]
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).reshape(-1, 128)


@pytest.mark.parametrize("order", ["sorted", "shuffled"])
def test_every_finite_bf16_pattern_rowwise(mx, order):
    check_rowwise(mx, _all_finite_bf16(order))


@pytest.mark.parametrize("order", ["sorted", "shuffled"])
def test_every_finite_bf16_pattern_colwise(mx, order):
    check_colwise(mx, _all_finite_bf16(order))


def test_scale_range_blocks(mx):
    """Blocks spanning every scale exponent: randn * 2^e, e in [-140, 120]."""
    rng = np.random.default_rng(3)
    R, C = 512, 256
    e = rng.integers(-140, 121, size=(R, C // 32))
    v = rng.standard_normal((R, C)) * np.repeat(2.0 ** e, 32, axis=1)
    x = torch.from_numpy(v).to(torch.bfloat16)
    check_rowwise(mx, x)
    check_colwise(mx, x)


def test_hand_worked_blocks_on_gpu(mx):
    from tests.test_oracle_scalars import _bf16_bits, _golden_blocks
    rows = []
    for _, _, pairs in _golden_blocks():
        vals = [v for v, _ in pairs] + [0.0] * (32 - len(pairs))
        rows.append(_bf16_bits(vals))
    rows += [np.zeros(32, np.uint16)] * (4 - len(rows) % 4)
    x = torch.from_numpy(np.stack(rows).reshape(-1, 128).view(np.int16).copy()).view(torch.bfloat16)
    check_rowwise(mx, x)


@pytest.mark.parametrize("seed", range(3))
def test_grouped_rowwise_and_colwise(mx, seed):
    counts = np.array([0, 1, 31, 32, 33, 127, 128, 129, 0, 300, 7], dtype=np.int64)
    counts = np.random.default_rng(seed).permutation(counts)
    offs = wl.offsets_from_counts(counts)
    x = wl.with_outliers(wl.normal_bf16((int(offs[-1]), 384), 1.0, seed), 0.01, 1000.0, seed)
    check_rowwise(mx, x, offs)
    check_colwise(mx, x, offs)


def test_tiny_config(mx):
    w = wl.tiny()
    X, W, dY = wl.layer_tensors(w, w.layers[0])
    for t, offs in ((X, w.offsets), (dY, w.offsets), (W.reshape(-1, W.shape[-1]), None)):
        check_rowwise(mx, t, offs)
        check_colwise(mx, t, offs)


def test_zero_and_single_rows(mx):
    check_rowwise(mx, torch.zeros((1, 32), dtype=torch.bfloat16))
    check_colwise(mx, torch.zeros((1, 32), dtype=torch.bfloat16))
    check_rowwise(mx, wl.normal_bf16((3, 96), 1.0, 1), [0, 0, 3, 3])
    check_colwise(mx, wl.normal_bf16((3, 96), 1.0, 1), [0, 0, 3, 3])


def test_nonfinite_block_gets_nan_scale(mx):
    x = torch.zeros((1, 64), dtype=torch.bfloat16)
    x[0, 3] = float("inf")
    x[0, 40] = float("nan")
    x[0, 41] = 1.0
    check_rowwise(mx, x)
    check_colwise(mx, x.reshape(64, 1).repeat(1, 32).contiguous())


def test_bad_arguments_are_rejected(mx):
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):
        mx.mxfp8_quantize_rowwise(x)
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):
        mx.mxfp8_quantize_rowwise(x, scales=torch.empty(16, dtype=torch.uint8, device="cuda"),
                                  offs=torch.tensor([0, 2, 4, 4, 4, 4], dtype=torch.int32, device="cuda"))


def test_invalid_offsets_stay_in_bounds(mx):
    """Offsets that are not a valid prefix are clamped: no write lands
    outside the output buffers (guard bytes stay intact)."""
    R, C = 200, 128
    x = wl.normal_bf16((R, C), 1.0, 5).cuda()
    for bad in ([0, 150, 100, 200], [5, 300, 400, 900], [-7, 10, -3, 200]):
        offs = torch.tensor(bad, dtype=torch.int32, device="cuda")
        G = len(bad) - 1
        guard = 4096
        q = torch.full((R * C + guard,), 0xA5, dtype=torch.uint8, device="cuda")
        n = mx.mxfp8_rowwise_scale_bytes(R, C, G)
        sf = torch.full((n + guard,), 0xA5, dtype=torch.uint8, device="cuda")
        mx.mxfp8_quantize_rowwise(x, offs, q=q[: R * C].view(R, C), scales=sf[:n])
        ld = mx.mxfp8_colwise_ld(R, G)
        qT = torch.full((C * ld + guard,), 0xA5, dtype=torch.uint8, device="cuda")
        n2 = mx.mxfp8_colwise_scale_bytes(R, C, G)
        sfT = torch.full((n2 + guard,), 0xA5, dtype=torch.uint8, device="cuda")
        mx.mxfp8_quantize_colwise(x, offs, qT=qT[: C * ld].view(C, ld), scales=sfT[:n2])
        torch.cuda.synchronize()
        for buf, end in ((q, R * C), (sf, n), (qT, C * ld), (sfT, n2)):
            assert torch.all(buf[end:] == 0xA5)


@pytest.mark.parametrize("M,K", [(4096, 2048), (16384, 5120), (65536, 7168)])
def test_sweep_full_size_sampled(mx, M, K):
    """Quantiser sweep sizes: all rows/columns quantised on the GPU; a seeded
    sample of rows (rowwise) and of 32-row blocks x 64 columns (colwise)
    checked against the oracle."""
    x = wl.sweep_tensor(M, K)
    xd = x.cuda()
    q, sf = mx.mxfp8_quantize_rowwise(xd)
    qT, sfT = mx.mxfp8_quantize_colwise(xd)
    torch.cuda.synchronize()
    rng = np.random.default_rng(M + K)
    rows = np.sort(rng.choice(M, size=256, replace=False))
    rq, rsf = oracle.quantize_rowwise(x[torch.from_numpy(rows)])
    np.testing.assert_array_equal(np_u8(q[torch.from_numpy(rows).cuda()]), rq)
    gsf = np_u8(sf)
    pitch = oracle.rowwise_pitch(K)
    for i, r in enumerate(rows[:64]):
        for j in range(K // 32):
            assert gsf[oracle.sf_offset(int(r), j, pitch)] == rsf[oracle.sf_offset(i, j, pitch)]
    gqT, gsfT = np_u8(qT), np_u8(sfT)
    cpitch = oracle.colwise_pitch(M, 1)
    cols = np.sort(rng.choice(K, size=64, replace=False))
    for b in rng.choice(M // 32, size=16, replace=False):
        sub = x[32 * b:32 * b + 32][:, torch.from_numpy(cols)].contiguous()
        oq, osf = oracle.quantize_colwise(sub)
        np.testing.assert_array_equal(gqT[cols, 32 * b:32 * b + 32], oq[:, :32])
        for i, c in enumerate(cols):
            assert gsfT[oracle.sf_offset(int(c), int(b), cpitch)] == osf[oracle.sf_offset(i, 0, oracle.colwise_pitch(32, 1))]


@pytest.mark.parametrize("name", ["ds-v3-16b", "ds-v3-671b", "llama4-scout"])
def test_grouped_full_size_sampled_groups(mx, name):
    """Workload sizes with their real routing: whole groups sampled and
    quantised by the oracle as single groups; rowwise and colwise codes and
    scales must match the GPU's group-relative layout."""
    w = wl.WORKLOADS[name]()
    layer = w.layers[0]
    X, _, _ = wl.layer_tensors(w, layer)
    offs = w.offsets
    od = torch.from_numpy(offs).cuda()
    xd = X.cuda()
    q, sf = mx.mxfp8_quantize_rowwise(xd, od)
    qT, sfT = mx.mxfp8_quantize_colwise(xd, od)
    torch.cuda.synchronize()
    gq, gsf, gqT, gsfT = np_u8(q), np_u8(sf), np_u8(qT), np_u8(sfT)
    K = X.shape[1]
    E = w.E
    counts = np.diff(offs.astype(np.int64))
    RB = np.concatenate([[0], np.cumsum((counts + 127) // 128)])
    P = np.concatenate([[0], np.cumsum((counts + 31) // 32 * 32)])
    rpitch, cpitch = oracle.rowwise_pitch(K), oracle.colwise_pitch(w.M, E)
    rng = np.random.default_rng(11)
    for g in rng.choice(np.nonzero(counts)[0], size=2, replace=False):
        lo, hi, m = int(offs[g]), int(offs[g + 1]), int(counts[g])
        sub = X[lo:hi].contiguous()
        oq, osf = oracle.quantize_rowwise(sub)
        np.testing.assert_array_equal(gq[lo:hi], oq)
        for t in range(0, m, max(1, m // 17)):
            for j in range(0, K // 32, 7):
                assert gsf[oracle.sf_offset(128 * int(RB[g]) + t, j, rpitch)] == osf[oracle.sf_offset(t, j, rpitch)]
        oqT, osfT = oracle.quantize_colwise(sub)
        np.testing.assert_array_equal(gqT[:, P[g]:P[g] + (m + 31) // 32 * 32], oqT[:, :(m + 31) // 32 * 32])
        sp = oracle.colwise_pitch(m, 1)
        for c in range(0, K, 97):
            for j in range((m + 31) // 32):
                assert gsfT[oracle.sf_offset(c, 4 * int(RB[g]) + j, cpitch)] == osfT[oracle.sf_offset(c, j, sp)]


# ------------------------------------------------------------------ dual (rowwise + colwise from one read)
def check_dual(mx, x: torch.Tensor, offs=None):
    R, C = x.shape
    q, sf, qT, sfT = mx.mxfp8_quantize_dual(x.cuda(), _offs_dev(offs))
    torch.cuda.synchronize()
    rq, rsf = oracle.quantize_rowwise(x, offs)
    cq, csf = oracle.quantize_colwise(x, offs)
    RB, PG = oracle.group_blocks(offs, R)
    np.testing.assert_array_equal(np_u8(q), rq)
    n = RB * oracle.rowwise_pitch(C) * 512
    np.testing.assert_array_equal(np_u8(sf)[:n], rsf[:n])
    np.testing.assert_array_equal(np_u8(qT)[:, :PG], cq[:, :PG])
    pitch = oracle.colwise_pitch(R, 1 if offs is None else len(offs) - 1)
    g = np_u8(sfT)
    for rb in range((C + 127) // 128):
        a = rb * pitch
        np.testing.assert_array_equal(g[a * 512:(a + RB) * 512], csf[a * 512:(a + RB) * 512])


@pytest.mark.parametrize("order", ["sorted", "shuffled"])
def test_dual_every_finite_bf16_pattern(mx, order):
    check_dual(mx, _all_finite_bf16(order))


@pytest.mark.parametrize("seed", range(3))
def test_dual_grouped(mx, seed):
    counts = np.array([0, 1, 31, 32, 33, 127, 128, 129, 0, 300, 7], dtype=np.int64)
    counts = np.random.default_rng(seed + 10).permutation(counts)
    offs = wl.offsets_from_counts(counts)
    x = wl.with_outliers(wl.normal_bf16((int(offs[-1]), 416), 1.0, seed + 20), 0.01, 1000.0, seed)
    check_dual(mx, x, offs)


def test_dual_tiny_and_edges(mx):
    w = wl.tiny()
    X, W, dY = wl.layer_tensors(w, w.layers[0])
    check_dual(mx, X, w.offsets)
    check_dual(mx, W.reshape(-1, W.shape[-1]))
    check_dual(mx, torch.zeros((1, 32), dtype=torch.bfloat16))
    check_dual(mx, wl.normal_bf16((3, 96), 1.0, 1), [0, 0, 3, 3])


def test_dual_matches_separate_at_workload_size(mx):
    """DeepSeek-V3-16B-like X (49152 x 2048, 64 groups): dual output equals
    the separate rowwise and colwise kernels' output byte for byte."""
    w = wl.ds_v3_16b()
    X, _, _ = wl.layer_tensors(w, w.layers[0], device="cuda")
    od = torch.from_numpy(w.offsets).cuda()
    q, sf, qT, sfT = mx.mxfp8_quantize_dual(X, od)
    q2, sf2 = mx.mxfp8_quantize_rowwise(X, od)
    qT2, sfT2 = mx.mxfp8_quantize_colwise(X, od)
    torch.cuda.synchronize()
    RB, PG = oracle.group_blocks(w.offsets, w.M)
    assert torch.equal(q, q2)
    n = RB * oracle.rowwise_pitch(X.shape[1]) * 512
    assert torch.equal(sf[:n], sf2[:n])
    assert torch.equal(qT[:, :PG], qT2[:, :PG])
    pitch = oracle.colwise_pitch(w.M, w.E)
    for rb in range(X.shape[1] // 128):
        a = rb * pitch
        assert torch.equal(sfT[a * 512:(a + RB) * 512], sfT2[a * 512:(a + RB) * 512])


@pytest.mark.parametrize("kind", ["inf", "nan"])
def test_nonfinite_in_a_short_last_colwise_block(mx, kind):
    """A non-finite value in a group's short last 32-row block: the block
    gets the NaN scale and NaN codes on its real rows, while the pad columns
    up to the group's 32-padded end stay 0x00 (colwise and dual)."""
    counts = [70, 0, 150, 33]
    offs = wl.offsets_from_counts(counts)
    x = wl.normal_bf16((int(offs[-1]), 96), 1.0, 4)
    bad = float("inf") if kind == "inf" else float("nan")
    for r, c in ((200, 5), (3, 40), (252, 95)):   # group 2 block 4 (22 rows), a full block, group 3 block 1 (1 row)
        x[r, c] = bad
    check_colwise(mx, x, offs)
    check_dual(mx, x, offs)
