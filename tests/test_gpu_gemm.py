"""GPU parity of the grouped GEMMs (fwd, dgrad, wgrad) against the fp64
oracle on identical quantised inputs, through the C ABI (Python binding).

Tolerance (tests/helpers.py): normalised Frobenius error <= 5e-3 and
per-element relative error <= 2e-2 where |ref| > 1e-2 * rms(ref); an expert
with no rows must give exactly zero dW.  With small-integer operands every
product sum is an integer below 2^24, exact in fp32, so the bf16 outputs
must equal the rounded exact result bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.helpers import assert_gemm_close, bf16_round, f64, np_u8

pytestmark = pytest.mark.gpu

POISON = 0x7FC0  # bf16 NaN: any output element the kernel fails to write stays NaN


@pytest.fixture(params=["default", "1cta-ks1", "1cta-ks2", "pair-ks1", "pair-ks2"])
def tile_config(request):
    """Runs a test under the per-pass default tile configuration and under
    each forced one: 1-CTA 128x256 or CTA-pair 256x256 tiles, with 128-deep
    (ks1) or 256-deep (ks2) pipeline stages."""
    import mxfp8_grouped_gemm_quantize_b200 as m
    if request.param == "default":
        m.mxfp8_set_gemm_tiling(-1, -1)
    else:
        tiles, ks = request.param.split("-")
        m.mxfp8_set_gemm_tiling(1 if tiles == "pair" else 0, int(ks[-1]))
    yield request.param
    m.mxfp8_set_gemm_tiling(-1, -1)


@pytest.fixture(scope="module")
def mx():
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert m.mxfp8_device_supported(), "GPU tests need an sm_100 device"
    return m


def poisoned(shape, guard=2048):
    """bf16 output buffer filled with NaN plus a NaN guard tail."""
    n = int(np.prod(shape))
    buf = torch.full((n + guard,), POISON, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    return buf, buf[:n].view(*shape)


def guard_intact(buf, n):
    return bool(torch.all(buf[n:].view(torch.int16) == POISON))


class Case:
    """Quantises X, W, dY on the GPU for one grouped linear and keeps the
    bytes; checks them bit-exact against the oracle's quantisation."""

    def __init__(self, mx, X, W, dY, offs, check_quant=True):
        self.mx = mx
        self.X, self.W, self.dY = X, W, dY
        self.offs = np.asarray(offs, dtype=np.int32)
        self.E, self.N, self.K = W.shape
        self.M = X.shape[0]
        od = torch.from_numpy(self.offs).cuda()
        self.od = od
        Xd, Wd, dYd = X.cuda(), W.reshape(self.E * self.N, self.K).cuda(), dY.cuda()
        self.xq, self.xs = mx.mxfp8_quantize_rowwise(Xd, od)
        self.wq, self.ws = mx.mxfp8_quantize_rowwise(Wd)
        self.dyq, self.dys = mx.mxfp8_quantize_rowwise(dYd, od)
        self.wqT, self.wsT = mx.mxfp8_quantize_colwise(Wd)
        self.dyqT, self.dysT = mx.mxfp8_quantize_colwise(dYd, od)
        self.xqT, self.xsT = mx.mxfp8_quantize_colwise(Xd, od)
        torch.cuda.synchronize()
        if check_quant:
            np.testing.assert_array_equal(np_u8(self.xq), oracle.quantize_rowwise(X, self.offs)[0])
            np.testing.assert_array_equal(np_u8(self.dyq), oracle.quantize_rowwise(dY, self.offs)[0])
            np.testing.assert_array_equal(np_u8(self.wq), oracle.quantize_rowwise(W.reshape(-1, self.K))[0])
            _, PG = oracle.group_blocks(self.offs, self.M)
            np.testing.assert_array_equal(np_u8(self.xqT)[:, :PG], oracle.quantize_colwise(X, self.offs)[0][:, :PG])

    # dequantised operands (oracle, from the GPU's bytes)
    def deq(self):
        offs = self.offs
        Xd = oracle.dequantize_rowwise(np_u8(self.xq), np_u8(self.xs), offs)
        Wd = oracle.dequantize_rowwise(np_u8(self.wq), np_u8(self.ws)).reshape(self.E, self.N, self.K)
        dYd = oracle.dequantize_rowwise(np_u8(self.dyq), np_u8(self.dys), offs)
        WdT = oracle.dequantize_colwise(np_u8(self.wqT), np_u8(self.wsT), self.E * self.N).reshape(self.E, self.N, self.K)
        dYc = oracle.dequantize_colwise(np_u8(self.dyqT), np_u8(self.dysT), self.M, offs)
        Xc = oracle.dequantize_colwise(np_u8(self.xqT), np_u8(self.xsT), self.M, offs)
        return Xd, Wd, dYd, WdT, dYc, Xc

    def fwd(self, out=None):
        return self.mx.mxfp8_grouped_gemm_fwd(self.xq, self.xs, self.wq, self.ws, self.od, self.N, out=out)

    def dgrad(self, out=None):
        return self.mx.mxfp8_grouped_gemm_dgrad(self.dyq, self.dys, self.wqT, self.wsT, self.od, self.K, out=out)

    def wgrad(self, out=None):
        return self.mx.mxfp8_grouped_gemm_wgrad(self.dyqT, self.dysT, self.xqT, self.xsT, self.od, self.M, out=out)


def run_all_and_compare(c: Case, exact=False):
    M, N, K, E = c.M, c.N, c.K, c.E
    by, y = poisoned((M, N))
    bdx, dx = poisoned((M, K))
    bdw, dw = poisoned((E, N, K))
    c.fwd(y); c.dgrad(dx); c.wgrad(dw)
    torch.cuda.synchronize()
    assert guard_intact(by, M * N) and guard_intact(bdx, M * K) and guard_intact(bdw, E * N * K)
    Xd, Wd, dYd, WdT, dYc, Xc = c.deq()
    ref_y = oracle.gemm_fwd(Xd, Wd, c.offs)
    ref_dx = oracle.gemm_dgrad(dYd, WdT, c.offs)
    ref_dw = oracle.gemm_wgrad(dYc, Xc, c.offs)
    gy, gdx, gdw = f64(y), f64(dx), f64(dw)
    if exact:
        np.testing.assert_array_equal(gy, bf16_round(ref_y))
        np.testing.assert_array_equal(gdx, bf16_round(ref_dx))
        np.testing.assert_array_equal(gdw, bf16_round(ref_dw))
    else:
        assert_gemm_close(gy, ref_y, "fwd")
        assert_gemm_close(gdx, ref_dx, "dgrad")
        for e in range(E):
            assert_gemm_close(gdw[e], ref_dw[e], f"wgrad expert {e}")
    counts = np.diff(c.offs.astype(np.int64))
    for e in np.nonzero(counts == 0)[0]:
        assert np.all(gdw[e] == 0.0)
    return gy, gdx, gdw


def make_case(mx, counts, N, K, seed=0, w_std=1.0, check_quant=True):
    offs = wl.offsets_from_counts(counts)
    M, E = int(offs[-1]), len(counts)
    X = wl.normal_bf16((M, K), 1.0, seed + 1)
    W = wl.normal_bf16((E, N, K), w_std, seed + 2)
    dY = wl.normal_bf16((M, N), 1.0, seed + 3)
    return Case(mx, X, W, dY, offs, check_quant)


def test_tiny_config(mx, tile_config):
    w = wl.tiny()
    X, W, dY = wl.layer_tensors(w, w.layers[0])
    run_all_and_compare(Case(mx, X, W, dY, w.offsets))


@pytest.mark.parametrize("seed", range(3))
def test_tiny_random_counts(mx, seed):
    run_all_and_compare(make_case(mx, wl.tiny_random(seed), 128, 256, seed))


def test_ragged_multi_tile(mx, tile_config):
    """Several 128x256 tiles per group, ragged tails, an empty expert, a
    partial output tile (N = 384) and a partial K block (K = 416)."""
    run_all_and_compare(make_case(mx, [0, 1, 129, 300, 77, 255], 384, 416, seed=7))


def test_small_integer_operands_exact(mx, tile_config):
    counts = [0, 7, 21, 36, 200, 1, 130]
    offs = wl.offsets_from_counts(counts)
    M, E, N, K = int(offs[-1]), len(counts), 256, 512
    X = wl.integer_bf16((M, K), -14, 14, 1)
    W = wl.integer_bf16((E, N, K), -14, 14, 2)
    dY = wl.integer_bf16((M, N), -14, 14, 3)
    run_all_and_compare(Case(mx, X, W, dY, offs), exact=True)


def test_ragged_tails_of_every_pair_shape_exact(mx, tile_config):
    """CTA pairs compute a group's last r < 256 rows as a swapped tile of
    round_up(r, 32) tokens; tails r = 31, 32, 33, 64, ..., 224, 225, 255 (and
    groups of exactly 256) cover every token-chunk count, both rounding cases
    and tails behind full 256-row blocks.  Integer operands make every pass
    exact; N = 640 leaves half of the last output-column block empty."""
    counts = [32, 64 + 256, 96, 128, 160 + 512, 192, 224, 31, 33, 225, 255, 256]
    offs = wl.offsets_from_counts(counts)
    M, E, N, K = int(offs[-1]), len(counts), 640, 256
    X = wl.integer_bf16((M, K), -14, 14, 11)
    W = wl.integer_bf16((E, N, K), -14, 14, 12)
    dY = wl.integer_bf16((M, N), -14, 14, 13)
    run_all_and_compare(Case(mx, X, W, dY, offs), exact=True)


def test_distinct_block_scales_pin_the_scale_layout(mx, tile_config):
    """Every 32-block gets its own power-of-two magnitude, so a scale read
    from the wrong row or block breaks parity."""
    counts = [50, 0, 170, 33]
    offs = wl.offsets_from_counts(counts)
    M, E, N, K = int(offs[-1]), len(counts), 256, 384
    rng = np.random.default_rng(5)

    def blocky(shape, axis_len):
        v = rng.standard_normal(shape)
        e = rng.integers(-6, 7, size=shape[:-1] + (shape[-1] // 32,))
        v = v * np.repeat(2.0 ** e, 32, axis=-1)
        return torch.from_numpy(v).to(torch.bfloat16)

    X = blocky((M, K), K)
    W = blocky((E, N, K), K)
    dY = blocky((M, N), N)
    run_all_and_compare(Case(mx, X, W, dY, offs))


@pytest.mark.parametrize("counts,N,K", [([1], 128, 32), ([0, 0, 5], 128, 64), ([300], 128, 160),
                                        ([3, 0, 0, 0], 256, 1024), ([129, 127], 512, 96),
                                        ([40, 0, 260], 384, 544), ([256, 512, 3], 256, 128)])
def test_edge_shapes(mx, tile_config, counts, N, K):
    run_all_and_compare(make_case(mx, counts, N, K, seed=sum(counts)))


def test_all_rows_in_one_expert(mx, tile_config):
    run_all_and_compare(make_case(mx, [0, 0, 400, 0], 256, 256, seed=3))


def test_zero_rows(mx, tile_config):
    """M = 0: fwd/dgrad have nothing to write; wgrad writes dW = 0."""
    c = make_case(mx, [0, 0], 128, 64, check_quant=False)
    bdw, dw = poisoned((2, 128, 64))
    c.wgrad(dw)
    y = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    assert torch.all(dw.float() == 0) and guard_intact(bdw, 2 * 128 * 64)


def test_bad_offsets_are_reported_and_nothing_is_written(mx):
    c = make_case(mx, [10, 20, 30], 128, 64, check_quant=False)
    for bad in ([0, 20, 10, 60], [1, 10, 30, 60], [0, 10, 30, 59]):
        od = torch.tensor(bad, dtype=torch.int32, device="cuda")
        work = mx.new_workspace(3, 60, 128, 64)
        by, y = poisoned((60, 128))
        mx.mxfp8_grouped_gemm_fwd(c.xq, c.xs, c.wq, c.ws, od, 128, out=y, work=work)
        assert mx.mxfp8_get_status(work) == 5
        assert torch.all(by.view(torch.int16) == POISON)
    work = mx.new_workspace(3, 60, 128, 64)
    c.mx.mxfp8_grouped_gemm_fwd(c.xq, c.xs, c.wq, c.ws, c.od, 128, work=work)
    assert mx.mxfp8_get_status(work) == 0


def test_bad_gemm_arguments_are_rejected(mx):
    c = make_case(mx, [10, 20], 128, 64, check_quant=False)
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):
        mx.mxfp8_grouped_gemm_fwd(c.xq, c.xs, c.wq, c.ws, c.od, 96)        # N % 128 != 0
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):
        mx.mxfp8_grouped_gemm_fwd(c.xq, c.xs[:16], c.wq, c.ws, c.od, 128)  # scale buffer too small


def _sampled_check(c: Case, rng, ns=384):
    M, N, K, E = c.M, c.N, c.K, c.E
    y = c.fwd(); dx = c.dgrad(); dw = c.wgrad()
    torch.cuda.synchronize()
    gy, gdx, gdw = f64(y), f64(dx), f64(dw)
    assert np.all(np.isfinite(gy)) and np.all(np.isfinite(gdx)) and np.all(np.isfinite(gdw))
    r = rng.integers(0, M, ns); cn = rng.integers(0, N, ns); ck = rng.integers(0, K, ns)
    ref = oracle.sample_fwd(np_u8(c.xq), np_u8(c.xs), np_u8(c.wq), np_u8(c.ws), c.offs, N, r, cn)
    assert_gemm_close(gy[r, cn], ref, "fwd (sampled)")
    ref = oracle.sample_dgrad(np_u8(c.dyq), np_u8(c.dys), np_u8(c.wqT), np_u8(c.wsT), c.offs, K, r, ck)
    assert_gemm_close(gdx[r, ck], ref, "dgrad (sampled)")
    ex = rng.integers(0, E, ns)
    ref = oracle.sample_wgrad(np_u8(c.dyqT), np_u8(c.dysT), np_u8(c.xqT), np_u8(c.xsT), c.offs, M, N, K, ex, cn, ck)
    assert_gemm_close(gdw[ex, cn, ck], ref, "wgrad (sampled)")


@pytest.mark.parametrize("name", ["ds-v3-16b", "ds-v3-671b", "llama4-scout"])
def test_workload_full_size_sampled(mx, name):
    """Full workload sizes and routing, in the launch configuration the
    benchmark times: every output computed on the GPU, a seeded sample of
    each checked against the oracle's dot products on the same bytes."""
    w = wl.WORKLOADS[name]()
    rng = np.random.default_rng(17)
    for layer in w.layers:
        X, W, dY = wl.layer_tensors(w, layer)
        _sampled_check(Case(mx, X, W, dY, w.offsets, check_quant=False), rng)


@pytest.mark.parametrize("seed", range(8))
def test_random_shapes(mx, tile_config, seed):
    """Seeded random problems: 1-24 experts with counts from 0 to 700 (a few
    empty), N a multiple of 128 up to 640, K a multiple of 32 up to 1024 -- so
    every tile shape meets full, ragged and swapped tiles, partial output
    blocks and partial K blocks in combinations no hand-picked case covers."""
    rng = np.random.default_rng(1000 + seed)
    E = int(rng.integers(1, 25))
    counts = rng.integers(0, 701, size=E)
    counts[rng.random(E) < 0.15] = 0
    N = 128 * int(rng.integers(1, 6))
    K = 32 * int(rng.integers(1, 33))
    run_all_and_compare(make_case(mx, counts.tolist(), N, K, seed=seed))


def test_the_largest_group_count(mx, tile_config):
    """MXF8_GEMM_MAX_GROUPS experts, most of them empty or tiny: the on-device
    schedule's prefix runs over eight warps' worth of groups and the wgrad
    longest-first ranking over all of them (ties between equal counts)."""
    rng = np.random.default_rng(256)
    counts = rng.choice([0, 0, 1, 3, 17, 40, 129, 260], size=mx.MXF8_GEMM_MAX_GROUPS).tolist()
    run_all_and_compare(make_case(mx, counts, 128, 96, seed=256))


def test_more_groups_than_the_limit_are_rejected(mx):
    E = mx.MXF8_GEMM_MAX_GROUPS + 1
    c = make_case(mx, [1] * 4, 128, 64, check_quant=False)
    od = torch.arange(E + 1, dtype=torch.int32, device="cuda").clamp(max=4)
    with pytest.raises(mx.MXFP8Error):
        mx.mxfp8_grouped_gemm_fwd(c.xq, c.xs, c.wq, c.ws, od, 128, work=mx.new_workspace(E, 4, 128, 64))
