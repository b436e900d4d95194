"""GPU parity of the NVFP4 quantisers (amax, rowwise, colwise) against the
oracle, byte for byte, through the C ABI.  The element codes are decided in
fp32 in the same operation order on both sides, so equality is exact."""
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


def _offs_dev(offs):
    return None if offs is None else torch.as_tensor(np.asarray(offs, dtype=np.int32)).cuda()


def check(mx, x: torch.Tensor, offs=None):
    R, C = x.shape
    xd = x.cuda()
    amax = mx.mxfp8_nvfp4_amax(xd)
    q, s = mx.mxfp8_nvfp4_quantize_rowwise(xd, amax, _offs_dev(offs))
    qT, sT = mx.mxfp8_nvfp4_quantize_colwise(xd, amax, _offs_dev(offs))
    torch.cuda.synchronize()
    ra = oracle.nvfp4_amax(x)
    assert np.float32(amax.item()) == ra
    S = oracle.nvfp4_tensor_scale(ra)
    o = offs if offs is not None else np.array([0, R], dtype=np.int32)
    G = len(o) - 1
    rq, rs = oracle.nvfp4_quantize_rowwise(x, S, o)
    np.testing.assert_array_equal(np_u8(q), rq)
    RB, RB64, PG = oracle.nvfp4_group_blocks(o, R)
    n = RB * oracle.nvfp4_rowwise_pitch(C) * 512
    np.testing.assert_array_equal(np_u8(s)[:n], rs[:n])
    cq, cs = oracle.nvfp4_quantize_colwise(x, S, o)
    np.testing.assert_array_equal(np_u8(qT)[:, :PG // 2], cq[:, :PG // 2])
    pitch = oracle.nvfp4_colwise_pitch(R, G)
    g = np_u8(sT)
    for rb in range((C + 127) // 128):
        a = rb * pitch
        np.testing.assert_array_equal(g[a * 512:(a + RB64) * 512], cs[a * 512:(a + RB64) * 512])


def test_single_group_shapes(mx):
    check(mx, wl.normal_bf16((256, 128), 1.0, 1))
    check(mx, wl.normal_bf16((100, 192), 3.0, 2))     # ragged rows, cols % 128 == 64


@pytest.mark.parametrize("seed", range(3))
def test_grouped(mx, seed):
    counts = np.array([0, 1, 15, 16, 17, 63, 64, 65, 0, 129, 300, 7], dtype=np.int64)
    np.random.default_rng(seed).shuffle(counts)
    offs = wl.offsets_from_counts(counts)
    check(mx, wl.normal_bf16((int(offs[-1]), 256), 1.0, 10 + seed), offs)


def test_wide_dynamic_range_and_zero_blocks(mx):
    """Blocks with their own magnitudes (the E4M3 scale underflows to 0 for
    the smallest ones), all-zero blocks, and a few large outliers."""
    rng = np.random.default_rng(4)
    R, C = 192, 256
    e = rng.integers(-30, 10, size=(R, C // 16))
    v = rng.standard_normal((R, C)) * np.repeat(2.0 ** e, 16, axis=1)
    v[:, 32:48] = 0.0
    v[5, 7] = 3e4
    x = torch.from_numpy(v).to(torch.bfloat16)
    offs = wl.offsets_from_counts([50, 0, 142])
    check(mx, x, offs)


def test_all_zero_tensor(mx):
    check(mx, torch.zeros((128, 64), dtype=torch.bfloat16))


def test_every_finite_bf16_magnitude_as_block_amax(mx):
    """Every finite bf16 pattern appears in some block, exercising every scale
    the E4M3 rounding of amax * S / 6 produces."""
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    b = b[((b >> 7) & 0xFF) != 0xFF]
    b = np.random.default_rng(5).permutation(b)
    b = b[: (b.size // 256) * 256]
    x = torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).reshape(-1, 256)
    check(mx, x)


def test_workload_size_sampled(mx):
    """DeepSeek-V3-16B-like X (49152 x 2048, 64 groups): amax and a seeded
    sample of rows / columns against the oracle's blocks."""
    w = wl.WORKLOADS["ds-v3-16b"]()
    X, _, _ = wl.layer_tensors(w, w.layers[0])
    od = _offs_dev(w.offsets)
    xd = X.cuda()
    amax = mx.mxfp8_nvfp4_amax(xd)
    q, s = mx.mxfp8_nvfp4_quantize_rowwise(xd, amax, od)
    torch.cuda.synchronize()
    ra = oracle.nvfp4_amax(X)
    assert np.float32(amax.item()) == ra
    S = oracle.nvfp4_tensor_scale(ra)
    rows = np.random.default_rng(6).choice(X.shape[0], 64, replace=False)
    qn = np_u8(q)
    xu = X.view(torch.int16).numpy().view(np.uint16)
    for r in rows:
        for j in range(0, X.shape[1] // 16, 7):
            codes, _ = oracle.nvfp4_quantize_block(xu[r, 16 * j:16 * j + 16], S)
            packed = codes[0::2] | (codes[1::2] << 4)
            np.testing.assert_array_equal(qn[r, 8 * j:8 * j + 8], packed)


def test_bad_arguments(mx):
    x = torch.zeros((64, 96), dtype=torch.bfloat16, device="cuda")
    amax = mx.mxfp8_nvfp4_amax(x)
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):
        mx.mxfp8_nvfp4_quantize_rowwise(x, amax)          # cols % 64 != 0
