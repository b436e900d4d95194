"""GPU parity of the quantising epilogue (fwd and dgrad GEMMs that also write
their output as MXFP8).

The quantised copies are defined as the MXFP8 quantisation of the GEMM's own
bf16 output with the GEMM's groups, so they are checked byte for byte:
against the oracle's quantisers applied to that output, and against the
library's separate quantisers (whole buffers, pre-filled with a sentinel, so
a byte written by one side and not the other also fails).  The bf16 output
itself must be identical to the plain GEMM's, whose parity with the fp64
oracle is covered in test_gpu_gemm.py."""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.helpers import np_u8, u16
from tests.test_gpu_gemm import Case, guard_intact, make_case, poisoned, tile_config  # noqa: F401

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5


@pytest.fixture(scope="module")
def mx():
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert m.mxfp8_device_supported(), "GPU tests need an sm_100 device"
    return m


def _filled(*shape):
    return torch.full(shape, SENTINEL, dtype=torch.uint8, device="cuda")


def _buffers(mx, M, C, E):
    ld = mx.mxfp8_colwise_ld(M, E)
    return ((_filled(M, C), _filled(max(mx.mxfp8_rowwise_scale_bytes(M, C, E), 16))),
            (_filled(C, ld), _filled(max(mx.mxfp8_colwise_scale_bytes(M, C, E), 16))))


def fused(mx, c: Case, mode, out=True, rowwise=True, colwise=True):
    """Runs the fused GEMM into sentinel-filled buffers; returns (y, row, col)."""
    M, E = c.M, c.E
    C = c.N if mode == "fwd" else c.K
    rb, cb = _buffers(mx, M, C, E)
    by = y = None
    if out:
        by, y = poisoned((M, C))
    args = dict(out=y, rowwise=rb if rowwise else None, colwise=cb if colwise else None)
    if mode == "fwd":
        mx.mxfp8_grouped_gemm_fwd_quant(c.xq, c.xs, c.wq, c.ws, c.od, c.N, **args)
    else:
        mx.mxfp8_grouped_gemm_dgrad_quant(c.dyq, c.dys, c.wqT, c.wsT, c.od, c.K, **args)
    torch.cuda.synchronize()
    if out:
        assert guard_intact(by, M * C)
    return y, rb, cb


def check_mode(mx, c: Case, mode):
    M, E = c.M, c.E
    C = c.N if mode == "fwd" else c.K
    plain = c.fwd() if mode == "fwd" else c.dgrad()
    y, (q, s), (qT, sT) = fused(mx, c, mode)
    assert torch.equal(y.view(torch.int16), plain.view(torch.int16)), "bf16 output differs from the plain GEMM"

    # the library's quantisers on the same bf16 output, into sentinel buffers
    (q2, s2), (qT2, sT2) = _buffers(mx, M, C, E)
    mx.mxfp8_quantize_rowwise(plain, c.od, q=q2, scales=s2)
    mx.mxfp8_quantize_colwise(plain, c.od, qT=qT2, scales=sT2)
    torch.cuda.synchronize()
    assert torch.equal(q, q2) and torch.equal(s, s2), "rowwise copy differs from mxfp8_quantize_rowwise"
    assert torch.equal(qT, qT2) and torch.equal(sT, sT2), "colwise copy differs from mxfp8_quantize_colwise"

    # the oracle's quantisers on the same bf16 output
    ybf = plain.cpu()
    rq, rs = oracle.quantize_rowwise(ybf, c.offs)
    np.testing.assert_array_equal(np_u8(q), rq)
    RB, PG = oracle.group_blocks(c.offs, M)
    n = RB * oracle.rowwise_pitch(C) * 512
    np.testing.assert_array_equal(np_u8(s)[:n], rs[:n])
    rqT, rsT = oracle.quantize_colwise(ybf, c.offs)
    np.testing.assert_array_equal(np_u8(qT)[:, :PG], rqT[:, :PG])
    pitch = oracle.colwise_pitch(M, E)
    gsT = np_u8(sT)
    for rb in range((C + 127) // 128):
        a = rb * pitch
        np.testing.assert_array_equal(gsT[a * 512:(a + RB) * 512], rsT[a * 512:(a + RB) * 512])
    return y, (q, s), (qT, sT)


CASES = {
    # several tiles per group, ragged tails, an empty expert, a partial
    # output tile, a partial K block
    "ragged": ([0, 1, 129, 300, 77, 255], 384, 416),
    # output columns not a multiple of 128 (dgrad: K = 544) -- partial scale atoms
    "partial_atoms": ([40, 0, 260], 384, 544),
    "tiny": ([0, 7, 21, 36], 128, 256),
    "one_expert": ([0, 0, 400, 0], 256, 256),
}


@pytest.mark.parametrize("mode", ["fwd", "dgrad"])
@pytest.mark.parametrize("name", list(CASES))
def test_quantising_epilogue(mx, tile_config, name, mode):
    counts, N, K = CASES[name]
    check_mode(mx, make_case(mx, counts, N, K, seed=len(counts) + N), mode)


@pytest.mark.parametrize("mode", ["fwd", "dgrad"])
@pytest.mark.parametrize("seed", range(3))
def test_quantising_epilogue_random_shapes(mx, tile_config, seed, mode):
    """Seeded random problems: 1-16 experts, counts 0-600 (some empty), N a
    multiple of 128 up to 640, K a multiple of 32 up to 768 -- partial scale
    atoms, ragged and swapped tiles in every tile shape."""
    rng = np.random.default_rng(4000 + seed)
    E = int(rng.integers(1, 17))
    counts = rng.integers(0, 601, size=E)
    counts[rng.random(E) < 0.15] = 0
    N, K = 128 * int(rng.integers(1, 6)), 32 * int(rng.integers(1, 25))
    check_mode(mx, make_case(mx, counts.tolist(), N, K, seed=seed, check_quant=False), mode)


@pytest.mark.parametrize("mode", ["fwd", "dgrad"])
def test_distinct_block_magnitudes_and_overflow(mx, tile_config, mode):
    """Rows of X and dY scaled by powers of two from 2^-30 to 2^40 give
    output blocks over a wide scale range; a few rows scaled by 2^120 make
    the fp32 accumulators overflow, so their blocks take the NaN-scale path."""
    counts = [70, 0, 150, 33]
    offs = wl.offsets_from_counts(counts)
    M, E, N, K = int(offs[-1]), len(counts), 256, 256
    rng = np.random.default_rng(11)
    e = rng.integers(-30, 41, size=(M, 1)).astype(np.float64)
    e[[3, 100, 200]] = 120.0
    X = torch.from_numpy(rng.standard_normal((M, K)) * 2.0 ** e).to(torch.bfloat16)
    dY = torch.from_numpy(rng.standard_normal((M, N)) * 2.0 ** e).to(torch.bfloat16)
    W = torch.from_numpy(rng.standard_normal((E, N, K)) * 2.0 ** 20).to(torch.bfloat16)
    c = Case(mx, X, W, dY, offs, check_quant=False)
    y, (q, s), _ = check_mode(mx, c, mode)
    assert not torch.isfinite(y.float()).all(), "the overflow rows should produce non-finite outputs"
    assert (s == 0xFF).any(), "expected NaN scales for the overflowed blocks"


@pytest.mark.parametrize("mode", ["fwd", "dgrad"])
def test_each_output_alone(mx, tile_config, mode):
    """Any subset of {bf16, rowwise, colwise} gives the same bytes (in CTA
    pairs the groups' ragged tiles run swapped, with their own drain)."""
    c = make_case(mx, [0, 1, 129, 300, 77, 255], 384, 416, seed=7)
    y_all, r_all, c_all = fused(mx, c, mode)
    _, r_only, _ = fused(mx, c, mode, out=False, colwise=False)
    _, _, c_only = fused(mx, c, mode, out=False, rowwise=False)
    y_only, r_none, c_none = fused(mx, c, mode, rowwise=False, colwise=False)
    assert torch.equal(y_only.view(torch.int16), y_all.view(torch.int16))
    for a, b in zip(r_only, r_all):
        assert torch.equal(a, b)
    for a, b in zip(c_only, c_all):
        assert torch.equal(a, b)
    for t in (*r_none, *c_none):   # skipped layouts are not touched
        assert bool((t == SENTINEL).all())


def test_quantising_epilogue_argument_errors(mx):
    c = make_case(mx, [10, 20], 128, 64, check_quant=False)
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):   # nothing to write
        mx.mxfp8_grouped_gemm_fwd_quant(c.xq, c.xs, c.wq, c.ws, c.od, 128, out=None, rowwise=None, colwise=None)
    (q, s), _ = _buffers(mx, c.M, 128, c.E)
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):   # rowwise scale buffer too small
        mx.mxfp8_grouped_gemm_fwd_quant(c.xq, c.xs, c.wq, c.ws, c.od, 128, rowwise=(q, s[:16]), colwise=None)


@pytest.mark.parametrize("name", ["ds-v3-16b", "ds-v3-671b"])
def test_quantising_epilogue_full_size(mx, name):
    """Full workload sizes in the default launch configuration: the fused
    copies equal the separate quantisers' output on the plain GEMM's bf16
    result, whole buffers compared on the GPU."""
    w = wl.WORKLOADS[name]()
    layer = w.layers[0]
    X, W, dY = wl.layer_tensors(w, layer)
    c = Case(mx, X, W, dY, w.offsets, check_quant=False)
    for mode in ("fwd", "dgrad"):
        M, C = c.M, (c.N if mode == "fwd" else c.K)
        plain = c.fwd() if mode == "fwd" else c.dgrad()
        y, (q, s), (qT, sT) = fused(mx, c, mode)
        (q2, s2), (qT2, sT2) = _buffers(mx, M, C, c.E)
        mx.mxfp8_quantize_dual(plain, c.od, q=q2, scales=s2, qT=qT2, scalesT=sT2)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), plain.view(torch.int16))
        assert torch.equal(q, q2) and torch.equal(s, s2) and torch.equal(qT, qT2) and torch.equal(sT, sT2)
        del y, q, s, qT, sT, q2, s2, qT2, sT2, plain
        torch.cuda.empty_cache()
