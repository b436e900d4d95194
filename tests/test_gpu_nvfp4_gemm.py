"""GPU parity of the NVFP4 grouped GEMMs (fwd, dgrad, wgrad) against the fp64
oracle on identical quantised inputs: the oracle dequantises the GPU's own
NVFP4 bytes (code * E4M3 scale / tensor scale) and forms the per-expert
products in fp64; the GPU accumulates in fp32.  Same tolerance as the MXFP8
GEMMs (tests/helpers.py)."""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.helpers import assert_gemm_close, f64, np_u8

pytestmark = pytest.mark.gpu

POISON = 0x7FC0


@pytest.fixture(scope="module")
def mx():
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert m.mxfp8_device_supported(), "GPU tests need an sm_100 device"
    return m


@pytest.fixture(params=["default", "pair"])
def fp4_tiling(mx, request):
    """The NVFP4 GEMM in its default 1-CTA tiles and in CTA pairs (each group's
    ragged last tile swapped)."""
    mx.mxfp8_set_gemm_tiling(1 if request.param == "pair" else -1, -1)
    yield request.param
    mx.mxfp8_set_gemm_tiling(-1, -1)


class Fp4Case:
    def __init__(self, mx, X, W, dY, offs):
        self.mx, self.offs = mx, np.asarray(offs, dtype=np.int32)
        self.E, self.N, self.K = W.shape
        self.M = X.shape[0]
        self.od = torch.from_numpy(self.offs).cuda()
        Xd, Wd, dYd = X.cuda(), W.reshape(self.E * self.N, self.K).cuda(), dY.cuda()
        self.ax, self.aw, self.ady = mx.mxfp8_nvfp4_amax(Xd), mx.mxfp8_nvfp4_amax(Wd), mx.mxfp8_nvfp4_amax(dYd)
        self.xq, self.xs = mx.mxfp8_nvfp4_quantize_rowwise(Xd, self.ax, self.od)
        self.wq, self.ws = mx.mxfp8_nvfp4_quantize_rowwise(Wd, self.aw)
        self.dyq, self.dys = mx.mxfp8_nvfp4_quantize_rowwise(dYd, self.ady, self.od)
        self.wqT, self.wsT = mx.mxfp8_nvfp4_quantize_colwise(Wd, self.aw)
        self.dyqT, self.dysT = mx.mxfp8_nvfp4_quantize_colwise(dYd, self.ady, self.od)
        self.xqT, self.xsT = mx.mxfp8_nvfp4_quantize_colwise(Xd, self.ax, self.od)
        torch.cuda.synchronize()
        S = lambda a: oracle.nvfp4_tensor_scale(np.float32(a.item()))  # noqa: E731
        self.Sx, self.Sw, self.Sdy = S(self.ax), S(self.aw), S(self.ady)

    def refs(self):
        o, E, N, K, M = self.offs, self.E, self.N, self.K, self.M
        Xd = oracle.nvfp4_dequantize_rowwise(np_u8(self.xq), np_u8(self.xs), self.Sx, o)
        Wd = oracle.nvfp4_dequantize_rowwise(np_u8(self.wq), np_u8(self.ws), self.Sw).reshape(E, N, K)
        dYd = oracle.nvfp4_dequantize_rowwise(np_u8(self.dyq), np_u8(self.dys), self.Sdy, o)
        WdT = oracle.nvfp4_dequantize_colwise(np_u8(self.wqT), np_u8(self.wsT), E * N, self.Sw).reshape(E, N, K)
        dYc = oracle.nvfp4_dequantize_colwise(np_u8(self.dyqT), np_u8(self.dysT), M, self.Sdy, o)
        Xc = oracle.nvfp4_dequantize_colwise(np_u8(self.xqT), np_u8(self.xsT), M, self.Sx, o)
        return (oracle.gemm_fwd(Xd, Wd, o), oracle.gemm_dgrad(dYd, WdT, o), oracle.gemm_wgrad(dYc, Xc, o))

    def run(self):
        mx = self.mx
        y = mx.mxfp8_nvfp4_grouped_gemm_fwd(self.xq, self.xs, self.ax, self.wq, self.ws, self.aw, self.od, self.N)
        dx = mx.mxfp8_nvfp4_grouped_gemm_dgrad(self.dyq, self.dys, self.ady, self.wqT, self.wsT, self.aw, self.od,
                                               self.K)
        dw = mx.mxfp8_nvfp4_grouped_gemm_wgrad(self.dyqT, self.dysT, self.ady, self.xqT, self.xsT, self.ax, self.od,
                                               self.M)
        torch.cuda.synchronize()
        return y, dx, dw


def check(mx, counts, N, K, seed=0):
    offs = wl.offsets_from_counts(counts)
    M, E = int(offs[-1]), len(counts)
    c = Fp4Case(mx, wl.normal_bf16((M, K), 1.0, seed + 1), wl.normal_bf16((E, N, K), 1.0, seed + 2),
                wl.normal_bf16((M, N), 1.0, seed + 3), offs)
    y, dx, dw = c.run()
    ry, rdx, rdw = c.refs()
    assert_gemm_close(f64(y), ry, "nvfp4 fwd")
    assert_gemm_close(f64(dx), rdx, "nvfp4 dgrad")
    gdw = f64(dw)
    for e in range(E):
        if counts[e] == 0:
            assert np.all(gdw[e] == 0.0)
        else:
            assert_gemm_close(gdw[e], rdw[e], f"nvfp4 wgrad expert {e}")


def test_tiny(mx, fp4_tiling):
    check(mx, [0, 7, 21, 36], 128, 256)


def test_ragged_multi_tile(mx, fp4_tiling):
    """Several tiles per group, ragged tails, an empty expert, a partial output
    tile (N = 384) and a partial K block (K = 448: one full 256-element block
    and one of three MMAs)."""
    check(mx, [0, 1, 129, 300, 77, 255], 384, 448, seed=7)


@pytest.mark.parametrize("counts,N,K", [([1], 128, 64), ([0, 0, 5], 128, 128), ([300], 256, 320),
                                        ([129, 127], 512, 192), ([70, 0, 33, 200], 256, 1024)])
def test_edge_shapes(mx, fp4_tiling, counts, N, K):
    check(mx, counts, N, K, seed=sum(counts))


@pytest.mark.parametrize("seed", range(4))
def test_random_shapes(mx, fp4_tiling, seed):
    """Seeded random problems (1-16 experts, counts 0-600 with some empty,
    N a multiple of 128 up to 512, K a multiple of 64 up to 1024) in both
    tile shapes."""
    rng = np.random.default_rng(2000 + seed)
    E = int(rng.integers(1, 17))
    counts = rng.integers(0, 601, size=E)
    counts[rng.random(E) < 0.15] = 0
    check(mx, counts.tolist(), 128 * int(rng.integers(1, 5)), 64 * int(rng.integers(1, 17)), seed=seed)


def test_ragged_tails_of_every_pair_shape(mx, fp4_tiling):
    """Group tails r = 31..255 around the multiples of 32 (the swapped tiles of
    CTA pairs have N = round_up(r, 32)), groups of exactly 256 rows and a half
    empty last output-column block (N = 640)."""
    check(mx, [32, 64 + 256, 96, 128, 160 + 512, 192, 224, 31, 33, 225, 255, 256], 640, 512, seed=21)


def test_full_size_sampled_ds_v3_16b(mx):
    """The DeepSeek-V3-16B-like gate/up linear at full size: outputs sampled
    against the oracle's dot products of the dequantised operands."""
    w = wl.WORKLOADS["ds-v3-16b"]()
    L = w.layers[0]
    X, W, dY = wl.layer_tensors(w, L)
    c = Fp4Case(mx, X, W, dY, w.offsets)
    y, dx, dw = c.run()
    rng = np.random.default_rng(3)
    o = c.offs
    r = rng.integers(0, c.M, 128)
    cn = rng.integers(0, c.N, 128)
    ck = rng.integers(0, c.K, 128)
    xq, xs = np_u8(c.xq), np_u8(c.xs)
    wq, ws = np_u8(c.wq), np_u8(c.ws)
    # dequantise only the rows needed (one expert's W rows per sample)
    gy = f64(y)
    group = np.searchsorted(o, r, side="right") - 1
    ref = np.zeros(r.size)
    xd_rows = {}
    for i, (ri, ni, gi) in enumerate(zip(r, cn, group)):
        if ri not in xd_rows:
            xd_rows[ri] = oracle.nvfp4_dequantize_rowwise(xq[ri:ri + 1], _row_scales(xs, ri, o, c.K), c.Sx)[0]
        wrow = int(gi) * c.N + int(ni)
        wd = oracle.nvfp4_dequantize_rowwise(wq[wrow:wrow + 1], _row_scales(ws, wrow, None, c.K), c.Sw)[0]
        ref[i] = float(np.dot(xd_rows[ri], wd))
    assert_gemm_close(gy[r, cn], ref, "nvfp4 fwd (sampled)")
    assert np.all(np.isfinite(f64(dx)[r[:16]])) and np.all(np.isfinite(f64(dw)[:, cn[:8], :][:, :, ck[:8]]))


def _nvfp4_rows(q, sf, C, row0, atom_row0, n, S):
    """Rows row0 .. row0 + n - 1 of a rowwise NVFP4 operand (their scale rows
    start at 128-row atom row atom_row0), dequantised: fp64 [n, C]."""
    pitch = oracle.nvfp4_rowwise_pitch(C)
    nb = (n + 127) // 128
    atoms = np.ascontiguousarray(sf[atom_row0 * pitch * 512:(atom_row0 + nb) * pitch * 512])
    return oracle.nvfp4_dequantize_rowwise(np.ascontiguousarray(q[row0:row0 + n]), atoms, S)


def _nvfp4_cols(qT, sfT, pitch, col0, atom_col0, n, S):
    """Logical rows col0 .. col0 + n - 1 of a colwise NVFP4 operand (codes
    from element column col0 of qT, an even number; scales from 64-row atom
    column atom_col0 of every 128-row atom row), dequantised: fp64 [n, C]."""
    C = qT.shape[0]
    ld = oracle.nvfp4_colwise_ld(n, 1) // 2
    sub = np.zeros((C, ld), dtype=np.uint8)
    nbytes = (n + 1) // 2
    sub[:, :nbytes] = qT[:, col0 // 2:col0 // 2 + nbytes]
    rb, na = (C + 127) // 128, (n + 63) // 64
    atoms = np.asarray(sfT[:rb * pitch * 512]).reshape(rb, pitch, 512)[:, atom_col0:atom_col0 + na]
    return oracle.nvfp4_dequantize_colwise(sub, np.ascontiguousarray(atoms).reshape(-1), n, S)


def test_whole_tensors_ds_v3_671b_gate_up(mx):
    """The DeepSeek-V3-671B-like gate/up linear at full size in the default
    launch configuration: every output element of fwd, dgrad and wgrad,
    expert by expert, against the oracle's fp64 product of the GPU's own
    NVFP4 bytes (zero dW for an expert without rows)."""
    w = wl.WORKLOADS["ds-v3-671b"]()
    L = w.layers[0]
    X, W, dY = wl.layer_tensors(w, L)
    c = Fp4Case(mx, X, W, dY, w.offsets)
    del X, W, dY
    y, dx, dw = c.run()
    o = np.asarray(c.offs, np.int64)
    m = np.diff(o)
    E, N, K, M = c.E, c.N, c.K, c.M
    RB = np.concatenate([[0], np.cumsum((m + 127) // 128)])
    Q = np.concatenate([[0], np.cumsum((m + 63) // 64)])
    P = np.concatenate([[0], np.cumsum((m + 31) // 32 * 32)])
    xq, xs, wq, ws = np_u8(c.xq), np_u8(c.xs), np_u8(c.wq), np_u8(c.ws)
    dyq, dys, wqT, wsT = np_u8(c.dyq), np_u8(c.dys), np_u8(c.wqT), np_u8(c.wsT)
    pitch_w = oracle.nvfp4_colwise_pitch(E * N, 1)
    for e in range(E):
        lo, hi = int(o[e]), int(o[e + 1])
        if hi == lo:
            continue
        We = _nvfp4_rows(wq, ws, K, e * N, e * N // 128, N, c.Sw)
        Xe = _nvfp4_rows(xq, xs, K, lo, int(RB[e]), hi - lo, c.Sx)
        assert_gemm_close(f64(y[lo:hi]), Xe @ We.T, f"nvfp4 fwd expert {e}")
        dYe = _nvfp4_rows(dyq, dys, N, lo, int(RB[e]), hi - lo, c.Sdy)
        WeT = _nvfp4_cols(wqT, wsT, pitch_w, e * N, e * N // 64, N, c.Sw)
        assert_gemm_close(f64(dx[lo:hi]), dYe @ WeT, f"nvfp4 dgrad expert {e}")
    del xq, xs, wq, ws, dyq, dys, wqT, wsT
    dyqT, dysT, xqT, xsT = np_u8(c.dyqT), np_u8(c.dysT), np_u8(c.xqT), np_u8(c.xsT)
    pitch = oracle.nvfp4_colwise_pitch(M, E)
    for e in range(E):
        got = f64(dw[e])
        if m[e] == 0:
            assert np.all(got == 0.0), f"nvfp4 wgrad: empty expert {e} is not zero"
            continue
        dYc = _nvfp4_cols(dyqT, dysT, pitch, int(P[e]), int(Q[e]), int(m[e]), c.Sdy)
        Xc = _nvfp4_cols(xqT, xsT, pitch, int(P[e]), int(Q[e]), int(m[e]), c.Sx)
        assert_gemm_close(got, dYc.T @ Xc, f"nvfp4 wgrad expert {e}")


def _row_scales(sf, row, offs, C):
    """The scale atom bytes of one row, re-packed as a single-row buffer in the
    same layout (row 0 of a one-group matrix)."""
    pitch = (C + 63) // 64
    if offs is None:
        pr = row
    else:
        m = np.diff(offs)
        g = int(np.searchsorted(offs, row, side="right") - 1)
        pr = int(((m[:g] + 127) // 128).sum()) * 128 + (row - int(offs[g]))
    out = np.zeros(pitch * 512, dtype=np.uint8)
    for j in range(C // 16):
        src = ((pr // 128) * pitch + j // 4) * 512 + (pr % 32) * 16 + ((pr % 128) // 32) * 4 + j % 4
        out[(j // 4) * 512 + j % 4] = sf[src]
    return out
