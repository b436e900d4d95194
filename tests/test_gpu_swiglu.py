"""GPU parity of the gate/up forward GEMM fused with SwiGLU and MXFP8
quantisation (mxfp8_grouped_gemm_fwd_swiglu).

h = silu(gate) * up from the gate/up GEMM's fp32 accumulators (gate =
output columns 0..I-1, up = I..2I-1), rounded once to bf16:
- h is checked against the oracle's SwiGLU of its fp64 GEMM on the same
  quantised bytes, with the GEMM tolerance (normalised Frobenius error
  <= 5e-3 and per-element relative error <= 2e-2 where |ref| > 1e-2 rms);
- the MXFP8 copies are defined as the MXFP8 quantisation of that bf16 h
  with the GEMM's groups, so they are compared byte for byte with the
  oracle's quantisers applied to the kernel's own h and with the library's
  separate quantisers (whole sentinel-filled buffers).
The pages give no formula for the activation between the two linears; the
expert pipeline is on opensourcebeat.com, section "Двухсторонняя атака:
MXFP8 и DeepEP"."""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.helpers import assert_gemm_close, np_u8
from tests.test_gpu_gemm import guard_intact, poisoned, tile_config  # noqa: F401

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


class Op:
    """Quantised X and W (gate/up weights [E, 2I, K]) of one grouped linear."""

    def __init__(self, mx, X, W, offs):
        self.mx = mx
        self.offs = np.asarray(offs, np.int32)
        self.od = torch.from_numpy(self.offs).cuda()
        self.E, self.N, self.K = W.shape
        self.M = X.shape[0]
        self.xq, self.xs = mx.mxfp8_quantize_rowwise(X.cuda(), self.od)
        self.wq, self.ws = mx.mxfp8_quantize_rowwise(W.reshape(self.E * self.N, self.K).cuda())
        torch.cuda.synchronize()

    def run(self, out=True, rowwise=True, colwise=True):
        M, I, E = self.M, self.N // 2, self.E
        rb, cb = _buffers(self.mx, M, I, E)
        bh = h = None
        if out:
            bh, h = poisoned((M, I))
        self.mx.mxfp8_grouped_gemm_fwd_swiglu(self.xq, self.xs, self.wq, self.ws, self.od, self.N, out=h,
                                              rowwise=rb if rowwise else None, colwise=cb if colwise else None)
        torch.cuda.synchronize()
        if out:
            assert guard_intact(bh, M * I)
        return h, rb, cb

    def reference_h(self):
        """Oracle: fp64 gate/up GEMM per expert on the GPU's bytes, then SwiGLU
        (fp64, one bf16 rounding) -> float64 values of the bf16 h."""
        M, I = self.M, self.N // 2
        Y = np.zeros((M, self.N))
        for e, lo, hi, ye in oracle.fwd_by_expert(np_u8(self.xq), np_u8(self.xs), np_u8(self.wq), np_u8(self.ws),
                                                  self.offs, self.N):
            Y[lo:hi] = ye
        hb = oracle.swiglu(Y)
        return (hb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check(mx, op: Op):
    M, I, E = op.M, op.N // 2, op.E
    h, (q, s), (qT, sT) = op.run()
    assert_gemm_close(h.double().cpu().numpy(), op.reference_h(), "swiglu h")
    # the MXFP8 copies: the library's quantisers and the oracle's on the kernel's own h
    (q2, s2), (qT2, sT2) = _buffers(mx, M, I, E)
    mx.mxfp8_quantize_rowwise(h, op.od, q=q2, scales=s2)
    mx.mxfp8_quantize_colwise(h, op.od, qT=qT2, scales=sT2)
    torch.cuda.synchronize()
    assert torch.equal(q, q2) and torch.equal(s, s2), "rowwise copy differs from mxfp8_quantize_rowwise"
    assert torch.equal(qT, qT2) and torch.equal(sT, sT2), "colwise copy differs from mxfp8_quantize_colwise"
    hb = h.cpu()
    rq, rs = oracle.quantize_rowwise(hb, op.offs)
    np.testing.assert_array_equal(np_u8(q), rq)
    RB, PG = oracle.group_blocks(op.offs, M)
    n = RB * oracle.rowwise_pitch(I) * 512
    np.testing.assert_array_equal(np_u8(s)[:n], rs[:n])
    rqT, rsT = oracle.quantize_colwise(hb, op.offs)
    np.testing.assert_array_equal(np_u8(qT)[:, :PG], rqT[:, :PG])
    pitch = oracle.colwise_pitch(M, E)
    gsT = np_u8(sT)
    for rb in range((I + 127) // 128):
        a = rb * pitch
        np.testing.assert_array_equal(gsT[a * 512:(a + RB) * 512], rsT[a * 512:(a + RB) * 512])
    return h, (q, s), (qT, sT)


def _op(mx, counts, N, K, seed, w_std=0.3):
    offs = wl.offsets_from_counts(counts)
    M, E = int(offs[-1]), len(counts)
    X = wl.normal_bf16((M, K), 1.0, seed + 1)
    W = wl.normal_bf16((E, N, K), w_std, seed + 2)
    return Op(mx, X, W, offs)


@pytest.mark.parametrize("counts,N,K", [([0, 1, 129, 300, 77, 255], 512, 416), ([0, 7, 21, 36], 256, 256),
                                        ([40, 0, 260], 768, 544), ([0, 0, 400, 0], 256, 128)])
def test_swiglu_epilogue(mx, tile_config, counts, N, K):
    check(mx, _op(mx, counts, N, K, seed=N + K))


@pytest.mark.parametrize("seed", range(3))
def test_swiglu_random_shapes(mx, tile_config, seed):
    """Seeded random problems: 1-16 experts, counts 0-600 (some empty), N a
    multiple of 256 up to 1024, K a multiple of 32 up to 768."""
    rng = np.random.default_rng(3000 + seed)
    E = int(rng.integers(1, 17))
    counts = rng.integers(0, 601, size=E)
    counts[rng.random(E) < 0.15] = 0
    check(mx, _op(mx, counts.tolist(), 256 * int(rng.integers(1, 5)), 32 * int(rng.integers(1, 25)), seed=seed))


def test_each_output_alone(mx):
    """Any subset of {bf16 h, rowwise, colwise} gives the same bytes, and a
    skipped layout is not touched."""
    op = _op(mx, [0, 1, 129, 300, 77, 255], 512, 416, seed=3)
    h_all, r_all, c_all = op.run()
    _, r_only, _ = op.run(out=False, colwise=False)
    _, _, c_only = op.run(out=False, rowwise=False)
    h_only, r_none, c_none = op.run(rowwise=False, colwise=False)
    assert torch.equal(h_only.view(torch.int16), h_all.view(torch.int16))
    for a, b in zip(r_only, r_all):
        assert torch.equal(a, b)
    for a, b in zip(c_only, c_all):
        assert torch.equal(a, b)
    for t in (*r_none, *c_none):
        assert bool((t == SENTINEL).all())


def test_swiglu_argument_errors(mx):
    op = _op(mx, [10, 20], 384, 64, seed=5)     # N = 384: I = 192 is not a multiple of 128
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):
        mx.mxfp8_grouped_gemm_fwd_swiglu(op.xq, op.xs, op.wq, op.ws, op.od, 384)
    op = _op(mx, [10, 20], 256, 64, seed=6)
    with pytest.raises(mx.MXFP8Error, match="INVALID_ARG"):     # nothing to write
        mx.mxfp8_grouped_gemm_fwd_swiglu(op.xq, op.xs, op.wq, op.ws, op.od, 256, out=None, rowwise=None,
                                         colwise=None)


@pytest.mark.parametrize("name", ["ds-v3-16b", "ds-v3-671b", "llama4-scout"])
def test_swiglu_full_size(mx, name):
    """The gate/up linear of each MoE workload at full size: h against the
    oracle (every element), MXFP8 copies byte for byte."""
    w = wl.WORKLOADS[name]()
    L = w.layers[0]
    X, W, _ = wl.layer_tensors(w, L, device="cuda")
    op = Op(mx, X, W, w.offsets)
    del X, W
    torch.cuda.empty_cache()
    check(mx, op)
