"""Whole-tensor parity at the full workload sizes, in the launch
configuration the benchmark times.

For every grouped linear of the three MoE workloads (DeepSeek-V3-16B-like,
DeepSeek-V3-671B-like, Llama-4-Scout-like: shapes and routing of the model
pages, synthetic draws) and for every size of the quantiser sweep:

- quantisers: every code byte and every defined scale byte (pads included)
  of X, W and dY, rowwise and colwise, equals the oracle's quantisation of
  the same bf16 tensor -- the dual kernel (the one the training step runs)
  and the separate rowwise / colwise kernels;
- grouped GEMMs: every output element of fwd, dgrad and wgrad, expert by
  expert, against the oracle's fp64 product of the dequantised GPU bytes
  (normalised Frobenius error <= 5e-3, per-element relative error <= 2e-2
  where |ref| > 1e-2 * rms(ref); an expert without rows has exactly zero
  dW); outputs start NaN-poisoned with a NaN guard tail, so an element the
  kernel skips or a write past the end fails.

MXFP8 block rules: OCP MX v1.0 (opensourcebeat.com, "Enabling up to 41%
faster pre-training: MXFP8 and DeepEP ...", FAQ "What is MXFP8?"); one
grouped GEMM over every expert's real token count (iitak.ru, "NVIDIA ...
JAX", Transformer Engine paragraph).
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.helpers import assert_gemm_close

pytestmark = pytest.mark.gpu

POISON = 0x7FC0


@pytest.fixture(scope="module")
def mx():
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert m.mxfp8_device_supported(), "GPU tests need an sm_100 device"
    return m


def _u8(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def _poisoned(shape, guard=4096):
    n = int(np.prod(shape))
    buf = torch.full((n + guard,), POISON, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    return buf, buf[:n].view(*shape)


def _guard_intact(buf, n):
    return bool(torch.all(buf[n:].view(torch.int16) == POISON))


def _defined_scale_bytes_colwise(sfT: np.ndarray, C: int, pitch: int, RB: int) -> np.ndarray:
    """The colwise scale atoms the layout defines: atom columns < RB_G of
    every atom row."""
    rb = (C + 127) // 128
    return np.asarray(sfT[:rb * pitch * 512]).reshape(rb, pitch, 512)[:, :RB]


def quantise_and_check(mx, x: torch.Tensor, offs: np.ndarray | None):
    """Quantises the device tensor x with the dual kernel and the separate
    kernels, checks every defined byte against the oracle and returns the
    dual kernel's (q, sf, qT, sfT) on the device."""
    R, C = x.shape
    G = 1 if offs is None else len(offs) - 1
    od = None if offs is None else torch.from_numpy(np.asarray(offs, np.int32)).cuda()
    q, sf, qT, sfT = mx.mxfp8_quantize_dual(x, od)
    q2, sf2 = mx.mxfp8_quantize_rowwise(x, od)
    qT2, sfT2 = mx.mxfp8_quantize_colwise(x, od)
    torch.cuda.synchronize()
    RB, PG = oracle.group_blocks(offs, R)
    n_row = RB * oracle.rowwise_pitch(C) * 512
    pitch = oracle.colwise_pitch(R, G)
    xh = x.cpu()
    rq, rsf = oracle.quantize_rowwise(xh, offs)
    gq = _u8(q)
    assert np.array_equal(gq, rq), "rowwise codes differ from the oracle"
    assert np.array_equal(_u8(sf)[:n_row], rsf[:n_row]), "rowwise scales differ from the oracle"
    assert torch.equal(q, q2) and torch.equal(sf[:n_row], sf2[:n_row]), "rowwise kernel differs from the dual kernel"
    del rq, rsf, gq
    cq, csf = oracle.quantize_colwise(xh, offs)
    del xh
    assert np.array_equal(_u8(qT[:, :PG]), cq[:, :PG]), "colwise codes differ from the oracle"
    assert np.array_equal(_defined_scale_bytes_colwise(_u8(sfT), C, pitch, RB),
                          _defined_scale_bytes_colwise(csf, C, pitch, RB)), "colwise scales differ from the oracle"
    assert torch.equal(qT[:, :PG], qT2[:, :PG]), "colwise kernel differs from the dual kernel"
    assert np.array_equal(_defined_scale_bytes_colwise(_u8(sfT2), C, pitch, RB),
                          _defined_scale_bytes_colwise(_u8(sfT), C, pitch, RB)), "colwise kernel scales differ"
    del cq, csf, q2, sf2, qT2, sfT2
    return q, sf, qT, sfT


@pytest.mark.parametrize("name,layer", [(n, i) for n in ("ds-v3-16b", "ds-v3-671b", "llama4-scout") for i in (0, 1)])
def test_workload_whole_tensors(mx, name, layer):
    w = wl.WORKLOADS[name]()
    L = w.layers[layer]
    E, M, N, K = w.E, w.M, L.N, L.K
    offs = w.offsets
    od = torch.from_numpy(offs).cuda()
    X, W, dY = wl.layer_tensors(w, L, device="cuda")
    W2 = W.reshape(E * N, K)
    del W
    xq, xs, xqT, xsT = quantise_and_check(mx, X, offs)
    wq, ws, wqT, wsT = quantise_and_check(mx, W2, None)
    dyq, dys, dyqT, dysT = quantise_and_check(mx, dY, offs)
    del X, W2, dY
    torch.cuda.empty_cache()

    work = mx.new_workspace(E, M, N, K)
    by, y = _poisoned((M, N))
    bdx, dx = _poisoned((M, K))
    bdw, dw = _poisoned((E, N, K))
    mx.mxfp8_grouped_gemm_fwd(xq, xs, wq, ws, od, N, out=y, work=work)
    mx.mxfp8_grouped_gemm_dgrad(dyq, dys, wqT, wsT, od, K, out=dx, work=work)
    mx.mxfp8_grouped_gemm_wgrad(dyqT, dysT, xqT, xsT, od, M, out=dw, work=work)
    assert mx.mxfp8_get_status(work) == 0
    assert _guard_intact(by, M * N) and _guard_intact(bdx, M * K) and _guard_intact(bdw, E * N * K)

    h = {k: _u8(v) for k, v in dict(xq=xq, xs=xs, wq=wq, ws=ws, dyq=dyq, dys=dys).items()}
    for e, lo, hi, ref in oracle.fwd_by_expert(h["xq"], h["xs"], h["wq"], h["ws"], offs, N):
        assert_gemm_close(y[lo:hi].double().cpu().numpy(), ref, f"{name} {L.name} fwd expert {e}")
    del h["xq"], h["xs"], h["wq"], h["ws"]
    h.update(wqT=_u8(wqT), wsT=_u8(wsT))
    for e, lo, hi, ref in oracle.dgrad_by_expert(h["dyq"], h["dys"], h["wqT"], h["wsT"], offs, K):
        assert_gemm_close(dx[lo:hi].double().cpu().numpy(), ref, f"{name} {L.name} dgrad expert {e}")
    h.clear()
    h.update(dyqT=_u8(dyqT), dysT=_u8(dysT), xqT=_u8(xqT), xsT=_u8(xsT))
    for e, ref in oracle.wgrad_by_expert(h["dyqT"], h["dysT"], h["xqT"], h["xsT"], offs, M):
        got = dw[e].double().cpu().numpy()
        if offs[e + 1] == offs[e]:
            assert np.all(got == 0.0), f"{name} {L.name} wgrad: empty expert {e} is not zero"
        else:
            assert_gemm_close(got, ref, f"{name} {L.name} wgrad expert {e}")


@pytest.mark.parametrize("M,K", wl.quantiser_sweep())
def test_sweep_whole_tensors(mx, M, K):
    """The quantiser sweep (one group; N(0,1), 0.1 % outliers x1000, 1 % of
    aligned 32x32 tiles zeroed): every byte of both layouts from the dual
    kernel and the separate kernels equals the oracle."""
    x = wl.sweep_tensor(M, K, device="cuda")
    quantise_and_check(mx, x, None)
