"""The GEMM's bounded pipeline waits, exercised on the GPU without faulting it.

With the library's test switch mxfp8_testing_stall_first_stage on, the
producer of every CTA (both CTAs of a pair) leaves its first pipeline stage
unfilled (no copies, no arrival): the wait on it is a flag that nothing sets.  The wait must give up after its limit, the
kernel must drain what it had in flight and return, the device status must
read MXF8_ERR_TIMEOUT, and the context must stay usable: the next launch
without the hook produces the oracle's result."""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.helpers import np_u8

pytestmark = pytest.mark.gpu

TIMEOUT = 6   # MXF8_ERR_TIMEOUT


@pytest.fixture(scope="module")
def mx():
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert m.mxfp8_device_supported(), "GPU tests need an sm_100 device"
    return m


@pytest.fixture
def tiling(mx, request):
    mx.mxfp8_set_gemm_tiling(*request.param)
    yield request.param
    mx.mxfp8_set_gemm_tiling(-1, -1)


def _operands(mx, counts, N, K):
    offs = wl.offsets_from_counts(counts)
    M = int(offs[-1])
    X = wl.normal_bf16((M, K), 1.0, 71)
    W = wl.normal_bf16((len(counts) * N, K), 0.05, 72)
    dY = wl.normal_bf16((M, N), 1.0, 73)
    return offs, M, X, W, dY


# 1-CTA tiles (the library's rule at these sizes) and CTA pairs with both stage depths
@pytest.mark.parametrize("tiling", [(-1, -1), (1, 1), (1, 2)], indirect=True, ids=["1cta", "pair-ks1", "pair-ks2"])
def test_unfilled_stage_times_out_and_the_context_stays_usable(mx, tiling):
    counts = [0, 150, 300, 62]
    E, N, K = len(counts), 256, 512
    offs, M, X, W, _ = _operands(mx, counts, N, K)
    od = torch.from_numpy(offs).cuda()
    xq, xs = mx.mxfp8_quantize_rowwise(X.cuda(), od)
    wq, ws = mx.mxfp8_quantize_rowwise(W.cuda())
    work = mx.new_workspace(E, M, N, K)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")

    mx.mxfp8_testing_stall_first_stage(True)
    try:
        mx.mxfp8_grouped_gemm_fwd(xq, xs, wq, ws, od, N, out=y, work=work)
        torch.cuda.synchronize()
    finally:
        mx.mxfp8_testing_stall_first_stage(False)
    assert mx.mxfp8_get_status(work) == TIMEOUT

    mx.mxfp8_grouped_gemm_fwd(xq, xs, wq, ws, od, N, out=y, work=work)
    torch.cuda.synchronize()
    assert mx.mxfp8_get_status(work) == 0
    Xd = oracle.dequantize_rowwise(np_u8(xq), np_u8(xs), offs)
    Wd = oracle.dequantize_rowwise(np_u8(wq), np_u8(ws)).reshape(E, N, K)
    ref = oracle.gemm_fwd(Xd, Wd, offs)
    got = y.double().cpu().numpy()
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err <= 5e-3


def test_wgrad_unfilled_stage_times_out_and_the_context_stays_usable(mx):
    """wgrad tiles have per-expert K loops (an empty expert has none): the
    stop still reaches every role."""
    counts = [0, 150, 300, 62]
    E, N, K = len(counts), 256, 512
    offs, M, X, _, dY = _operands(mx, counts, N, K)
    od = torch.from_numpy(offs).cuda()
    dyqT, dysT = mx.mxfp8_quantize_colwise(dY.cuda(), od)
    xqT, xsT = mx.mxfp8_quantize_colwise(X.cuda(), od)
    work = mx.new_workspace(E, M, N, K)
    dw = torch.full((E, N, K), float("nan"), dtype=torch.bfloat16, device="cuda")
    mx.mxfp8_testing_stall_first_stage(True)
    try:
        mx.mxfp8_grouped_gemm_wgrad(dyqT, dysT, xqT, xsT, od, M, out=dw, work=work)
        torch.cuda.synchronize()
    finally:
        mx.mxfp8_testing_stall_first_stage(False)
    assert mx.mxfp8_get_status(work) == TIMEOUT
    mx.mxfp8_grouped_gemm_wgrad(dyqT, dysT, xqT, xsT, od, M, out=dw, work=work)
    torch.cuda.synchronize()
    assert mx.mxfp8_get_status(work) == 0
    dYd = oracle.dequantize_colwise(np_u8(dyqT), np_u8(dysT), M, offs)
    Xd = oracle.dequantize_colwise(np_u8(xqT), np_u8(xsT), M, offs)
    ref = oracle.gemm_wgrad(dYd, Xd, offs)
    got = dw.double().cpu().numpy()
    assert np.all(got[0] == 0)
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err <= 5e-3
