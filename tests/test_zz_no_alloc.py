"""The forward grouped GEMM entry point that allocates nothing.

Some callers cannot hand the library a workspace: a plugin inside an engine
that owns the whole device-memory budget and forbids cudaMalloc, or a loop
that cannot afford the device synchronisation an allocation may cause.
mxfp8_grouped_gemm_fwd_noalloc serves them from a static scratch array built
into the library.  This test calls it through the C ABI twice in a row (the
second call reuses the scratch the first one left behind) and checks each
result against the ordinary mxfp8_grouped_gemm_fwd: the same kernel on the
same bytes, so the outputs must be identical bit for bit (tighter than the
GEMM tolerance the other tests use).  It lives in its own file, collected last, and passes
whether it runs alone in a fresh process or after the rest of the suite.
"""
import ctypes

import pytest
import torch

from mxfp8_grouped_gemm_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_noalloc_forward_matches_workspace_forward_twice():
    import mxfp8_grouped_gemm_quantize_b200 as mx
    assert torch.cuda.is_available() and mx.mxfp8_device_supported(), "needs an sm_100 GPU"
    counts = [0, 7, 130, 300, 33, 1]
    offs = wl.offsets_from_counts(counts)
    M, E, N, K = int(offs[-1]), len(counts), 384, 416
    X = wl.normal_bf16((M, K), 1.0, 41).cuda()
    W = wl.normal_bf16((E * N, K), 0.5, 42).cuda()
    od = torch.from_numpy(offs).cuda()
    xq, xs = mx.mxfp8_quantize_rowwise(X, od)
    wq, ws = mx.mxfp8_quantize_rowwise(W)
    ref = mx.mxfp8_grouped_gemm_fwd(xq, xs, wq, ws, od, N)
    torch.cuda.synchronize()

    L = mx.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = ctypes.c_int32(-1)
        rc = L.mxfp8_grouped_gemm_fwd_noalloc(xq.data_ptr(), xs.data_ptr(), xs.numel(), wq.data_ptr(),
                                              ws.data_ptr(), ws.numel(), od.data_ptr(), E, M, N, K,
                                              y.data_ptr(), ctypes.byref(status), stream)
        assert rc == 0, f"call {call}: {mx.lib().mxfp8_status_string(rc).decode()}"
        assert status.value == 0, f"call {call}: device status {status.value}"
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), f"call {call}: output differs from the forward"
