"""MXFP8 quantisation and dropless grouped GEMM for B200 (sm_100a).

A thin ctypes binding over ``libmxfp8.so`` (the C ABI in ``include/mxfp8.h``).
The functions carry the C names and only marshal arguments: PyTorch supplies
device memory and the current stream, every step runs in the library's CUDA
kernels.  There is no fallback: if the library is missing or the device is not
sm_100 the calls raise.

MXFP8 = 32-element blocks sharing one power-of-two scale (opensourcebeat.com,
"Enabling up to 41% faster pre-training: MXFP8 and DeepEP ...", FAQ), with the
OCP MX v1.0 E8M0/E4M3 rules; the grouped GEMM runs every expert on its real
token count (iitak.ru, "NVIDIA ... JAX", Transformer Engine paragraph).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxfp8.so")
_LIB = None

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_vp = ctypes.c_void_p

MXF8_OK = 0
MXF8_GEMM_MAX_GROUPS = 256
STATUS_NAMES = {0: "MXF8_OK", 1: "MXF8_ERR_INVALID_ARG", 2: "MXF8_ERR_ALIGNMENT", 3: "MXF8_ERR_UNSUPPORTED",
                4: "MXF8_ERR_CUDA", 5: "MXF8_ERR_BAD_OFFSETS", 6: "MXF8_ERR_TIMEOUT", 7: "MXF8_ERR_BAD_ROUTING"}

EXPORTED = ("mxfp8_rowwise_scale_bytes", "mxfp8_colwise_pitch", "mxfp8_colwise_scale_bytes", "mxfp8_colwise_ld",
            "mxfp8_workspace_bytes", "mxfp8_quantize_rowwise", "mxfp8_quantize_colwise",
            "mxfp8_grouped_gemm_fwd", "mxfp8_grouped_gemm_dgrad", "mxfp8_grouped_gemm_wgrad",
            "mxfp8_get_status", "mxfp8_status_string", "mxfp8_last_cuda_error", "mxfp8_device_supported",
            "mxfp8_grouped_gemm_fwd_noalloc", "mxfp8_quantize_dual", "mxfp8_grouped_gemm_fwd_quant",
            "mxfp8_grouped_gemm_dgrad_quant", "mxfp8_moe_plan_workspace_bytes", "mxfp8_moe_plan",
            "mxfp8_permute_quantize_dual", "mxfp8_moe_combine", "mxfp8_nvfp4_rowwise_scale_bytes",
            "mxfp8_nvfp4_colwise_pitch", "mxfp8_nvfp4_colwise_scale_bytes", "mxfp8_nvfp4_colwise_ld",
            "mxfp8_nvfp4_amax", "mxfp8_nvfp4_quantize_rowwise", "mxfp8_nvfp4_quantize_colwise",
            "mxfp8_nvfp4_grouped_gemm_fwd", "mxfp8_nvfp4_grouped_gemm_dgrad", "mxfp8_nvfp4_grouped_gemm_wgrad",
            "mxfp8_set_gemm_tiling", "mxfp8_testing_stall_first_stage", "mxfp8_grouped_gemm_fwd_swiglu",
            "mxfp8_ep_record_bytes", "mxfp8_ep_plan_workspace_bytes", "mxfp8_ep_plan", "mxfp8_ep_pack",
            "mxfp8_ep_unpack", "mxfp8_gather_rows")


class MXFP8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if _LIB is not None:
            detail = _LIB.mxfp8_status_string(status).decode()
            if status == 4:
                detail += ": " + _LIB.mxfp8_last_cuda_error().decode()
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({detail})")


def lib() -> ctypes.CDLL:
    """Loads libmxfp8.so; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mxfp8_grouped_gemm_quantize_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for n in ("mxfp8_rowwise_scale_bytes", "mxfp8_colwise_scale_bytes"):
            getattr(L, n).restype = _i64
            getattr(L, n).argtypes = [_i64, _i64, _i32]
        for n in ("mxfp8_colwise_pitch", "mxfp8_colwise_ld"):
            getattr(L, n).restype = _i64
            getattr(L, n).argtypes = [_i64, _i32]
        L.mxfp8_workspace_bytes.restype = _i64
        L.mxfp8_workspace_bytes.argtypes = [_i32, _i64, _i64, _i64]
        L.mxfp8_quantize_rowwise.restype = _i32
        L.mxfp8_quantize_rowwise.argtypes = [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _i64, _vp]
        L.mxfp8_quantize_colwise.restype = _i32
        L.mxfp8_quantize_colwise.argtypes = [_vp, _i64, _i64, _vp, _i32, _vp, _i64, _vp, _i64, _vp]
        L.mxfp8_quantize_dual.restype = _i32
        L.mxfp8_quantize_dual.argtypes = [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _i64, _vp, _i64, _vp, _i64, _vp]
        for n in ("mxfp8_grouped_gemm_fwd", "mxfp8_grouped_gemm_dgrad", "mxfp8_grouped_gemm_wgrad"):
            getattr(L, n).restype = _i32
            getattr(L, n).argtypes = [_vp, _vp, _i64, _vp, _vp, _i64, _vp, _i32, _i64, _i64, _i64, _vp, _vp, _i64, _vp]
        for n in ("mxfp8_grouped_gemm_fwd_quant", "mxfp8_grouped_gemm_dgrad_quant", "mxfp8_grouped_gemm_fwd_swiglu"):
            getattr(L, n).restype = _i32
            getattr(L, n).argtypes = [_vp, _vp, _i64, _vp, _vp, _i64, _vp, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _i64,
                                      _vp, _i64, _vp, _i64, _vp, _i64, _vp]
        L.mxfp8_moe_plan_workspace_bytes.restype = _i64
        L.mxfp8_moe_plan_workspace_bytes.argtypes = [_i64, _i32, _i32]
        L.mxfp8_moe_plan.restype = _i32
        L.mxfp8_moe_plan.argtypes = [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _i64, _vp]
        L.mxfp8_permute_quantize_dual.restype = _i32
        L.mxfp8_permute_quantize_dual.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _i32, _vp, _vp, _i64, _vp, _i64,
                                                  _vp, _i64, _vp]
        L.mxfp8_moe_combine.restype = _i32
        L.mxfp8_moe_combine.argtypes = [_vp, _i64, _i64, _vp, _vp, _i64, _i32, _vp, _vp]
        for n in ("mxfp8_nvfp4_rowwise_scale_bytes", "mxfp8_nvfp4_colwise_scale_bytes"):
            getattr(L, n).restype = _i64
            getattr(L, n).argtypes = [_i64, _i64, _i32]
        for n in ("mxfp8_nvfp4_colwise_pitch", "mxfp8_nvfp4_colwise_ld"):
            getattr(L, n).restype = _i64
            getattr(L, n).argtypes = [_i64, _i32]
        L.mxfp8_nvfp4_amax.restype = _i32
        L.mxfp8_nvfp4_amax.argtypes = [_vp, _i64, _vp, _vp]
        L.mxfp8_nvfp4_quantize_rowwise.restype = _i32
        L.mxfp8_nvfp4_quantize_rowwise.argtypes = [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _i64, _vp]
        L.mxfp8_nvfp4_quantize_colwise.restype = _i32
        L.mxfp8_nvfp4_quantize_colwise.argtypes = [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _i64, _vp, _i64, _vp]
        for n in ("mxfp8_nvfp4_grouped_gemm_fwd", "mxfp8_nvfp4_grouped_gemm_dgrad", "mxfp8_nvfp4_grouped_gemm_wgrad"):
            getattr(L, n).restype = _i32
            getattr(L, n).argtypes = [_vp, _vp, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _i32, _i64, _i64, _i64, _vp,
                                      _vp, _i64, _vp]
        L.mxfp8_grouped_gemm_fwd_noalloc.restype = _i32
        L.mxfp8_grouped_gemm_fwd_noalloc.argtypes = [_vp, _vp, _i64, _vp, _vp, _i64, _vp, _i32, _i64, _i64, _i64, _vp,
                                                     ctypes.POINTER(_i32), _vp]
        L.mxfp8_ep_record_bytes.restype = _i64
        L.mxfp8_ep_record_bytes.argtypes = [_i64]
        L.mxfp8_ep_plan_workspace_bytes.restype = _i64
        L.mxfp8_ep_plan_workspace_bytes.argtypes = [_i64, _i32]
        L.mxfp8_ep_plan.restype = _i32
        L.mxfp8_ep_plan.argtypes = [_vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp]
        L.mxfp8_ep_pack.restype = _i32
        L.mxfp8_ep_pack.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _vp]
        L.mxfp8_ep_unpack.restype = _i32
        L.mxfp8_ep_unpack.argtypes = [_vp, _i64, _i64, _vp, _vp, _i32, _vp, _i64, _vp, _i32, _vp, _vp, _i64, _vp]
        L.mxfp8_gather_rows.restype = _i32
        L.mxfp8_gather_rows.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp, _vp]
        L.mxfp8_get_status.restype = _i32
        L.mxfp8_get_status.argtypes = [_vp, _vp, ctypes.POINTER(_i32)]
        L.mxfp8_status_string.restype = ctypes.c_char_p
        L.mxfp8_status_string.argtypes = [_i32]
        L.mxfp8_last_cuda_error.restype = ctypes.c_char_p
        L.mxfp8_device_supported.restype = _i32
        L.mxfp8_set_gemm_tiling.restype = _i32
        L.mxfp8_set_gemm_tiling.argtypes = [_i32, _i32]
        L.mxfp8_testing_stall_first_stage.restype = None
        L.mxfp8_testing_stall_first_stage.argtypes = [_i32]
        _LIB = L
    return _LIB


def _check(status: int, where: str):
    if status != MXF8_OK:
        raise MXFP8Error(status, where)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors"
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _groups(offs: torch.Tensor | None) -> int:
    if offs is None:
        return 1
    assert offs.dtype == torch.int32 and offs.is_cuda
    return offs.numel() - 1


# ------------------------------------------------------------------ sizes
def mxfp8_rowwise_scale_bytes(rows: int, cols: int, num_groups: int = 1) -> int:
    return lib().mxfp8_rowwise_scale_bytes(rows, cols, num_groups)


def mxfp8_colwise_pitch(rows: int, num_groups: int = 1) -> int:
    return lib().mxfp8_colwise_pitch(rows, num_groups)


def mxfp8_colwise_scale_bytes(rows: int, cols: int, num_groups: int = 1) -> int:
    return lib().mxfp8_colwise_scale_bytes(rows, cols, num_groups)


def mxfp8_colwise_ld(rows: int, num_groups: int = 1) -> int:
    return lib().mxfp8_colwise_ld(rows, num_groups)


def mxfp8_workspace_bytes(num_groups: int, M: int, N: int, K: int) -> int:
    return lib().mxfp8_workspace_bytes(num_groups, M, N, K)


def _u8(n: int, device) -> torch.Tensor:
    return torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ quantisers
def mxfp8_quantize_rowwise(x: torch.Tensor, offs: torch.Tensor | None = None, q=None, scales=None, stream=None):
    """x: bf16 [rows, cols] -> (q uint8 [rows, cols], scales uint8 atoms)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    R, C = x.shape
    G = _groups(offs)
    q = q if q is not None else torch.empty((R, C), dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else _u8(mxfp8_rowwise_scale_bytes(R, C, G), x.device)
    _check(lib().mxfp8_quantize_rowwise(_ptr(x), R, C, _ptr(offs), G, _ptr(q), _ptr(scales), scales.numel(),
                                        _stream(stream)), "mxfp8_quantize_rowwise")
    return q, scales


def mxfp8_quantize_colwise(x: torch.Tensor, offs: torch.Tensor | None = None, qT=None, scales=None, stream=None):
    """x: bf16 [rows, cols] -> (qT uint8 [cols, ldT], scales uint8 atoms)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    R, C = x.shape
    G = _groups(offs)
    ld = mxfp8_colwise_ld(R, G)
    qT = qT if qT is not None else torch.empty((C, ld), dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else _u8(mxfp8_colwise_scale_bytes(R, C, G), x.device)
    _check(lib().mxfp8_quantize_colwise(_ptr(x), R, C, _ptr(offs), G, _ptr(qT), ld, _ptr(scales), scales.numel(),
                                        _stream(stream)), "mxfp8_quantize_colwise")
    return qT, scales


def mxfp8_quantize_dual(x: torch.Tensor, offs: torch.Tensor | None = None, q=None, scales=None, qT=None,
                        scalesT=None, stream=None):
    """x: bf16 [rows, cols] -> (q, scales, qT, scalesT): both layouts from one read."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    R, C = x.shape
    G = _groups(offs)
    ld = mxfp8_colwise_ld(R, G)
    q = q if q is not None else torch.empty((R, C), dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else _u8(mxfp8_rowwise_scale_bytes(R, C, G), x.device)
    qT = qT if qT is not None else torch.empty((C, ld), dtype=torch.uint8, device=x.device)
    scalesT = scalesT if scalesT is not None else _u8(mxfp8_colwise_scale_bytes(R, C, G), x.device)
    _check(lib().mxfp8_quantize_dual(_ptr(x), R, C, _ptr(offs), G, _ptr(q), _ptr(scales), scales.numel(), _ptr(qT),
                                     ld, _ptr(scalesT), scalesT.numel(), _stream(stream)), "mxfp8_quantize_dual")
    return q, scales, qT, scalesT


# ------------------------------------------------------------------ grouped GEMMs
def new_workspace(E: int, M: int, N: int, K: int, device="cuda") -> torch.Tensor:
    return torch.zeros(mxfp8_workspace_bytes(E, M, N, K), dtype=torch.uint8, device=device)


def _gemm(fn: str, a, as_, b, bs, offs, M, N, K, out, work, stream):
    E = _groups(offs)
    work = work if work is not None else new_workspace(E, M, N, K, out.device)
    _check(getattr(lib(), fn)(_ptr(a), _ptr(as_), as_.numel(), _ptr(b), _ptr(bs), bs.numel(), _ptr(offs), E,
                              M, N, K, _ptr(out), _ptr(work), work.numel(), _stream(stream)), fn)
    return out


def mxfp8_grouped_gemm_fwd(xq, xs, wq, ws, offs, N: int, out=None, work=None, stream=None):
    """Y[M, N] = X_e W_e^T per expert.  xq/xs rowwise(X, offs); wq/ws rowwise(W as [E*N, K])."""
    M, K = xq.shape
    out = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    return _gemm("mxfp8_grouped_gemm_fwd", xq, xs, wq, ws, offs, M, N, K, out, work, stream)


def mxfp8_grouped_gemm_dgrad(dyq, dys, wqT, wsT, offs, K: int, out=None, work=None, stream=None):
    """dX[M, K] = dY_e W_e.  dyq/dys rowwise(dY, offs); wqT/wsT colwise(W as [E*N, K])."""
    M, N = dyq.shape
    out = out if out is not None else torch.empty((M, K), dtype=torch.bfloat16, device=dyq.device)
    return _gemm("mxfp8_grouped_gemm_dgrad", dyq, dys, wqT, wsT, offs, M, N, K, out, work, stream)


def mxfp8_grouped_gemm_wgrad(dyqT, dysT, xqT, xsT, offs, M: int, out=None, work=None, stream=None):
    """dW[E, N, K] = dY_e^T X_e.  dyqT/dysT colwise(dY, offs); xqT/xsT colwise(X, offs)."""
    N, K = dyqT.shape[0], xqT.shape[0]
    E = _groups(offs)
    out = out if out is not None else torch.empty((E, N, K), dtype=torch.bfloat16, device=dyqT.device)
    return _gemm("mxfp8_grouped_gemm_wgrad", dyqT, dysT, xqT, xsT, offs, M, N, K, out, work, stream)


def _gemm_quant(fn, a, a_s, b, b_s, offs, M, N, K, C, out, rowwise, colwise, work, stream):
    E = _groups(offs)
    dev = a.device
    q = scales = qT = scalesT = None
    ld = mxfp8_colwise_ld(M, E)
    if rowwise is True:
        rowwise = (torch.empty((M, C), dtype=torch.uint8, device=dev), _u8(mxfp8_rowwise_scale_bytes(M, C, E), dev))
    if rowwise:
        q, scales = rowwise
    if colwise is True:
        colwise = (torch.empty((C, ld), dtype=torch.uint8, device=dev), _u8(mxfp8_colwise_scale_bytes(M, C, E), dev))
    if colwise:
        qT, scalesT = colwise
    work = work if work is not None else new_workspace(E, M, N, K, dev)
    _check(getattr(lib(), fn)(_ptr(a), _ptr(a_s), a_s.numel(), _ptr(b), _ptr(b_s), b_s.numel(), _ptr(offs), E, M, N,
                              K, _ptr(out), _ptr(q), _ptr(scales), scales.numel() if scales is not None else 0,
                              _ptr(qT), ld, _ptr(scalesT), scalesT.numel() if scalesT is not None else 0,
                              _ptr(work), work.numel(), _stream(stream)), fn)
    return out, q, scales, qT, scalesT


def mxfp8_grouped_gemm_fwd_quant(xq, xs, wq, ws, offs, N: int, out=True, rowwise=True, colwise=True, work=None,
                                 stream=None):
    """Forward GEMM whose epilogue also writes Y as MXFP8, byte for byte what
    mxfp8_quantize_rowwise / _colwise(Y, offs) give.  out / rowwise / colwise:
    True = allocate, False/None = skip, or the buffers ((q, scales) and
    (qT, scalesT) for the quantised copies).  Returns (y, q, scales, qT, scalesT)."""
    M, K = xq.shape
    if out is True:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    return _gemm_quant("mxfp8_grouped_gemm_fwd_quant", xq, xs, wq, ws, offs, M, N, K, N, out if isinstance(out, torch.Tensor) else None, rowwise,
                       colwise, work, stream)


def mxfp8_grouped_gemm_dgrad_quant(dyq, dys, wqT, wsT, offs, K: int, out=True, rowwise=True, colwise=True,
                                   work=None, stream=None):
    """Dgrad GEMM whose epilogue also writes dX as MXFP8 (see
    mxfp8_grouped_gemm_fwd_quant).  Returns (dx, q, scales, qT, scalesT)."""
    M, N = dyq.shape
    if out is True:
        out = torch.empty((M, K), dtype=torch.bfloat16, device=dyq.device)
    return _gemm_quant("mxfp8_grouped_gemm_dgrad_quant", dyq, dys, wqT, wsT, offs, M, N, K, K, out if isinstance(out, torch.Tensor) else None, rowwise,
                       colwise, work, stream)


def mxfp8_grouped_gemm_fwd_swiglu(xq, xs, wq, ws, offs, N: int, out=True, rowwise=True, colwise=True, work=None,
                                  stream=None):
    """Gate/up forward GEMM fused with SwiGLU: h = silu(Y[:, :N/2]) * Y[:, N/2:]
    for Y = X_e W_e^T, written as bf16 [M, N/2] and/or MXFP8 (the bytes
    mxfp8_quantize_rowwise / _colwise(h, offs) give).  Arguments as
    mxfp8_grouped_gemm_fwd_quant.  Returns (h, q, scales, qT, scalesT)."""
    M, K = xq.shape
    if out is True:
        out = torch.empty((M, N // 2), dtype=torch.bfloat16, device=xq.device)
    return _gemm_quant("mxfp8_grouped_gemm_fwd_swiglu", xq, xs, wq, ws, offs, M, N, K, N // 2,
                       out if isinstance(out, torch.Tensor) else None, rowwise, colwise, work, stream)


def mxfp8_grouped_gemm_fwd_noalloc(xq, xs, wq, ws, offs, N: int, out=None, stream=None, want_status=False):
    """Forward grouped GEMM with the library's static scratch instead of a
    workspace, for callers that cannot allocate device memory.  With
    want_status the call synchronises the stream and returns (out, status)."""
    M, K = xq.shape
    E = _groups(offs)
    out = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    st = _i32(-1)
    _check(lib().mxfp8_grouped_gemm_fwd_noalloc(_ptr(xq), _ptr(xs), xs.numel(), _ptr(wq), _ptr(ws), ws.numel(),
                                                _ptr(offs), E, M, N, K, _ptr(out),
                                                ctypes.byref(st) if want_status else None, _stream(stream)),
           "mxfp8_grouped_gemm_fwd_noalloc")
    return (out, int(st.value)) if want_status else out


def mxfp8_get_status(work: torch.Tensor, stream=None) -> int:
    st = _i32(0)
    _check(lib().mxfp8_get_status(_ptr(work), _stream(stream), ctypes.byref(st)), "mxfp8_get_status")
    return int(st.value)


def mxfp8_device_supported() -> bool:
    return bool(lib().mxfp8_device_supported())


def mxfp8_set_gemm_tiling(cta_pair: int = -1, stage_k: int = -1) -> None:
    """Process-wide override of the grouped GEMMs' tile configuration
    (-1 = the library's rule; cta_pair 0/1 = 1-CTA / CTA-pair tiles; stage_k
    1/2 = 128- / 256-deep K stages).  Results do not change, only speed."""
    _check(lib().mxfp8_set_gemm_tiling(int(cta_pair), int(stage_k)), "mxfp8_set_gemm_tiling")


def mxfp8_testing_stall_first_stage(enable: bool) -> None:
    """Test switch: while on, every grouped GEMM launch leaves its first
    pipeline stage unfilled and ends with MXF8_ERR_TIMEOUT after its 2 s
    bounded wait (the workspace status reports it)."""
    lib().mxfp8_testing_stall_first_stage(1 if enable else 0)


# ------------------------------------------------------------------ MoE dispatch / combine
def mxfp8_moe_plan(idx: torch.Tensor, num_experts: int, work=None, stream=None):
    """idx: int32 [T, k] expert ids -> (offs int32 [E+1], perm int32 [T*k], inv int32 [T, k], work).
    Pairs grouped by expert in ascending (token, slot) order; mxfp8_get_status(work) reports ids out of range."""
    assert idx.dtype == torch.int32 and idx.dim() == 2
    T, k = idx.shape
    dev = idx.device
    offs = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)[: T * k]
    inv = torch.empty((T, k), dtype=torch.int32, device=dev)
    need = lib().mxfp8_moe_plan_workspace_bytes(T, k, num_experts)
    work = work if work is not None else torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib().mxfp8_moe_plan(_ptr(idx), T, k, num_experts, _ptr(offs), _ptr(perm), _ptr(inv), _ptr(work),
                                work.numel(), _stream(stream)), "mxfp8_moe_plan")
    return offs, perm, inv, work


def mxfp8_permute_quantize_dual(x: torch.Tensor, perm: torch.Tensor, offs: torch.Tensor, q=None, scales=None, qT=None,
                                scalesT=None, stream=None):
    """Quantises Xp = x[perm] (grouped by offs) into both MXFP8 layouts without
    materialising Xp -> (q, scales, qT, scalesT), as mxfp8_quantize_dual(x[perm], offs)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and perm.dtype == torch.int32
    T, C = x.shape
    R = perm.numel()
    G = _groups(offs)
    ld = mxfp8_colwise_ld(R, G)
    q = q if q is not None else torch.empty((R, C), dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else _u8(mxfp8_rowwise_scale_bytes(R, C, G), x.device)
    qT = qT if qT is not None else torch.empty((C, ld), dtype=torch.uint8, device=x.device)
    scalesT = scalesT if scalesT is not None else _u8(mxfp8_colwise_scale_bytes(R, C, G), x.device)
    _check(lib().mxfp8_permute_quantize_dual(_ptr(x), T, C, _ptr(perm) if R else None, R, _ptr(offs), G, _ptr(q),
                                             _ptr(scales), scales.numel(), _ptr(qT), ld, _ptr(scalesT),
                                             scalesT.numel(), _stream(stream)), "mxfp8_permute_quantize_dual")
    return q, scales, qT, scalesT


def mxfp8_moe_combine(yp: torch.Tensor, inv: torch.Tensor, w: torch.Tensor, out=None, stream=None):
    """y[t] = sum_j w[t, j] * yp[inv[t, j]] (fp64 sum, one bf16 rounding) -> bf16 [T, cols]."""
    assert yp.dtype == torch.bfloat16 and inv.dtype == torch.int32 and w.dtype == torch.float32
    rows, C = yp.shape
    T, k = inv.shape
    out = out if out is not None else torch.empty((T, C), dtype=torch.bfloat16, device=yp.device)
    _check(lib().mxfp8_moe_combine(_ptr(yp) if rows else None, rows, C, _ptr(inv), _ptr(w), T, k, _ptr(out),
                                   _stream(stream)), "mxfp8_moe_combine")
    return out


# ------------------------------------------------------------------ expert-parallel dispatch
def mxfp8_ep_record_bytes(cols: int) -> int:
    return int(lib().mxfp8_ep_record_bytes(cols))


def mxfp8_ep_plan(idx: torch.Tensor, num_experts: int, num_ranks: int, work=None, stream=None):
    """idx: int32 [T, k] global expert ids -> (counts int32 [2P], rec_token int32 [T*min(k,P)],
    pair_expert int32 [T*k], pair_rec int32 [T*k], ret_pos int32 [T, k], work); the first
    sum(counts[:P]) records and sum(counts[P:]) pairs are written."""
    assert idx.dtype == torch.int32 and idx.dim() == 2
    T, k = idx.shape
    dev = idx.device
    P = num_ranks
    counts = torch.empty(2 * P, dtype=torch.int32, device=dev)
    rec_token = torch.empty(max(T * min(k, P), 1), dtype=torch.int32, device=dev)
    pair_expert = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    pair_rec = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    ret_pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    need = lib().mxfp8_ep_plan_workspace_bytes(T, P)
    work = work if work is not None else torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib().mxfp8_ep_plan(_ptr(idx) if T else None, T, k, num_experts, P, _ptr(counts), _ptr(rec_token),
                               _ptr(pair_expert), _ptr(pair_rec), _ptr(ret_pos) if T else None, _ptr(work),
                               work.numel(), _stream(stream)), "mxfp8_ep_plan")
    return counts, rec_token, pair_expert, pair_rec, ret_pos, work


def mxfp8_ep_pack(x: torch.Tensor, rec_token: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """x: bf16 [T, cols]; rec_token int32 [R] -> records uint8 [R, mxfp8_ep_record_bytes(cols)]."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and rec_token.dtype == torch.int32
    T, C = x.shape
    R = rec_token.numel()
    out = out if out is not None else torch.empty((R, mxfp8_ep_record_bytes(C)), dtype=torch.uint8, device=x.device)
    _check(lib().mxfp8_ep_pack(_ptr(x) if x.numel() else None, T, C, _ptr(rec_token) if R else None, R,
                               _ptr(out) if R else None, _stream(stream)), "mxfp8_ep_pack")
    return out


def mxfp8_ep_unpack(records: torch.Tensor, cols: int, pair_rec: torch.Tensor, src_base: torch.Tensor,
                    perm: torch.Tensor, offs: torch.Tensor, q=None, scales=None, stream=None):
    """Received records and pair entries -> (q uint8 [rows, cols], scales): the grouped rows'
    rowwise MXFP8; src_base int32 [2(P+1)] on the device (first pair, then first record, of each source)."""
    assert records.dtype == torch.uint8 and pair_rec.dtype == torch.int32 and perm.dtype == torch.int32
    assert src_base.dtype == torch.int32 and src_base.is_cuda
    R = records.shape[0]
    rows = perm.numel()
    G = _groups(offs)
    P = src_base.numel() // 2 - 1
    dev = records.device
    q = q if q is not None else torch.empty((rows, cols), dtype=torch.uint8, device=dev)
    scales = scales if scales is not None else _u8(mxfp8_rowwise_scale_bytes(rows, cols, G), dev)
    _check(lib().mxfp8_ep_unpack(_ptr(records) if R else None, R, cols, _ptr(pair_rec) if rows else None,
                                 _ptr(src_base), P, _ptr(perm) if rows else None, rows, _ptr(offs), G,
                                 _ptr(q) if rows else None, _ptr(scales), scales.numel(), _stream(stream)),
           "mxfp8_ep_unpack")
    return q, scales


def mxfp8_gather_rows(src: torch.Tensor, idx: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """out[i] = src[idx[i]] (rows of a 2-D tensor; zero rows for indices out of range)."""
    assert src.dim() == 2 and idx.dtype == torch.int32
    n = idx.numel()
    row_bytes = src.shape[1] * src.element_size()
    out = out if out is not None else torch.empty((n, src.shape[1]), dtype=src.dtype, device=src.device)
    _check(lib().mxfp8_gather_rows(_ptr(src) if src.numel() else None, src.shape[0], row_bytes,
                                   _ptr(idx) if n else None, n, _ptr(out) if n else None, _stream(stream)),
           "mxfp8_gather_rows")
    return out


# ------------------------------------------------------------------ NVFP4
def mxfp8_nvfp4_amax(x: torch.Tensor, amax=None, stream=None) -> torch.Tensor:
    """Largest |x| of a bf16 tensor -> fp32 device scalar (shape [1])."""
    assert x.dtype == torch.bfloat16
    amax = amax if amax is not None else torch.empty(1, dtype=torch.float32, device=x.device)
    _check(lib().mxfp8_nvfp4_amax(_ptr(x) if x.numel() else None, x.numel(), _ptr(amax), _stream(stream)),
           "mxfp8_nvfp4_amax")
    return amax


def mxfp8_nvfp4_quantize_rowwise(x, amax, offs=None, q=None, scales=None, stream=None):
    """x: bf16 [rows, cols] -> (q uint8 [rows, cols/2], scales); amax from mxfp8_nvfp4_amax."""
    R, C = x.shape
    G = _groups(offs)
    q = q if q is not None else torch.empty((R, C // 2), dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else _u8(lib().mxfp8_nvfp4_rowwise_scale_bytes(R, C, G), x.device)
    _check(lib().mxfp8_nvfp4_quantize_rowwise(_ptr(x), R, C, _ptr(offs), G, _ptr(amax), _ptr(q), _ptr(scales),
                                              scales.numel(), _stream(stream)), "mxfp8_nvfp4_quantize_rowwise")
    return q, scales


def mxfp8_nvfp4_quantize_colwise(x, amax, offs=None, qT=None, scales=None, stream=None):
    """x: bf16 [rows, cols] -> (qT uint8 [cols, ld/2], scales); ld = mxfp8_nvfp4_colwise_ld(rows, G) elements."""
    R, C = x.shape
    G = _groups(offs)
    ld = lib().mxfp8_nvfp4_colwise_ld(R, G)
    qT = qT if qT is not None else torch.empty((C, ld // 2), dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else _u8(lib().mxfp8_nvfp4_colwise_scale_bytes(R, C, G), x.device)
    _check(lib().mxfp8_nvfp4_quantize_colwise(_ptr(x), R, C, _ptr(offs), G, _ptr(amax), _ptr(qT), ld, _ptr(scales),
                                              scales.numel(), _stream(stream)), "mxfp8_nvfp4_quantize_colwise")
    return qT, scales


def _nvfp4_gemm(fn, a, a_s, a_amax, b, b_s, b_amax, offs, M, N, K, out, work, stream):
    E = _groups(offs)
    work = work if work is not None else new_workspace(E, M, N, K, out.device)
    _check(getattr(lib(), fn)(_ptr(a), _ptr(a_s), a_s.numel(), _ptr(a_amax), _ptr(b), _ptr(b_s), b_s.numel(),
                              _ptr(b_amax), _ptr(offs), E, M, N, K, _ptr(out), _ptr(work), work.numel(),
                              _stream(stream)), fn)
    return out


def mxfp8_nvfp4_grouped_gemm_fwd(xq, xs, x_amax, wq, ws, w_amax, offs, N: int, out=None, work=None, stream=None):
    """Y[M, N] from NVFP4 rowwise(X, offs) [M, K/2] and rowwise(W as [E*N, K]) with their amaxes."""
    M, K = xq.shape[0], xq.shape[1] * 2
    out = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    return _nvfp4_gemm("mxfp8_nvfp4_grouped_gemm_fwd", xq, xs, x_amax, wq, ws, w_amax, offs, M, N, K, out, work,
                       stream)


def mxfp8_nvfp4_grouped_gemm_dgrad(dyq, dys, dy_amax, wqT, wsT, w_amax, offs, K: int, out=None, work=None,
                                   stream=None):
    """dX[M, K] from NVFP4 rowwise(dY, offs) and colwise(W as [E*N, K])."""
    M, N = dyq.shape[0], dyq.shape[1] * 2
    out = out if out is not None else torch.empty((M, K), dtype=torch.bfloat16, device=dyq.device)
    return _nvfp4_gemm("mxfp8_nvfp4_grouped_gemm_dgrad", dyq, dys, dy_amax, wqT, wsT, w_amax, offs, M, N, K, out,
                       work, stream)


def mxfp8_nvfp4_grouped_gemm_wgrad(dyqT, dysT, dy_amax, xqT, xsT, x_amax, offs, M: int, out=None, work=None,
                                   stream=None):
    """dW[E, N, K] from NVFP4 colwise(dY, offs) and colwise(X, offs)."""
    N, K = dyqT.shape[0], xqT.shape[0]
    E = _groups(offs)
    out = out if out is not None else torch.empty((E, N, K), dtype=torch.bfloat16, device=dyqT.device)
    return _nvfp4_gemm("mxfp8_nvfp4_grouped_gemm_wgrad", dyqT, dysT, dy_amax, xqT, xsT, x_amax, offs, M, N, K, out,
                       work, stream)
