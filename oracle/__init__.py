"""CPU oracle for MXFP8 quantisation and the MoE grouped GEMM (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does.  The arithmetic lives in ``mxfp8_oracle.c`` (plain C, fp64), which
shares no source with the CUDA library.  This wrapper only marshals numpy
arrays; bf16 tensors travel as their uint16 bit patterns.

What each function follows is stated in the C file's header: MXFP8 = blocks
of 32 elements sharing one power-of-two exponent (opensourcebeat.com,
"Enabling up to 41% faster pre-training: MXFP8 and DeepEP ...", FAQ), with
the OCP MX v1.0 E8M0/E4M3 rules; the grouped GEMM runs each expert on its
real token count (iitak.ru, "NVIDIA ... JAX", Transformer Engine paragraph).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_vp = ctypes.c_void_p


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_bf16_to_double.restype = ctypes.c_double
        L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_double]
        L.orc_scale_exponent.restype = ctypes.c_int
        L.orc_scale_exponent.argtypes = [ctypes.c_double]
        L.orc_e4m3_encode_array.argtypes = [_vp, _i64, _vp]
        L.orc_e4m3_decode_array.argtypes = [_vp, _i64, _vp]
        L.orc_scale_exponent_array.argtypes = [_vp, _i64, _vp]
        L.orc_quantize_block.argtypes = [_vp, ctypes.c_int, _i64, _vp, _i64, _vp]
        L.orc_sf_offset.restype = _i64
        L.orc_sf_offset.argtypes = [_i64, _i64, _i64]
        L.orc_rowwise_pitch.restype = _i64
        L.orc_rowwise_pitch.argtypes = [_i64]
        L.orc_colwise_pitch.restype = _i64
        L.orc_colwise_pitch.argtypes = [_i64, _i32]
        L.orc_colwise_ld.restype = _i64
        L.orc_colwise_ld.argtypes = [_i64, _i32]
        L.orc_check_offsets.argtypes = [_vp, _i32, _i64]
        for name in ("orc_quantize_rowwise", "orc_quantize_colwise"):
            getattr(L, name).argtypes = [_vp, _i64, _i64, _vp, _i32, _vp, _vp]
        for name in ("orc_dequantize_rowwise", "orc_dequantize_colwise"):
            getattr(L, name).argtypes = [_vp, _vp, _i64, _i64, _vp, _i32, _vp]
        for name in ("orc_gemm_fwd", "orc_gemm_dgrad", "orc_gemm_wgrad"):
            getattr(L, name).argtypes = [_vp, _vp, _vp, _i32, _i64, _i64, _i64, _vp]
        for name in ("orc_sample_fwd", "orc_sample_dgrad"):
            getattr(L, name).argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64,
                                         _i64, _vp, _vp, _vp]
        L.orc_sample_wgrad.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64,
                                       _i64, _vp, _vp, _vp, _vp]
        for name in ("orc_baseline_fwd_f32", "orc_baseline_dgrad_f32", "orc_baseline_wgrad_f32"):
            getattr(L, name).argtypes = [_vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _i64, _vp]
        L.orc_baseline_quantize_rows.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp]
        L.orc_threads.restype = ctypes.c_int
        L.orc_moe_plan.argtypes = [_vp, _i64, _i32, _i32, _vp, _vp, _vp]
        L.orc_moe_combine.argtypes = [_vp, _i64, _i64, _vp, _vp, _i64, _i32, _vp]
        L.orc_bf16_from_double.restype = ctypes.c_uint16
        L.orc_bf16_from_double.argtypes = [ctypes.c_double]
        L.orc_bf16_from_double_array.argtypes = [_vp, _i64, _vp]
        L.orc_ep_plan.restype = _i64
        L.orc_ep_plan.argtypes = [_vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]
        L.orc_ep_record_bytes.restype = _i64
        L.orc_ep_record_bytes.argtypes = [_i64]
        L.orc_ep_pack.argtypes = [_vp, _i64, _i64, _vp, _i64, _vp]
        L.orc_ep_unpack.argtypes = [_vp, _i64, _i64, _vp, _vp, _i32, _vp, _i64, _vp, _i32, _vp, _vp]
        L.orc_silu.restype = ctypes.c_double
        L.orc_silu.argtypes = [ctypes.c_double]
        L.orc_swiglu.argtypes = [_vp, _i64, _i64, _vp]
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_e2m1_encode.argtypes = [ctypes.c_double]
        L.orc_e2m1_encode_array.argtypes = [_vp, _i64, _vp]
        L.orc_nvfp4_tensor_scale.restype = ctypes.c_float
        L.orc_nvfp4_tensor_scale.argtypes = [ctypes.c_float]
        L.orc_nvfp4_quantize_block.argtypes = [_vp, ctypes.c_int, _i64, ctypes.c_float, _vp, _i64, _vp]
        L.orc_nvfp4_colwise_pitch.restype = _i64
        L.orc_nvfp4_colwise_pitch.argtypes = [_i64, _i32]
        L.orc_nvfp4_colwise_ld.restype = _i64
        L.orc_nvfp4_colwise_ld.argtypes = [_i64, _i32]
        for name in ("orc_nvfp4_quantize_rowwise", "orc_nvfp4_quantize_colwise"):
            getattr(L, name).argtypes = [_vp, _i64, _i64, _vp, _i32, ctypes.c_float, _vp, _vp]
        for name in ("orc_nvfp4_dequantize_rowwise", "orc_nvfp4_dequantize_colwise"):
            getattr(L, name).argtypes = [_vp, _vp, _i64, _i64, _vp, _i32, ctypes.c_float, _vp]
        _LIB = L
    return _LIB


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _u16(x) -> np.ndarray:
    """bf16 bit patterns as a contiguous uint16 numpy array (torch or numpy input)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16
    return x


def _offs(offs, rows):
    if offs is None:
        return None, 1
    o = np.ascontiguousarray(np.asarray(offs, dtype=np.int32))
    return o, len(o) - 1


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (offsets or sizes)")


# ---------------------------------------------------------------- scalars
def bf16_to_double(b: int) -> float:
    return lib().orc_bf16_to_double(b)


def e4m3_decode(b) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint8))
    out = np.empty(b.shape, dtype=np.float64)
    lib().orc_e4m3_decode_array(_p(b), b.size, _p(out))
    return out


def e4m3_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def scale_exponent(amax) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(amax, dtype=np.float64))
    out = np.empty(a.shape, dtype=np.int32)
    lib().orc_scale_exponent_array(_p(a), a.size, _p(out))
    return out


def quantize_block(x_u16) -> tuple[np.ndarray, int]:
    """One block (<= 32 values) -> (codes, scale byte)."""
    x = _u16(x_u16).reshape(-1)
    codes = np.empty(x.size, dtype=np.uint8)
    sb = np.zeros(1, dtype=np.uint8)
    lib().orc_quantize_block(_p(x), int(x.size), 1, _p(codes), 1, _p(sb))
    return codes, int(sb[0])


# ---------------------------------------------------------------- layouts
def sf_offset(row: int, col: int, pitch: int) -> int:
    return lib().orc_sf_offset(row, col, pitch)


def rowwise_pitch(C: int) -> int:
    return lib().orc_rowwise_pitch(C)


def colwise_pitch(R: int, G: int) -> int:
    return lib().orc_colwise_pitch(R, G)


def colwise_ld(R: int, G: int) -> int:
    return lib().orc_colwise_ld(R, G)


def _nb128(R: int, G: int) -> int:
    return 0 if R == 0 else (R + 127) // 128 + G - 1


def rowwise_scale_bytes(R: int, C: int, G: int) -> int:
    return _nb128(R, G) * rowwise_pitch(C) * 512


def colwise_scale_bytes(R: int, C: int, G: int) -> int:
    return ((C + 127) // 128) * colwise_pitch(R, G) * 512


def group_blocks(offs, R):
    """(RB_G, P_G): 128-row blocks and 32-padded rows over all groups."""
    if offs is None:
        return (R + 127) // 128, (R + 31) // 32 * 32
    m = np.diff(np.asarray(offs, dtype=np.int64))
    return int(((m + 127) // 128).sum()), int(((m + 31) // 32 * 32).sum())


# ---------------------------------------------------------------- quantisers
def quantize_rowwise(x, offs=None):
    """x: bf16 [R, C] -> (q uint8 [R, C], sf uint8 [bound]); only the first
    RB_G*pitch*512 scale bytes are defined."""
    xu = _u16(x)
    R, C = xu.shape
    o, G = _offs(offs, R)
    q = np.zeros((R, C), dtype=np.uint8)
    sf = np.zeros(max(rowwise_scale_bytes(R, C, G), 512), dtype=np.uint8)
    _check(lib().orc_quantize_rowwise(_p(xu), R, C, _p(o), G, _p(q), _p(sf)), "quantize_rowwise")
    return q, sf


def quantize_colwise(x, offs=None):
    """x: bf16 [R, C] -> (qT uint8 [C, ldT], sfT uint8 [bound]); columns of qT
    beyond P_G and atoms with block column >= RB_G are not defined."""
    xu = _u16(x)
    R, C = xu.shape
    o, G = _offs(offs, R)
    qT = np.zeros((C, colwise_ld(R, G)), dtype=np.uint8)
    sf = np.zeros(max(colwise_scale_bytes(R, C, G), 512), dtype=np.uint8)
    _check(lib().orc_quantize_colwise(_p(xu), R, C, _p(o), G, _p(qT), _p(sf)), "quantize_colwise")
    return qT, sf


def dequantize_rowwise(q, sf, offs=None) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    R, C = q.shape
    o, G = _offs(offs, R)
    out = np.zeros((R, C), dtype=np.float64)
    _check(lib().orc_dequantize_rowwise(_p(q), _p(sf), R, C, _p(o), G, _p(out)), "dequantize_rowwise")
    return out


def dequantize_colwise(qT, sf, R: int, offs=None) -> np.ndarray:
    qT = np.ascontiguousarray(qT, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    C = qT.shape[0]
    o, G = _offs(offs, R)
    assert qT.shape[1] == colwise_ld(R, G)
    out = np.zeros((R, C), dtype=np.float64)
    _check(lib().orc_dequantize_colwise(_p(qT), _p(sf), R, C, _p(o), G, _p(out)), "dequantize_colwise")
    return out


# ---------------------------------------------------------------- GEMMs (fp64)
def gemm_fwd(X, W, offs) -> np.ndarray:
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    o, E = _offs(offs, X.shape[0])
    M, K = X.shape
    N = W.shape[1]
    assert W.shape == (E, N, K)
    Y = np.zeros((M, N), dtype=np.float64)
    _check(lib().orc_gemm_fwd(_p(X), _p(W), _p(o), E, M, N, K, _p(Y)), "gemm_fwd")
    return Y


def gemm_dgrad(dY, W, offs) -> np.ndarray:
    dY = np.ascontiguousarray(dY, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    o, E = _offs(offs, dY.shape[0])
    M, N = dY.shape
    K = W.shape[2]
    assert W.shape == (E, N, K)
    dX = np.zeros((M, K), dtype=np.float64)
    _check(lib().orc_gemm_dgrad(_p(dY), _p(W), _p(o), E, M, N, K, _p(dX)), "gemm_dgrad")
    return dX


def gemm_wgrad(dY, X, offs) -> np.ndarray:
    dY = np.ascontiguousarray(dY, dtype=np.float64)
    X = np.ascontiguousarray(X, dtype=np.float64)
    o, E = _offs(offs, dY.shape[0])
    M, N = dY.shape
    K = X.shape[1]
    dW = np.zeros((E, N, K), dtype=np.float64)
    _check(lib().orc_gemm_wgrad(_p(dY), _p(X), _p(o), E, M, N, K, _p(dW)), "gemm_wgrad")
    return dW


# ---------------------------------------------------------------- full-size GEMMs, one expert at a time
# The grouped GEMM's definition (iitak.ru, "NVIDIA ... JAX", Transformer
# Engine paragraph: every expert on its own token rows) applied per expert to
# operands the C dequantisers above decode from the library layout; the
# per-expert product is a library matmul in fp64 (numpy), so full workload
# sizes finish in seconds.  Pinned against the triple-loop orc_gemm_* on
# small inputs in the CPU tests.

def _rows_prefix(counts, unit):
    return np.concatenate([[0], np.cumsum((np.asarray(counts, np.int64) + unit - 1) // unit)]).astype(np.int64)


def rowwise_rows(q, sf, C: int, row0: int, atom_row0: int, n: int) -> np.ndarray:
    """fp64 [n, C]: rows row0 .. row0+n-1 of a rowwise operand whose scale
    rows for them start at atom row atom_row0 (a group's first row, or any
    multiple of 128 inside a one-group operand)."""
    if n == 0:
        return np.zeros((0, C))
    pitch = rowwise_pitch(C)
    a0 = atom_row0 * pitch * 512
    a1 = (atom_row0 + (n + 127) // 128) * pitch * 512
    return dequantize_rowwise(np.ascontiguousarray(q[row0:row0 + n]), np.ascontiguousarray(sf[a0:a1]))


def colwise_rows(qT, sfT, pitch: int, col0: int, atom_col0: int, n: int) -> np.ndarray:
    """fp64 [n, C] (C = qT rows): logical rows stored from code column col0
    and scale-atom column atom_col0 of a colwise operand whose atom pitch is
    `pitch` (a group's rows, or a 128-aligned run inside a one-group
    operand)."""
    C = qT.shape[0]
    if n == 0:
        return np.zeros((0, C))
    sub = np.zeros((C, colwise_ld(n, 1)), dtype=np.uint8)
    sub[:, :n] = qT[:, col0:col0 + n]
    rb = (C + 127) // 128
    atoms = np.asarray(sfT[:rb * pitch * 512]).reshape(rb, pitch, 512)[:, atom_col0:atom_col0 + (n + 127) // 128]
    return dequantize_colwise(sub, np.ascontiguousarray(atoms).reshape(-1), n)


def fwd_by_expert(xq, xs, wq, ws, offs, N: int):
    """Yields (e, lo, hi, Y_e) with Y_e = deq(X_e) deq(W_e)^T in fp64; X
    rowwise grouped by offs, W rowwise [E*N, K] quantised as one group."""
    o = np.asarray(offs, np.int64)
    cnt = np.diff(o)
    RB = _rows_prefix(cnt, 128)
    K = xq.shape[1]
    for e in range(len(cnt)):
        lo, hi = int(o[e]), int(o[e + 1])
        if hi == lo:
            continue
        Xe = rowwise_rows(xq, xs, K, lo, int(RB[e]), hi - lo)
        We = rowwise_rows(wq, ws, K, e * N, e * N // 128, N)
        yield e, lo, hi, Xe @ We.T


def dgrad_by_expert(dyq, dys, wqT, wsT, offs, K: int):
    """Yields (e, lo, hi, dX_e) with dX_e = deq(dY_e) deq(W_e) in fp64; dY
    rowwise grouped by offs, W colwise (logical [E*N, K], one group)."""
    o = np.asarray(offs, np.int64)
    cnt = np.diff(o)
    RB = _rows_prefix(cnt, 128)
    N = dyq.shape[1]
    E = len(cnt)
    pitch_w = colwise_pitch(E * N, 1)
    for e in range(E):
        lo, hi = int(o[e]), int(o[e + 1])
        if hi == lo:
            continue
        dYe = rowwise_rows(dyq, dys, N, lo, int(RB[e]), hi - lo)
        We = colwise_rows(wqT[:K], wsT, pitch_w, e * N, e * N // 128, N)
        yield e, lo, hi, dYe @ We


def wgrad_by_expert(dyqT, dysT, xqT, xsT, offs, M: int):
    """Yields (e, dW_e) with dW_e = deq(dY_e)^T deq(X_e) in fp64 for every
    expert (zero for an expert without rows); dY and X colwise grouped by
    offs."""
    o = np.asarray(offs, np.int64)
    cnt = np.diff(o)
    E = len(cnt)
    RB = _rows_prefix(cnt, 128)
    P = np.concatenate([[0], np.cumsum((cnt + 31) // 32 * 32)])
    pitch = colwise_pitch(M, E)
    N, K = dyqT.shape[0], xqT.shape[0]
    for e in range(E):
        m = int(cnt[e])
        if m == 0:
            yield e, np.zeros((N, K))
            continue
        dYe = colwise_rows(dyqT, dysT, pitch, int(P[e]), int(RB[e]), m)
        Xe = colwise_rows(xqT, xsT, pitch, int(P[e]), int(RB[e]), m)
        yield e, dYe.T @ Xe


# ---------------------------------------------------------------- sampled outputs
def sample_fwd(xq, xs, wq, ws, offs, N, rows, cols) -> np.ndarray:
    xq = np.ascontiguousarray(xq, np.uint8); xs = np.ascontiguousarray(xs, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8); ws = np.ascontiguousarray(ws, np.uint8)
    o, E = _offs(offs, xq.shape[0])
    M, K = xq.shape
    r = np.ascontiguousarray(rows, np.int64); c = np.ascontiguousarray(cols, np.int64)
    out = np.zeros(r.size, dtype=np.float64)
    _check(lib().orc_sample_fwd(_p(xq), _p(xs), _p(wq), _p(ws), _p(o), E, M, N, K, r.size,
                                _p(r), _p(c), _p(out)), "sample_fwd")
    return out


def sample_dgrad(dyq, dys, wqT, wsT, offs, K, rows, cols) -> np.ndarray:
    dyq = np.ascontiguousarray(dyq, np.uint8); dys = np.ascontiguousarray(dys, np.uint8)
    wqT = np.ascontiguousarray(wqT, np.uint8); wsT = np.ascontiguousarray(wsT, np.uint8)
    o, E = _offs(offs, dyq.shape[0])
    M, N = dyq.shape
    r = np.ascontiguousarray(rows, np.int64); c = np.ascontiguousarray(cols, np.int64)
    out = np.zeros(r.size, dtype=np.float64)
    _check(lib().orc_sample_dgrad(_p(dyq), _p(dys), _p(wqT), _p(wsT), _p(o), E, M, N, K, r.size,
                                  _p(r), _p(c), _p(out)), "sample_dgrad")
    return out


def sample_wgrad(dyqT, dysT, xqT, xsT, offs, M, N, K, experts, rows, cols) -> np.ndarray:
    dyqT = np.ascontiguousarray(dyqT, np.uint8); dysT = np.ascontiguousarray(dysT, np.uint8)
    xqT = np.ascontiguousarray(xqT, np.uint8); xsT = np.ascontiguousarray(xsT, np.uint8)
    o, E = _offs(offs, M)
    e = np.ascontiguousarray(experts, np.int32)
    r = np.ascontiguousarray(rows, np.int64); c = np.ascontiguousarray(cols, np.int64)
    out = np.zeros(r.size, dtype=np.float64)
    _check(lib().orc_sample_wgrad(_p(dyqT), _p(dysT), _p(xqT), _p(xsT), _p(o), E, M, N, K, r.size,
                                  _p(e), _p(r), _p(c), _p(out)), "sample_wgrad")
    return out


# ---------------------------------------------------------------- CPU baseline (fp32 accumulate)
def threads() -> int:
    return lib().orc_threads()


def baseline_fwd_f32(X_u16, W_u16, offs, N, row_lo, row_hi, out=None):
    X = _u16(X_u16); W = _u16(W_u16)
    o, E = _offs(offs, X.shape[0])
    M, K = X.shape
    Y = out if out is not None else np.zeros((M, N), dtype=np.float32)
    _check(lib().orc_baseline_fwd_f32(_p(X), _p(W), _p(o), E, M, N, K, row_lo, row_hi, _p(Y)), "baseline_fwd")
    return Y


def baseline_dgrad_f32(dY_u16, W_u16, offs, K, row_lo, row_hi, out=None):
    dY = _u16(dY_u16); W = _u16(W_u16)
    o, E = _offs(offs, dY.shape[0])
    M, N = dY.shape
    dX = out if out is not None else np.zeros((M, K), dtype=np.float32)
    _check(lib().orc_baseline_dgrad_f32(_p(dY), _p(W), _p(o), E, M, N, K, row_lo, row_hi, _p(dX)), "baseline_dgrad")
    return dX


def baseline_wgrad_f32(dY_u16, X_u16, offs, n_lo, n_hi, out=None):
    dY = _u16(dY_u16); X = _u16(X_u16)
    o, E = _offs(offs, dY.shape[0])
    M, N = dY.shape
    K = X.shape[1]
    dW = out if out is not None else np.zeros((E, N, K), dtype=np.float32)
    _check(lib().orc_baseline_wgrad_f32(_p(dY), _p(X), _p(o), E, M, N, K, n_lo, n_hi, _p(dW)), "baseline_wgrad")
    return dW


def baseline_quantize_rows(x_u16, row_lo, row_hi):
    x = _u16(x_u16)
    R, C = x.shape
    q = np.zeros((R, C), dtype=np.uint8)
    s = np.zeros((R, C // 32), dtype=np.uint8)
    lib().orc_baseline_quantize_rows(_p(x), C, row_lo, row_hi, _p(q), _p(s))
    return q, s


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("annotations", "ctypes", "np", "os")]


# ---------------------------------------------------------------- MoE dispatch plan / combine
def moe_plan(idx, E: int):
    """idx: int [T, k] expert ids -> (offs int32 [E+1], perm int32 [T*k], inv int32 [T, k]).
    Pairs grouped by expert in ascending (token, slot) order."""
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    T, k = idx.shape
    offs = np.zeros(E + 1, dtype=np.int32)
    perm = np.zeros(T * k, dtype=np.int32)
    inv = np.zeros((T, k), dtype=np.int32)
    _check(lib().orc_moe_plan(_p(idx), T, k, E, _p(offs), _p(perm), _p(inv)), "moe_plan")
    return offs, perm, inv


def bf16_from_double(v) -> np.ndarray:
    """Nearest-even bf16 bits (uint16) of float64 values."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.zeros(a.shape, dtype=np.uint16)
    lib().orc_bf16_from_double_array(_p(a), a.size, _p(out))
    return out


def moe_combine(yp, inv, w) -> np.ndarray:
    """yp: bf16 [rows, C]; inv int [T, k]; w float32 [T, k] -> bf16 bits [T, C]:
    y[t] = sum_j w[t, j] * yp[inv[t, j]], in fp64, rounded once to bf16."""
    ypu = _u16(yp)
    rows, C = ypu.shape
    inv = np.ascontiguousarray(np.asarray(inv, dtype=np.int32))
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float32))
    T, k = inv.shape
    y = np.zeros((T, C), dtype=np.uint16)
    _check(lib().orc_moe_combine(_p(ypu), rows, C, _p(inv), _p(w), T, k, _p(y)), "moe_combine")
    return y


# ---------------------------------------------------------------- expert-parallel dispatch
class EpPlan:
    """The send side of one dispatch (see orc_ep_plan)."""

    def __init__(self, counts, rec_token, pair_expert, pair_rec, ret_pos, bad):
        self.counts, self.rec_token, self.pair_expert, self.pair_rec = counts, rec_token, pair_expert, pair_rec
        self.ret_pos, self.bad = ret_pos, bad

    @property
    def num_ranks(self) -> int:
        return self.counts.size // 2

    def records_to(self, p: int) -> slice:
        c = self.counts[: self.num_ranks]
        return slice(int(c[:p].sum()), int(c[: p + 1].sum()))

    def pairs_to(self, p: int) -> slice:
        c = self.counts[self.num_ranks:]
        return slice(int(c[:p].sum()), int(c[: p + 1].sum()))


def ep_plan(idx, E: int, P: int) -> EpPlan:
    """idx: int [T, k] global expert ids; P ranks owning E/P consecutive experts each."""
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    T, k = idx.shape
    cap = max(T * k, 1)
    counts = np.zeros(2 * P, dtype=np.int32)
    rec_token = np.zeros(cap, dtype=np.int32)
    pair_expert = np.zeros(cap, dtype=np.int32)
    pair_rec = np.zeros(cap, dtype=np.int32)
    ret_pos = np.zeros((T, k), dtype=np.int32)
    bad = lib().orc_ep_plan(_p(idx), T, k, E, P, _p(counts), _p(rec_token), _p(pair_expert), _p(pair_rec),
                            _p(ret_pos))
    if bad < 0:
        raise ValueError("ep_plan: P < 1 or E not a positive multiple of P")
    R, S = int(counts[:P].sum()), int(counts[P:].sum())
    return EpPlan(counts, rec_token[:R].copy(), pair_expert[:S].copy(), pair_rec[:S].copy(), ret_pos, int(bad))


def ep_record_bytes(C: int) -> int:
    return int(lib().orc_ep_record_bytes(C))


def ep_pack(x, rec_token) -> np.ndarray:
    """x: bf16 [T, C] -> records uint8 [R, ep_record_bytes(C)] (rowwise MXFP8 of row rec_token[i])."""
    xu = _u16(x)
    T, C = xu.shape
    rt = np.ascontiguousarray(np.asarray(rec_token, dtype=np.int32))
    out = np.zeros((rt.size, ep_record_bytes(C)), dtype=np.uint8)
    _check(lib().orc_ep_pack(_p(xu), T, C, _p(rt), rt.size, _p(out)), "ep_pack")
    return out


def ep_source_bases(recv_counts) -> np.ndarray:
    """recv_counts int [2P] (records from each source, then pairs from each
    source) -> src_base int32 [2(P+1)]: pair bases then record bases."""
    c = np.asarray(recv_counts, dtype=np.int64)
    P = c.size // 2
    rec, pairs = c[:P], c[P:]
    return np.concatenate([[0], np.cumsum(pairs), [0], np.cumsum(rec)]).astype(np.int32)


def ep_unpack(records, C: int, pair_rec, src_base, perm, offs):
    """Received records + pair entries -> rowwise MXFP8 (q [M, C], sf) of the
    grouped rows, as quantize_rowwise would write them."""
    rec = np.ascontiguousarray(records, dtype=np.uint8)
    R = rec.shape[0]
    pr = np.ascontiguousarray(np.asarray(pair_rec, dtype=np.int32))
    sb = np.ascontiguousarray(np.asarray(src_base, dtype=np.int32))
    pm = np.ascontiguousarray(np.asarray(perm, dtype=np.int32))
    M = pm.size
    o, G = _offs(offs, M)
    P = sb.size // 2 - 1
    q = np.zeros((M, C), dtype=np.uint8)
    sf = np.zeros(max(rowwise_scale_bytes(M, C, G), 512), dtype=np.uint8)
    _check(lib().orc_ep_unpack(_p(rec), R, C, _p(pr), _p(sb), P, _p(pm), M, _p(o), G, _p(q), _p(sf)), "ep_unpack")
    return q, sf


# ---------------------------------------------------------------- NVFP4
def e2m1_decode(nibbles) -> np.ndarray:
    n = np.asarray(nibbles, dtype=np.uint8).reshape(-1)
    return np.array([lib().orc_e2m1_decode(int(b)) for b in n], dtype=np.float64)


def e2m1_encode(v) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.zeros(a.shape, dtype=np.uint8)
    lib().orc_e2m1_encode_array(_p(a), a.size, _p(out))
    return out


def nvfp4_tensor_scale(amax: float) -> np.float32:
    return np.float32(lib().orc_nvfp4_tensor_scale(float(np.float32(amax))))


def nvfp4_amax(x) -> np.float32:
    """Largest |x| of a bf16 tensor, as fp32 (exact)."""
    xu = _u16(x)
    return np.float32(np.abs((xu.astype(np.uint32) << 16).view(np.float32)).max()) if xu.size else np.float32(0)


def nvfp4_quantize_block(x_u16, S) -> tuple[np.ndarray, int]:
    xu = np.ascontiguousarray(np.asarray(x_u16, dtype=np.uint16))
    codes = np.zeros(xu.size, dtype=np.uint8)
    sb = np.zeros(1, dtype=np.uint8)
    lib().orc_nvfp4_quantize_block(_p(xu), xu.size, 1, float(S), _p(codes), 1, _p(sb))
    return codes, int(sb[0])


def nvfp4_rowwise_pitch(C: int) -> int:
    return (C + 63) // 64


def nvfp4_colwise_pitch(R: int, G: int) -> int:
    return lib().orc_nvfp4_colwise_pitch(R, G)


def nvfp4_colwise_ld(R: int, G: int) -> int:
    """Row length of the colwise codes in ELEMENTS (bytes = half)."""
    return lib().orc_nvfp4_colwise_ld(R, G)


def nvfp4_rowwise_scale_bytes(R: int, C: int, G: int) -> int:
    return _nb128(R, G) * nvfp4_rowwise_pitch(C) * 512


def nvfp4_colwise_scale_bytes(R: int, C: int, G: int) -> int:
    return ((C + 127) // 128) * max(nvfp4_colwise_pitch(R, G), 0) * 512


def nvfp4_group_blocks(offs, R):
    """(RB_G, RB64_G, P_G): 128-row blocks, 64-row blocks and 32-padded rows over all groups."""
    m = np.diff(np.asarray(offs if offs is not None else [0, R], dtype=np.int64))
    return int(((m + 127) // 128).sum()), int(((m + 63) // 64).sum()), int(((m + 31) // 32 * 32).sum())


def nvfp4_quantize_rowwise(x, S, offs=None):
    """x: bf16 [R, C] -> (q uint8 [R, C/2] packed, sf uint8 atoms)."""
    xu = _u16(x)
    R, C = xu.shape
    o, G = _offs(offs, R)
    q = np.zeros((R, C // 2), dtype=np.uint8)
    sf = np.zeros(max(nvfp4_rowwise_scale_bytes(R, C, G), 512), dtype=np.uint8)
    _check(lib().orc_nvfp4_quantize_rowwise(_p(xu), R, C, _p(o), G, float(S), _p(q), _p(sf)), "nvfp4_quantize_rowwise")
    return q, sf


def nvfp4_quantize_colwise(x, S, offs=None):
    """x: bf16 [R, C] -> (qT uint8 [C, ld/2] packed, sfT uint8 atoms)."""
    xu = _u16(x)
    R, C = xu.shape
    o, G = _offs(offs, R)
    qT = np.zeros((C, nvfp4_colwise_ld(R, G) // 2), dtype=np.uint8)
    sf = np.zeros(max(nvfp4_colwise_scale_bytes(R, C, G), 512), dtype=np.uint8)
    _check(lib().orc_nvfp4_quantize_colwise(_p(xu), R, C, _p(o), G, float(S), _p(qT), _p(sf)), "nvfp4_quantize_colwise")
    return qT, sf


def nvfp4_dequantize_rowwise(q, sf, S, offs=None) -> np.ndarray:
    q = np.ascontiguousarray(q)
    R, C = q.shape[0], q.shape[1] * 2
    o, G = _offs(offs, R)
    out = np.zeros((R, C), dtype=np.float64)
    _check(lib().orc_nvfp4_dequantize_rowwise(_p(q), _p(np.ascontiguousarray(sf)), R, C, _p(o), G, float(S), _p(out)),
           "nvfp4_dequantize_rowwise")
    return out


def nvfp4_dequantize_colwise(qT, sf, R: int, S, offs=None) -> np.ndarray:
    qT = np.ascontiguousarray(qT)
    C = qT.shape[0]
    o, G = _offs(offs, R)
    out = np.zeros((R, C), dtype=np.float64)
    _check(lib().orc_nvfp4_dequantize_colwise(_p(qT), _p(np.ascontiguousarray(sf)), R, C, _p(o), G, float(S),
                                              _p(out)), "nvfp4_dequantize_colwise")
    return out


# ---------------------------------------------------------------- SwiGLU between the two linears
def silu(g: float) -> float:
    """silu(g) = g / (1 + exp(-g)) in fp64."""
    return lib().orc_silu(float(g))


def swiglu(Y) -> np.ndarray:
    """Y: fp64 [M, 2I] gate/up output (gate = columns 0..I-1, up = I..2I-1)
    -> bf16 bits [M, I] of silu(gate) * up, fp64 then one nearest-even rounding."""
    Y = np.ascontiguousarray(np.asarray(Y, dtype=np.float64))
    M, N2 = Y.shape
    assert N2 % 2 == 0
    h = np.zeros((M, N2 // 2), dtype=np.uint16)
    _check(lib().orc_swiglu(_p(Y), M, N2 // 2, _p(h)), "swiglu")
    return h
