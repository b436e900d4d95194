"""Shared test helpers: conversions and the GEMM tolerance contract."""
import numpy as np
import torch

# GEMM tolerance for fp32-accumulated MXFP8 products written as bf16,
# against the fp64 oracle on identical quantised inputs:
FROB_TOL = 5e-3        # ||G - R||_F / ||R||_F
ELEM_TOL = 2e-2        # |G - R| / |R| where |R| > ELEM_FLOOR * rms(R)
ELEM_FLOOR = 1e-2


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy bit patterns (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def assert_gemm_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    nref = np.linalg.norm(ref)
    if nref == 0.0:
        assert np.all(got == 0.0), f"{what}: reference is zero but output is not"
        return
    frob = np.linalg.norm(got - ref) / nref
    assert frob <= FROB_TOL, f"{what}: normalised Frobenius error {frob:.3e} > {FROB_TOL}"
    rms = np.sqrt(np.mean(ref * ref))
    big = np.abs(ref) > ELEM_FLOOR * rms
    if np.any(big):
        rel = np.abs(got[big] - ref[big]) / np.abs(ref[big])
        worst = rel.max()
        assert worst <= ELEM_TOL, f"{what}: per-element relative error {worst:.3e} > {ELEM_TOL}"


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest even) and back, via torch."""
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()
