"""Pins for the oracle's grouped GEMMs (CPU).

Y_e = X_e W_e^T, dX_e = dY_e W_e, dW_e = dY_e^T X_e per expert on its real
token count (iitak.ru, "NVIDIA ... JAX", Transformer Engine grouped GEMM
paragraph; dropless: no capacity padding, no dropped tokens).  Checked by
brute force against numpy matmul, closed forms, invariants (counts sum to M,
empty experts give no rows and zero dW, expert permutation, the adjoint
identity) and the exact small-integer case.
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl


def _rand_case(seed, counts, N=24, K=40):
    rng = np.random.default_rng(seed)
    offs = wl.offsets_from_counts(counts)
    M, E = int(offs[-1]), len(counts)
    return offs, rng.standard_normal((M, K)), rng.standard_normal((E, N, K)), rng.standard_normal((M, N))


@pytest.mark.parametrize("seed", range(4))
def test_gemms_match_numpy_matmul_per_expert(seed):
    counts = wl.tiny_random(seed, E=5, M=37)
    offs, X, W, dY = _rand_case(seed, counts)
    Y, dX, dW = oracle.gemm_fwd(X, W, offs), oracle.gemm_dgrad(dY, W, offs), oracle.gemm_wgrad(dY, X, offs)
    for e in range(len(counts)):
        lo, hi = offs[e], offs[e + 1]
        np.testing.assert_allclose(Y[lo:hi], X[lo:hi] @ W[e].T, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dX[lo:hi], dY[lo:hi] @ W[e], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dW[e], dY[lo:hi].T @ X[lo:hi], rtol=1e-12, atol=1e-12)


def test_closed_forms():
    offs = wl.offsets_from_counts([3, 0, 5])
    M, E, N, K = 8, 3, 16, 64
    Y = oracle.gemm_fwd(np.full((M, K), 3.0), np.full((E, N, K), -2.0), offs)
    assert np.all(Y == K * 3.0 * -2.0)
    # identity weights return the input
    I = np.stack([np.eye(K)] * E)
    X = np.random.default_rng(0).standard_normal((M, K))
    np.testing.assert_array_equal(oracle.gemm_fwd(X, I, offs), X)
    # a one-hot row selects a weight column
    Xo = np.zeros((M, K)); Xo[4, 17] = 1.0
    W = np.random.default_rng(1).standard_normal((E, N, K))
    np.testing.assert_array_equal(oracle.gemm_fwd(Xo, W, offs)[4], W[2, :, 17])


def test_empty_experts_and_counts():
    counts = [0, 4, 0, 6, 0]
    offs, X, W, dY = _rand_case(3, counts)
    assert offs[-1] == sum(counts) == X.shape[0]
    dW = oracle.gemm_wgrad(dY, X, offs)
    for e in (0, 2, 4):
        assert np.all(dW[e] == 0.0)
    assert np.any(dW[1] != 0) and np.any(dW[3] != 0)


def test_expert_permutation_permutes_outputs():
    counts = [3, 5, 2]
    offs, X, W, dY = _rand_case(5, counts)
    perm = [2, 0, 1]
    rows = np.concatenate([np.arange(offs[e], offs[e + 1]) for e in perm])
    offs_p = wl.offsets_from_counts([counts[e] for e in perm])
    Y = oracle.gemm_fwd(X, W, offs)
    Yp = oracle.gemm_fwd(X[rows], W[perm], offs_p)
    np.testing.assert_array_equal(Yp, Y[rows])
    dWp = oracle.gemm_wgrad(dY[rows], X[rows], offs_p)
    np.testing.assert_array_equal(dWp, oracle.gemm_wgrad(dY, X, offs)[perm])


def test_small_integer_operands_are_exact_after_quantisation():
    """Integers in [-14, 14] quantise losslessly rowwise and colwise, so the
    GEMMs on the dequantised operands equal the exact integer matmul and the
    adjoint identity <dY, X W^T> = <dY W, X> holds exactly."""
    counts = [0, 7, 21, 36, 64]
    offs = wl.offsets_from_counts(counts)
    M, E, N, K = 128, 5, 64, 96
    X = wl.integer_bf16((M, K), -14, 14, 1)
    W = wl.integer_bf16((E, N, K), -14, 14, 2)
    dY = wl.integer_bf16((M, N), -14, 14, 3)
    Xi, Wi, dYi = (t.to(torch.int64).numpy() for t in (X, W, dY))
    xq, xs = oracle.quantize_rowwise(X, offs)
    np.testing.assert_array_equal(oracle.dequantize_rowwise(xq, xs, offs), Xi)
    xqT, xsT = oracle.quantize_colwise(X, offs)
    np.testing.assert_array_equal(oracle.dequantize_colwise(xqT, xsT, M, offs), Xi)
    wq, ws = oracle.quantize_rowwise(W.reshape(E * N, K))
    np.testing.assert_array_equal(oracle.dequantize_rowwise(wq, ws).reshape(E, N, K), Wi)
    Y = oracle.gemm_fwd(Xi.astype(float), Wi.astype(float), offs)
    dX = oracle.gemm_dgrad(dYi.astype(float), Wi.astype(float), offs)
    dW = oracle.gemm_wgrad(dYi.astype(float), Xi.astype(float), offs)
    for e in range(E):
        lo, hi = offs[e], offs[e + 1]
        assert np.array_equal(Y[lo:hi], Xi[lo:hi] @ Wi[e].T)
        assert np.array_equal(dX[lo:hi], dYi[lo:hi] @ Wi[e])
        assert np.array_equal(dW[e], dYi[lo:hi].T @ Xi[lo:hi])
    assert (dYi * Y).sum() == (dX * Xi).sum()
    assert (dW * Wi).sum() == (dYi * Y).sum()


def test_sampled_outputs_match_full_gemms():
    counts = [0, 9, 140, 33]
    offs = wl.offsets_from_counts(counts)
    M, E, N, K = 182, 4, 128, 96
    X = wl.normal_bf16((M, K), 1.0, 4)
    W = wl.normal_bf16((E, N, K), 0.5, 5)
    dY = wl.normal_bf16((M, N), 1.0, 6)
    xq, xs = oracle.quantize_rowwise(X, offs)
    wq, ws = oracle.quantize_rowwise(W.reshape(E * N, K))
    dyq, dys = oracle.quantize_rowwise(dY, offs)
    wqT, wsT = oracle.quantize_colwise(W.reshape(E * N, K))
    dyqT, dysT = oracle.quantize_colwise(dY, offs)
    xqT, xsT = oracle.quantize_colwise(X, offs)
    Xd = oracle.dequantize_rowwise(xq, xs, offs)
    Wd = oracle.dequantize_rowwise(wq, ws).reshape(E, N, K)
    dYd = oracle.dequantize_rowwise(dyq, dys, offs)
    WdT = oracle.dequantize_colwise(wqT, wsT, E * N).reshape(E, N, K)
    dYdc = oracle.dequantize_colwise(dyqT, dysT, M, offs)
    Xdc = oracle.dequantize_colwise(xqT, xsT, M, offs)
    rng = np.random.default_rng(0)
    r = rng.integers(0, M, 50); c = rng.integers(0, N, 50)
    np.testing.assert_allclose(oracle.sample_fwd(xq, xs, wq, ws, offs, N, r, c),
                               oracle.gemm_fwd(Xd, Wd, offs)[r, c], rtol=1e-13, atol=1e-13)
    ck = rng.integers(0, K, 50)
    np.testing.assert_allclose(oracle.sample_dgrad(dyq, dys, wqT, wsT, offs, K, r, ck),
                               oracle.gemm_dgrad(dYd, WdT, offs)[r, ck], rtol=1e-13, atol=1e-13)
    ex = rng.integers(0, E, 50)
    np.testing.assert_allclose(oracle.sample_wgrad(dyqT, dysT, xqT, xsT, offs, M, N, K, ex, c, ck),
                               oracle.gemm_wgrad(dYdc, Xdc, offs)[ex, c, ck], rtol=1e-13, atol=1e-13)


def test_fp32_baseline_tracks_fp64_definition():
    counts = [10, 0, 30]
    offs = wl.offsets_from_counts(counts)
    M, E, N, K = 40, 3, 32, 64
    X = wl.normal_bf16((M, K), 1.0, 7)
    W = wl.normal_bf16((E, N, K), 1.0, 8)
    dY = wl.normal_bf16((M, N), 1.0, 9)
    Xf, Wf, dYf = (t.to(torch.float64).numpy() for t in (X, W, dY))
    Y = oracle.baseline_fwd_f32(X, W.reshape(E * N, K), offs, N, 0, M)
    np.testing.assert_allclose(Y, oracle.gemm_fwd(Xf, Wf, offs), rtol=1e-4, atol=1e-4)
    dX = oracle.baseline_dgrad_f32(dY, W.reshape(E * N, K), offs, K, 0, M)
    np.testing.assert_allclose(dX, oracle.gemm_dgrad(dYf, Wf, offs), rtol=1e-4, atol=1e-4)
    dW = oracle.baseline_wgrad_f32(dY, X, offs, 0, N)
    np.testing.assert_allclose(dW, oracle.gemm_wgrad(dYf, Xf, offs), rtol=1e-4, atol=1e-4)


# ------------------------------------------------------------------ per-expert full-size forms
def _quantised_case(seed, counts, N=256, K=320):
    """Oracle-quantised operands (all layouts) of a grouped linear, with
    ragged groups that cross 128-row atom boundaries and an empty expert."""
    offs = wl.offsets_from_counts(counts)
    M, E = int(offs[-1]), len(counts)
    X = wl.normal_bf16((M, K), 1.0, seed + 1)
    W = wl.normal_bf16((E, N, K), 0.5, seed + 2)
    dY = wl.normal_bf16((M, N), 1.0, seed + 3)
    W2 = W.reshape(E * N, K)
    q = {"x": oracle.quantize_rowwise(X, offs), "w": oracle.quantize_rowwise(W2),
         "dy": oracle.quantize_rowwise(dY, offs), "wT": oracle.quantize_colwise(W2),
         "dyT": oracle.quantize_colwise(dY, offs), "xT": oracle.quantize_colwise(X, offs)}
    return offs, M, E, N, K, q


@pytest.mark.parametrize("seed,counts", [(0, [0, 130, 7, 300, 0, 129]), (1, [256, 1, 0, 40])])
def test_row_and_column_slices_equal_the_full_dequantisation(seed, counts):
    """rowwise_rows / colwise_rows of one group (or of a 128-aligned run of a
    one-group operand) equal the matching rows of the whole-tensor
    dequantisation."""
    offs, M, E, N, K, q = _quantised_case(seed, counts)
    cnt = np.diff(offs.astype(np.int64))
    RB = np.concatenate([[0], np.cumsum((cnt + 127) // 128)])
    P = np.concatenate([[0], np.cumsum((cnt + 31) // 32 * 32)])
    Xd = oracle.dequantize_rowwise(*q["x"], offs)
    Xc = oracle.dequantize_colwise(*q["xT"], M, offs)
    Wd = oracle.dequantize_rowwise(*q["w"])
    WdT = oracle.dequantize_colwise(*q["wT"], E * N)
    for e in range(E):
        lo, hi = int(offs[e]), int(offs[e + 1])
        np.testing.assert_array_equal(oracle.rowwise_rows(*q["x"], K, lo, int(RB[e]), hi - lo), Xd[lo:hi])
        np.testing.assert_array_equal(
            oracle.colwise_rows(*q["xT"], oracle.colwise_pitch(M, E), int(P[e]), int(RB[e]), hi - lo), Xc[lo:hi])
        np.testing.assert_array_equal(oracle.rowwise_rows(*q["w"], K, e * N, e * N // 128, N), Wd[e * N:(e + 1) * N])
        np.testing.assert_array_equal(
            oracle.colwise_rows(*q["wT"], oracle.colwise_pitch(E * N, 1), e * N, e * N // 128, N),
            WdT[e * N:(e + 1) * N])


@pytest.mark.parametrize("seed,counts", [(2, [0, 130, 7, 300, 0, 129]), (3, [5, 0, 0, 251])])
def test_per_expert_gemms_equal_the_triple_loop(seed, counts):
    """The per-expert BLAS forms used at full workload sizes give the
    triple-loop grouped GEMM of the whole dequantised operands (to fp64
    summation-order rounding), every expert, empty ones included."""
    offs, M, E, N, K, q = _quantised_case(seed, counts)
    Xd = oracle.dequantize_rowwise(*q["x"], offs)
    Wd = oracle.dequantize_rowwise(*q["w"]).reshape(E, N, K)
    dYd = oracle.dequantize_rowwise(*q["dy"], offs)
    WdT = oracle.dequantize_colwise(*q["wT"], E * N).reshape(E, N, K)
    dYc = oracle.dequantize_colwise(*q["dyT"], M, offs)
    Xc = oracle.dequantize_colwise(*q["xT"], M, offs)
    Y, dX, dW = oracle.gemm_fwd(Xd, Wd, offs), oracle.gemm_dgrad(dYd, WdT, offs), oracle.gemm_wgrad(dYc, Xc, offs)
    seen = set()
    for e, lo, hi, ye in oracle.fwd_by_expert(*q["x"], *q["w"], offs, N):
        np.testing.assert_allclose(ye, Y[lo:hi], rtol=1e-12, atol=1e-9)
        seen.add(e)
    assert seen == {e for e in range(E) if offs[e + 1] > offs[e]}
    for e, lo, hi, dxe in oracle.dgrad_by_expert(*q["dy"], *q["wT"], offs, K):
        np.testing.assert_allclose(dxe, dX[lo:hi], rtol=1e-12, atol=1e-9)
    got = dict(oracle.wgrad_by_expert(*q["dyT"], *q["xT"], offs, M))
    assert sorted(got) == list(range(E))
    for e in range(E):
        np.testing.assert_allclose(got[e], dW[e], rtol=1e-12, atol=1e-9)
        if offs[e + 1] == offs[e]:
            assert np.all(got[e] == 0.0)
