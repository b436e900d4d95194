"""Pins for the oracle's MXFP8 tensor quantisers and their data layouts (CPU).

Rowwise/colwise block placement is checked against an independent numpy
block quantiser that uses the ml_dtypes E4M3 codec; the scale swizzle is
checked against vLLM's ``to_blocked`` (the 128x4 block-scaling layout that
tcgen05 block-scaled MMA reads, implemented independently of this repo).
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).numpy().view(np.uint16)


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def np_block_quant(blocks: np.ndarray):
    """Independent reference: blocks [..., n] fp64 -> (deq [..., n], scale byte [...]).
    s = floor(log2 amax) - 8 via np.log2, clamped; codes via ml_dtypes."""
    amax = np.abs(blocks).max(axis=-1)
    with np.errstate(divide="ignore"):
        s = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 8, -127)
    s = np.clip(s, -127, 127).astype(np.int64)
    v = np.clip(np.ldexp(blocks, -s[..., None]), -448, 448)
    deq = np.ldexp(v.astype(ml_dtypes.float8_e4m3fn).astype(np.float64), s[..., None])
    return deq, (s + 127).astype(np.uint8)


def np_rowwise_ref(x: np.ndarray):
    R, C = x.shape
    deq, sb = np_block_quant(x.reshape(R, C // 32, 32))
    return deq.reshape(R, C), sb


def np_colwise_ref(x: np.ndarray, offs):
    """Group-relative column blocks; a short last block covers real rows only."""
    R, C = x.shape
    deq = np.zeros_like(x)
    scales = []
    for g in range(len(offs) - 1):
        lo, hi = offs[g], offs[g + 1]
        for t0 in range(lo, hi, 32):
            t1 = min(t0 + 32, hi)
            d, sb = np_block_quant(x[t0:t1].T)
            deq[t0:t1] = d.T
            scales.append(sb)
    return deq, scales


def _to_blocked(S: np.ndarray) -> np.ndarray:
    from vllm.model_executor.layers.quantization.qutlass_utils import to_blocked
    return to_blocked(torch.from_numpy(S), backend="torch").numpy().reshape(-1)


def test_swizzle_is_a_bijection_on_atoms():
    pitch = 3
    offs = sorted(oracle.sf_offset(r, c, pitch) for r in range(256) for c in range(12))
    assert offs == list(range(256 * 12))


@pytest.mark.parametrize("R,C", [(128, 128), (256, 384), (384, 2048)])
def test_rowwise_scale_layout_matches_to_blocked(R, C):
    x = wl.normal_bf16((R, C), 1.0, 11)
    # make each block's scale distinct-ish: multiply blocks by powers of two
    pw = torch.from_numpy(2.0 ** np.random.default_rng(1).integers(-20, 20, size=(R, C // 32))).float()
    x = (x.float() * pw.repeat_interleave(32, dim=1)).to(torch.bfloat16)
    q, sf = oracle.quantize_rowwise(x)
    _, sb = np_rowwise_ref(_f64(x))
    ncol = (C // 32 + 3) // 4 * 4
    S = np.zeros((R, ncol), dtype=np.uint8)
    S[:, : C // 32] = sb
    ref = _to_blocked(S)
    np.testing.assert_array_equal(sf[: ref.size], ref)


def test_rowwise_grouped_scale_layout_pads_each_group_to_128_rows():
    counts = [0, 7, 130, 1, 0, 200]
    offs = wl.offsets_from_counts(counts)
    R, C = int(offs[-1]), 256
    x = wl.normal_bf16((R, C), 3.0, 12)
    q, sf = oracle.quantize_rowwise(x, offs)
    _, sb = np_rowwise_ref(_f64(x))
    blocks = []
    for g in range(len(counts)):
        m = counts[g]
        nb = (m + 127) // 128
        S = np.zeros((nb * 128, 8), dtype=np.uint8)
        S[:m] = sb[offs[g]:offs[g + 1]]
        blocks.append(S)
    ref = _to_blocked(np.concatenate(blocks, axis=0))
    np.testing.assert_array_equal(sf[: ref.size], ref)
    assert sf.size >= ref.size


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rowwise_roundtrip_matches_numpy_reference(seed):
    counts = wl.tiny_random(seed, E=5, M=300)
    offs = wl.offsets_from_counts(counts)
    x = wl.with_outliers(wl.normal_bf16((300, 192), 1.0, seed), 0.01, 1000.0, seed)
    q, sf = oracle.quantize_rowwise(x, offs)
    deq = oracle.dequantize_rowwise(q, sf, offs)
    ref, _ = np_rowwise_ref(_f64(x))
    np.testing.assert_array_equal(deq, ref)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_colwise_roundtrip_matches_numpy_reference(seed):
    counts = np.array([0, 1, 31, 32, 33, 127, 128, 129, 0, 70], dtype=np.int64)
    counts = np.random.default_rng(seed).permutation(counts)
    offs = wl.offsets_from_counts(counts)
    R, C = int(offs[-1]), 160
    x = wl.with_outliers(wl.normal_bf16((R, C), 1.0, seed + 5), 0.01, 1000.0, seed)
    qT, sf = oracle.quantize_colwise(x, offs)
    deq = oracle.dequantize_colwise(qT, sf, R, offs)
    ref, _ = np_colwise_ref(_f64(x), offs)
    np.testing.assert_array_equal(deq, ref)


def test_colwise_layout_positions_and_pads():
    counts = [5, 0, 40]
    offs = wl.offsets_from_counts(counts)
    R, C = 45, 256
    x = wl.normal_bf16((R, C), 1.0, 3)
    qT, sf = oracle.quantize_colwise(x, offs)
    ldT = oracle.colwise_ld(R, 3)
    assert qT.shape == (C, ldT) and ldT % 128 == 0
    # group 0 at columns 0..4 (pad 5..31 zero), group 2 at 32..71 (pad 72..95 zero)
    assert np.all(qT[:, 5:32] == 0) and np.all(qT[:, 72:96] == 0)
    codes_g0, _ = oracle.quantize_block(_u16(x[0:5, 7].contiguous()))
    np.testing.assert_array_equal(qT[7, 0:5], codes_g0)
    codes_g2b1, sb = oracle.quantize_block(_u16(x[37:45, 9].contiguous()))
    np.testing.assert_array_equal(qT[9, 64:72], codes_g2b1)
    # scale of (col 9, group 2 block 1): block column 4*RB_2 + 1 = 4*1 + 1 = 5
    assert sf[oracle.sf_offset(9, 5, oracle.colwise_pitch(R, 3))] == sb


def test_colwise_scale_layout_matches_to_blocked():
    counts = [100, 0, 300]
    offs = wl.offsets_from_counts(counts)
    R, C = 400, 256
    x = wl.normal_bf16((R, C), 2.0, 9)
    qT, sf = oracle.quantize_colwise(x, offs)
    _, scales = np_colwise_ref(_f64(x), offs)
    # logical S^T [C, pitch*4]: group blocks at block column 4*RB_g + j
    pitch = oracle.colwise_pitch(R, 3)
    ST = np.zeros((C, pitch * 4), dtype=np.uint8)
    col = 0
    i = 0
    for g, m in enumerate(counts):
        for j in range((m + 31) // 32):
            ST[:, col + j] = scales[i]
            i += 1
        col += 4 * ((m + 127) // 128)
    ref = _to_blocked(ST)
    RB_G = sum((m + 127) // 128 for m in counts)
    for rb in range(C // 128):                     # only atoms with block column < RB_G are defined
        a = rb * pitch
        np.testing.assert_array_equal(sf[a * 512:(a + RB_G) * 512], ref[a * 512:(a + RB_G) * 512])


def test_offsets_must_be_a_valid_prefix():
    x = wl.normal_bf16((10, 32), 1.0, 0)
    for bad in ([0, 5, 4, 10], [1, 5, 10], [0, 5, 11]):
        with pytest.raises(ValueError):
            oracle.quantize_rowwise(x, bad)
        with pytest.raises(ValueError):
            oracle.quantize_colwise(x, bad)
