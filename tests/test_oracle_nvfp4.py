"""Pins for the oracle's NVFP4 rules (CPU only).

E2M1 encoding and decoding are pinned against ml_dtypes' float4_e2m1fn, the
E4M3 block scale against ml_dtypes' float8_e4m3fn, whole blocks against
hand-worked examples (tests/golden/nvfp4_blocks.txt) and an independent
numpy implementation of the block rule (fp32 arithmetic in the same order,
casts by ml_dtypes), the layouts against a numpy packer, and the
dequantisation against its error bounds."""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_blocks.txt")
F4, F8 = ml_dtypes.float4_e2m1fn, ml_dtypes.float8_e4m3fn


def _u16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_e2m1_decode_all_nibbles():
    ref = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    np.testing.assert_array_equal(oracle.e2m1_decode(np.arange(16)), ref)


def test_e2m1_encode_matches_ml_dtypes():
    bits = np.arange(1 << 16, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]
    v = (bits << 16).view(np.float32)                      # every finite bf16 value
    rng = np.random.default_rng(0)
    v = np.concatenate([v, (rng.standard_normal(100000) * 3).astype(np.float32),
                        np.arange(-700, 701, dtype=np.float32) / 100])
    np.testing.assert_array_equal(oracle.e2m1_encode(v.astype(np.float64)), v.astype(F4).view(np.uint8))


def test_tensor_scale():
    assert oracle.nvfp4_tensor_scale(2688.0) == np.float32(1.0)
    assert oracle.nvfp4_tensor_scale(0.0) == np.float32(1.0)
    for a in (1.0, 3.0, 1e-3, 1e6):
        assert oracle.nvfp4_tensor_scale(a) == np.float32(2688.0) / np.float32(a)


def test_hand_worked_blocks():
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, S, sb, pairs = [s.strip() for s in line.split("|")]
        vals, nibs = np.zeros(16), np.zeros(16, dtype=np.uint8)
        for i, pr in enumerate(pairs.split()):
            v, n = pr.split(":")
            vals[i], nibs[i] = float(v), int(n, 16)
        codes, got_sb = oracle.nvfp4_quantize_block(_u16(vals), float(S))
        assert got_sb == int(sb, 16), name
        np.testing.assert_array_equal(codes, nibs, err_msg=name)


def _numpy_block(xf32, S):
    """Independent restatement of the block rule with numpy fp32 and ml_dtypes casts."""
    S = np.float32(S)
    amax = np.float32(np.abs(xf32).max()) if xf32.size else np.float32(0)
    u = np.float32(np.float32(amax * S) / np.float32(6))
    sb = np.array([u], dtype=np.float32).astype(F8).view(np.uint8)[0]
    r = np.float32(np.array([sb], dtype=np.uint8).view(F8).astype(np.float32)[0])
    if r == 0:
        return np.zeros(xf32.size, dtype=np.uint8), sb
    w = (xf32 * S).astype(np.float32) / r
    return w.astype(np.float32).astype(F4).view(np.uint8), sb


def test_blocks_match_numpy_restatement():
    rng = np.random.default_rng(1)
    for trial in range(3000):
        n = 16 if trial % 5 else int(rng.integers(1, 16))
        e = rng.integers(-40, 20)
        x = (rng.standard_normal(n) * 2.0 ** e).astype(np.float32)
        if trial % 7 == 0:
            x[rng.integers(0, n)] = 0.0
        xb = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
        S = oracle.nvfp4_tensor_scale(np.float32(np.abs(xb).max() * 2.0 ** rng.integers(0, 6)))
        codes, sb = oracle.nvfp4_quantize_block(_u16(xb), S)
        rc, rsb = _numpy_block(xb, S)
        assert sb == rsb
        np.testing.assert_array_equal(codes, rc)


def _numpy_rowwise(x, S, offs):
    """Independent layout: pack nibbles, place scales with the 128x4 atom formula."""
    xf = x.float().numpy()
    R, C = xf.shape
    q = np.zeros((R, C // 2), dtype=np.uint8)
    pitch = (C + 63) // 64
    RB, _, _ = oracle.nvfp4_group_blocks(offs, R)
    m = np.diff(offs)
    nb = sum((mm + 127) // 128 for mm in m) + len(m)
    sf = np.zeros(max(nb * pitch * 512, 512), dtype=np.uint8)
    rb = 0
    for g in range(len(m)):
        for t in range(m[g]):
            r = offs[g] + t
            pr = 128 * rb + t
            for j in range(C // 16):
                c, sb = _numpy_block(xf[r, 16 * j:16 * j + 16], S)
                q[r, 8 * j:8 * j + 8] = c[0::2] | (c[1::2] << 4)
                atom = (pr // 128) * pitch + j // 4
                sf[atom * 512 + (pr % 32) * 16 + ((pr % 128) // 32) * 4 + j % 4] = sb
        rb += (m[g] + 127) // 128
    return q, sf


def test_rowwise_layout_matches_numpy_packer():
    offs = wl.offsets_from_counts([0, 7, 130, 3])
    x = wl.normal_bf16((int(offs[-1]), 128), 1.0, 3)
    S = oracle.nvfp4_tensor_scale(oracle.nvfp4_amax(x))
    q, sf = oracle.nvfp4_quantize_rowwise(x, S, offs)
    rq, rsf = _numpy_rowwise(x, S, np.asarray(offs))
    np.testing.assert_array_equal(q, rq)
    RB, _, _ = oracle.nvfp4_group_blocks(offs, int(offs[-1]))
    n = RB * 2 * 512
    np.testing.assert_array_equal(sf[:n], rsf[:n])


def test_colwise_is_rowwise_of_each_groups_transpose():
    """Colwise blocks of 16 rows restarting at each group: quantising each
    group's rows transposed (rowwise, padded with zero rows to 32) gives the
    same nibbles and the same block scales."""
    counts = [5, 0, 40, 17, 64]
    offs = wl.offsets_from_counts(counts)
    R, C = int(offs[-1]), 128
    x = wl.normal_bf16((R, C), 1.0, 4)
    S = oracle.nvfp4_tensor_scale(oracle.nvfp4_amax(x))
    qT, sfT = oracle.nvfp4_quantize_colwise(x, S, offs)
    pitch = oracle.nvfp4_colwise_pitch(R, len(counts))
    p0, rb64 = 0, 0
    xf = x.float().numpy()
    for g, m in enumerate(counts):
        lo = int(offs[g])
        for c in range(C):
            for b in range((m + 15) // 16):
                seg = xf[lo + 16 * b: lo + min(m, 16 * b + 16), c]
                codes, sb = _numpy_block(seg, S)
                for i, cd in enumerate(codes):
                    col = p0 + 16 * b + i
                    byte = qT[c, col // 2]
                    assert ((byte >> 4) if col & 1 else (byte & 15)) == cd
                blk = 4 * rb64 + b
                atom = (c // 128) * pitch + blk // 4
                assert sfT[atom * 512 + (c % 32) * 16 + ((c % 128) // 32) * 4 + blk % 4] == sb
            # pad nibbles up to the 32-padded end are zero
            for col in range(p0 + m, p0 + (m + 31) // 32 * 32):
                byte = qT[c, col // 2]
                assert ((byte >> 4) if col & 1 else (byte & 15)) == 0
        p0 += (m + 31) // 32 * 32
        rb64 += (m + 63) // 64


def test_dequantisation_error_bounds():
    rng = np.random.default_rng(6)
    offs = wl.offsets_from_counts([33, 100])
    x = wl.normal_bf16((133, 256), 1.0, 8)
    S = oracle.nvfp4_tensor_scale(oracle.nvfp4_amax(x))
    q, sf = oracle.nvfp4_quantize_rowwise(x, S, offs)
    d = oracle.nvfp4_dequantize_rowwise(q, sf, S, offs)
    xf = x.double().numpy()
    # per block: the E2M1 grid step is at most a quarter of the block's scaled amax band
    # (elements within [amax/2, amax] are off by <= 1/6 of amax after scale rounding)
    for r in range(0, 133, 7):
        for j in range(16):
            blk, dq = xf[r, 16 * j:16 * j + 16], d[r, 16 * j:16 * j + 16]
            amax = np.abs(blk).max()
            assert np.all(np.abs(dq - blk) <= amax * (1 / 6 + 1 / 16) + 1e-30)
    qT, sfT = oracle.nvfp4_quantize_colwise(x, S, offs)
    dT = oracle.nvfp4_dequantize_colwise(qT, sfT, 133, S, offs)
    assert np.abs(dT - xf).max() <= np.abs(xf).max() * 0.3


def test_ungrouped_equals_one_group():
    """No offsets means one group over all rows (quantise and dequantise, both layouts)."""
    x = wl.normal_bf16((100, 128), 1.0, 9)
    S = oracle.nvfp4_tensor_scale(oracle.nvfp4_amax(x))
    one = np.array([0, 100], dtype=np.int32)
    for fn in (oracle.nvfp4_quantize_rowwise, oracle.nvfp4_quantize_colwise):
        a, b = fn(x, S), fn(x, S, one)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])
    q, sf = oracle.nvfp4_quantize_rowwise(x, S)
    np.testing.assert_array_equal(oracle.nvfp4_dequantize_rowwise(q, sf, S), oracle.nvfp4_dequantize_rowwise(q, sf, S, one))
    qT, sfT = oracle.nvfp4_quantize_colwise(x, S)
    np.testing.assert_array_equal(oracle.nvfp4_dequantize_colwise(qT, sfT, 100, S),
                                  oracle.nvfp4_dequantize_colwise(qT, sfT, 100, S, one))
