"""Pins for the oracle's MXFP8 scalar rules (CPU only).

The rules (32-element blocks sharing one exponent -- opensourcebeat.com,
"Enabling up to 41% faster pre-training: MXFP8 and DeepEP ...", FAQ; OCP MX
v1.0 E8M0 scale and E4M3 elements) are pinned against:
hand-worked blocks (tests/golden/hand_blocks.txt), two independent library
codecs (ml_dtypes and torch float8), and properties of the definition.
"""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_blocks.txt")


def _val(tok: str) -> float:
    if tok.startswith("-2^"):
        return -(2.0 ** int(tok[3:]))
    if tok.startswith("2^"):
        return 2.0 ** int(tok[2:])
    return float(tok)


def _bf16_bits(vals) -> np.ndarray:
    t = torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _golden_blocks():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, sb, pairs = [p.strip() for p in line.split("|")]
        vc = [(_val(a), int(b, 16)) for a, b in (p.split(":") for p in pairs.split())]
        out.append((name, int(sb, 16), vc))
    return out


@pytest.mark.parametrize("name,scale_byte,pairs", _golden_blocks(), ids=lambda v: v if isinstance(v, str) else "")
def test_hand_worked_blocks(name, scale_byte, pairs):
    vals = [v for v, _ in pairs] + [0.0] * (32 - len(pairs))
    codes, sb = oracle.quantize_block(_bf16_bits(vals))
    assert sb == scale_byte, name
    for i, (_, code) in enumerate(pairs):
        assert codes[i] == code, (name, i, hex(codes[i]), hex(code))
    assert all(c in (0x00,) for c in codes[len(pairs):]), name


def _all_finite_bf16() -> np.ndarray:
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (b >> 7) & 0xFF
    return b[exp != 0xFF]


def _bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("s", [-127, -8, 0, 119])
def test_e4m3_encode_matches_ml_dtypes_and_torch(s):
    """Every finite bf16 pattern x at scale 2^s: oracle E4M3(x*2^-s) equals
    ml_dtypes' and torch's float8_e4m3fn cast of the value clipped to +-448."""
    x = _bf16_to_f64(_all_finite_bf16())
    v = np.ldexp(x, -s)
    got = oracle.e4m3_encode(v)
    clipped = np.clip(v, -448.0, 448.0)
    ref_ml = clipped.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ref_t = torch.from_numpy(clipped).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, ref_ml)
    np.testing.assert_array_equal(got, ref_t)


def test_e4m3_decode_matches_ml_dtypes():
    b = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(b)
    ref = b.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert set(b[nan].tolist()) == {0x7F, 0xFF}


def test_e4m3_encode_decode_roundtrip_all_codes():
    b = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(b)
    ok = ~np.isnan(v)
    np.testing.assert_array_equal(oracle.e4m3_encode(v[ok]), b[ok])


def test_scale_exponent_property_and_e8m0_bits():
    """For every positive finite bf16 amax: unless clamped, amax*2^-s lies in
    [256, 512) (the largest power of two not exceeding amax, over 2^emax with
    emax = 8); the scale byte equals ml_dtypes' float8_e8m0fnu bits of 2^s."""
    b = _all_finite_bf16()
    a = _bf16_to_f64(b)
    a = np.unique(np.abs(a))
    s = oracle.scale_exponent(a)
    pos = a > 0
    unclamped = pos & (s > -127)
    r = np.ldexp(a[unclamped], -s[unclamped])
    assert np.all((r >= 256.0) & (r < 512.0))
    clamped = pos & (s == -127)
    assert np.all(np.ldexp(a[clamped], 127) < 512.0)      # clamping never needs saturation
    assert np.all(s[~pos] == -127)
    assert s.max() == 119                                   # largest bf16 gives 2^127 / 2^8
    e8 = np.ldexp(1.0, s).astype(ml_dtypes.float8_e8m0fnu).view(np.uint8)
    np.testing.assert_array_equal(e8, (s + 127).astype(np.uint8))


def test_scale_byte_monotone_in_amax():
    a = np.sort(np.unique(np.abs(_bf16_to_f64(_all_finite_bf16()))))
    s = oracle.scale_exponent(a)
    assert np.all(np.diff(s) >= 0)


def test_nonfinite_amax_gives_nan_scale():
    assert oracle.scale_exponent([np.inf, np.nan]).tolist() == [128, 128]
    codes, sb = oracle.quantize_block(_bf16_bits([1.0, np.inf] + [0.0] * 30))
    assert sb == 0xFF and np.all(codes == 0x7F)


def test_dequantisation_error_bound():
    """Within a block: normal-range codes are within 2^-4 relative error (half
    a unit of 3 mantissa bits); subnormal-range codes within 2^(s-10)
    absolute; only values above 448*2^s saturate."""
    rng = np.random.default_rng(7)
    for trial in range(200):
        exp = rng.integers(-30, 30)
        vals = rng.standard_normal(32) * 2.0 ** exp
        if trial % 5 == 0:
            vals[rng.integers(32)] *= 1000.0
        bits = _bf16_bits(vals)
        x = _bf16_to_f64(bits)
        codes, sb = oracle.quantize_block(bits)
        s = sb - 127
        deq = oracle.e4m3_decode(codes) * 2.0 ** s
        v = np.ldexp(x, -s)
        normal = (np.abs(v) >= 2.0 ** -6) & (np.abs(v) <= 448.0)
        assert np.all(np.abs(deq[normal] - x[normal]) <= 2.0 ** -4 * np.abs(x[normal]))
        sub = np.abs(v) < 2.0 ** -6
        assert np.all(np.abs(deq[sub] - x[sub]) <= 2.0 ** (s - 10))
        sat = np.abs(v) > 448.0
        assert np.all(np.abs(deq[sat]) == 448.0 * 2.0 ** s)


def test_small_integers_roundtrip_exactly():
    """Blocks of integers with |x| <= 14: every value is exact in E4M3 after
    scaling, for every block amax 1..14 (the basis of the exact GEMM pins)."""
    for amax in range(1, 15):
        vals = list(range(-amax, amax + 1))
        vals = (vals * 2)[:32] if len(vals) < 32 else vals[:32]
        bits = _bf16_bits(vals)
        codes, sb = oracle.quantize_block(bits)
        deq = oracle.e4m3_decode(codes) * 2.0 ** (sb - 127)
        np.testing.assert_array_equal(deq, np.array(vals, dtype=np.float64))
