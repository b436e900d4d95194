"""Pins for the oracle's SwiGLU between the gate/up and down linears (CPU).

h = silu(g) * u with silu(g) = g / (1 + exp(-g)), gate g = columns 0..I-1 and
up u = columns I..2I-1 of the gate/up output, evaluated in fp64 and rounded
once to bf16.  The pages give no formula (the expert pipeline as a whole is on
opensourcebeat.com, section "Двухсторонняя атака: MXFP8 и DeepEP"); checked
against torch's float64 silu (an independent implementation) on every finite
bf16 gate value, closed forms and the odd-part identity, and the rounding
against torch's float32 -> bf16 conversion where fp32 holds the product
exactly.
"""
import numpy as np
import torch

import oracle


def _finite_bf16_values() -> np.ndarray:
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)].astype(np.float64)


def test_silu_equals_torch_on_every_bf16_gate():
    g = _finite_bf16_values()
    ref = torch.nn.functional.silu(torch.from_numpy(g)).numpy()
    got = np.array([oracle.silu(x) for x in g])
    big = np.abs(ref) > 1e-300
    np.testing.assert_allclose(got[big], ref[big], rtol=4e-16, atol=0)
    assert np.all(np.abs(got[~big]) <= 1e-300)


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    for x in (40.0, 100.0, 1e4):          # sigma(x) rounds to 1 in fp64
        assert oracle.silu(x) == x
    for x in (800.0, 1e4):                 # exp(x) overflows: silu(-x) is -0
        assert oracle.silu(-x) == 0.0
    assert abs(oracle.silu(1.0) - 1.0 / (1.0 + np.exp(-1.0))) <= 1e-16
    # silu(x) - silu(-x) = x (sigma(x) + sigma(-x) = 1)
    for x in np.linspace(-30, 30, 121):
        assert abs(oracle.silu(x) - oracle.silu(-x) - x) <= 4e-15 * max(1.0, abs(x))


def test_swiglu_takes_gate_then_up_columns_and_rounds_once():
    rng = np.random.default_rng(0)
    M, I = 7, 96
    Y = rng.standard_normal((M, 2 * I)) * 3
    h = oracle.swiglu(Y)
    g, u = Y[:, :I], Y[:, I:]
    exact = g / (1.0 + np.exp(-g)) * u
    np.testing.assert_array_equal(h, oracle.bf16_from_double(exact))
    # swapping the halves gives a different result (gate and up are not symmetric)
    assert not np.array_equal(oracle.swiglu(np.concatenate([u, g], axis=1)), h)


def test_swiglu_rounding_matches_torch_where_fp32_is_exact():
    # g = 50: sigma(g) rounds to 1 in fp64, so h = 50 u; with bf16 u the
    # product has at most 13 significant bits (exact in fp32) and only the
    # final rounding to bf16 remains, which torch's fp32 -> bf16 cast defines
    M, I = 3, 64
    u = torch.randn((M, I), generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).double().numpy()
    Y = np.concatenate([np.full((M, I), 50.0), u], axis=1)
    ref = torch.from_numpy((50.0 * u).astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(oracle.swiglu(Y), ref.view(np.uint16))
    assert not np.array_equal(oracle.swiglu(Y), torch.from_numpy(u).to(torch.bfloat16).view(torch.int16).numpy()
                              .view(np.uint16))
    Y0 = np.concatenate([np.zeros((M, I)), u], axis=1)
    assert np.all(oracle.swiglu(Y0) & 0x7FFF == 0)
