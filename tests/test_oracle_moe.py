"""Pins for the oracle's MoE dispatch plan, combine and bf16 rounding (CPU).

The plan groups the (token, slot) pairs by expert in ascending (token, slot)
order; it is pinned against a hand-worked example (tests/golden), against
numpy's stable argsort of the flattened expert ids (an independent library
routine that defines the same order), and against its invariants.  The bf16
rounding is pinned against exact rational arithmetic and torch's float32 ->
bf16 conversion; the combine against a closed form, an exact gather and a
float64 einsum."""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "moe_plan_small.txt")


def _golden():
    d = {}
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        d[key] = np.array([int(v) for v in vals], dtype=np.int64)
    return d


def test_plan_hand_example():
    g = _golden()
    E = int(g["E"][0])
    idx = g["idx"].reshape(-1, 2)
    offs, perm, inv = oracle.moe_plan(idx, E)
    np.testing.assert_array_equal(offs, g["offs"])
    np.testing.assert_array_equal(perm, g["perm"])
    np.testing.assert_array_equal(inv.reshape(-1), g["inv"])


def _random_routing(rng, T, k, E, skew=0.0):
    # distinct experts per token (top-k), optionally skewed towards low ids
    logits = rng.standard_normal((T, E)) - skew * np.log1p(np.arange(E))[None, :]
    return np.argsort(-logits, axis=1, kind="stable")[:, :k].astype(np.int32)


@pytest.mark.parametrize("T,k,E,skew", [(1, 1, 1, 0.0), (7, 2, 5, 0.0), (64, 6, 64, 0.0), (300, 8, 32, 1.5),
                                        (1000, 1, 16, 0.0), (257, 4, 9, 3.0)])
def test_plan_matches_stable_argsort(T, k, E, skew):
    rng = np.random.default_rng(T * 31 + k)
    idx = _random_routing(rng, T, k, E, skew)
    offs, perm, inv = oracle.moe_plan(idx, E)
    order = np.argsort(idx.reshape(-1), kind="stable")   # pairs in (expert, token, slot) order
    np.testing.assert_array_equal(perm, order // k)
    pos = np.empty(T * k, dtype=np.int64)
    pos[order] = np.arange(T * k)
    np.testing.assert_array_equal(inv.reshape(-1), pos)
    np.testing.assert_array_equal(np.diff(offs), np.bincount(idx.reshape(-1), minlength=E))


def test_plan_invariants_and_empty_experts():
    rng = np.random.default_rng(5)
    T, k, E = 500, 3, 40
    idx = rng.integers(0, 20, size=(T, k)).astype(np.int32)     # experts 20..39 stay empty
    offs, perm, inv = oracle.moe_plan(idx, E)
    assert offs[0] == 0 and offs[-1] == T * k and np.all(np.diff(offs) >= 0)
    assert np.all(np.diff(offs)[20:] == 0)
    t_of = np.repeat(np.arange(T), k)
    np.testing.assert_array_equal(perm[inv.reshape(-1)], t_of)          # inv and perm agree
    assert sorted(inv.reshape(-1).tolist()) == list(range(T * k))       # inv is a permutation
    for e in range(E):
        rows = np.arange(offs[e], offs[e + 1])
        pairs = np.argsort(inv.reshape(-1))[rows]
        assert np.all(idx.reshape(-1)[pairs] == e)                      # group holds expert e only
        assert np.all(np.diff(pairs) > 0)                               # ascending (token, slot)


def test_plan_rejects_bad_expert_ids():
    with pytest.raises(ValueError):
        oracle.moe_plan(np.array([[0, 3]]), 3)
    with pytest.raises(ValueError):
        oracle.moe_plan(np.array([[-1, 0]]), 3)


def _bf16_exact(v: float) -> int:
    """Nearest-even bf16 bits by exact rational arithmetic."""
    if v != v:
        return 0x7FC0
    sign = 0x8000 if np.signbit(v) else 0
    a = Fraction(abs(v))
    if a == 0:
        return sign
    best = None
    # candidates: every finite bf16 magnitude near a, found by binary search on the bit pattern
    lo, hi = 0, 0x7F80
    while lo < hi:                      # first pattern whose value >= a
        mid = (lo + hi) // 2
        if _val(mid) >= a:
            hi = mid
        else:
            lo = mid + 1
    cands = [c for c in (lo - 1, lo) if 0 <= c <= 0x7F7F]
    if lo == 0x7F80:                    # above the largest finite value
        big, top = _val(0x7F7F), Fraction(2) ** 128
        return sign | (0x7F80 if a >= (big + top) / 2 else 0x7F7F)
    for c in cands:
        d = abs(_val(c) - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return sign | best[1]


def _val(bits: int) -> Fraction:
    e, m = (bits >> 7) & 0xFF, bits & 0x7F
    if e == 0:
        return Fraction(m, 1) * Fraction(2) ** -133
    return Fraction(128 + m, 128) * Fraction(2) ** (e - 127)


def test_bf16_rounding_exact_rationals():
    rng = np.random.default_rng(9)
    vals = np.concatenate([
        rng.standard_normal(2000) * 2.0 ** rng.integers(-140, 128, 2000),
        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135,
         2.0 ** -126 - 2.0 ** -134, 3.3895313892515355e38, 3.39e38, 3.3961e38, 1e39, -1e39],
    ])
    got = oracle.bf16_from_double(vals)
    for v, g in zip(vals, got):
        assert int(g) == _bf16_exact(float(v)), v


def test_bf16_rounding_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(10)
    f = (rng.standard_normal(100000) * 2.0 ** rng.integers(-130, 120, 100000)).astype(np.float32)
    bits = np.arange(1 << 16, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]
    mids = ((bits << 16) | 0x8000).view(np.float32)       # exact midpoints between neighbours
    f = np.concatenate([f, mids, (bits << 16).view(np.float32)])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.bf16_from_double(f.astype(np.float64)), ref)


def _bf16_tensor(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def test_combine_closed_forms():
    rng = np.random.default_rng(11)
    T, k, E, C = 50, 3, 7, 64
    idx = _random_routing(rng, T, k, E)
    offs, perm, inv = oracle.moe_plan(idx, E)
    rows = T * k
    # constant rows c_r = r: y[t] = sum_j w[t, j] * inv[t, j]
    yp = _bf16_tensor(np.repeat(np.arange(rows, dtype=np.float32)[:, None], C, axis=1))
    w = rng.random((T, k)).astype(np.float32)
    y = oracle.moe_combine(yp, inv, w)
    ref = oracle.bf16_from_double((w.astype(np.float64) * inv).sum(axis=1))
    np.testing.assert_array_equal(y, np.repeat(ref[:, None], C, axis=1))
    # k = 1, w = 1: an exact gather of the expert rows
    idx1 = idx[:, :1]
    offs1, perm1, inv1 = oracle.moe_plan(idx1, E)
    yp1 = _bf16_tensor(rng.standard_normal((T, C)))
    y1 = oracle.moe_combine(yp1, inv1, np.ones((T, 1), dtype=np.float32))
    np.testing.assert_array_equal(y1, yp1.view(torch.int16).numpy().view(np.uint16)[inv1[:, 0]])
    # zero weights
    assert np.all(oracle.moe_combine(yp, inv, np.zeros((T, k), dtype=np.float32)) == 0)


def test_combine_matches_float64_einsum():
    rng = np.random.default_rng(12)
    T, k, E, C = 80, 6, 16, 96
    idx = _random_routing(rng, T, k, E)
    offs, perm, inv = oracle.moe_plan(idx, E)
    yp = _bf16_tensor(rng.standard_normal((T * k, C)))
    w = rng.random((T, k)).astype(np.float32)
    y = oracle.moe_combine(yp, inv, w)
    ypd = yp.float().numpy().astype(np.float64)
    ref = np.einsum("tk,tkc->tc", w.astype(np.float64), ypd[inv])
    np.testing.assert_array_equal(y, oracle.bf16_from_double(ref))
