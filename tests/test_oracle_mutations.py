"""The pins catch plausible mistakes.

Each mutant below is the MXFP8 block rule or a grouped GEMM with one
plausible mistake planted (an off-by-one exponent, ties rounded away from
zero, no saturation, a lost sign of zero, a wrong clamp, a dropped term, a
shifted group boundary, a transposed operand).  They are small CPU
restatements, not the oracle; the test checks that the oracle passes the pins
and that every mutant fails at least one of them, i.e. the pins would have
caught that mistake in the oracle.
"""
import math

import numpy as np
import pytest

import oracle
from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
from tests.test_oracle_scalars import _bf16_bits, _golden_blocks


def _e4m3(v, tie_even=True, saturate=True, keep_sign=True):
    """E4M3 code of a real value (1 sign, 4 exponent bits, bias 7, 3 mantissa bits)."""
    sign = 0x80 if (math.copysign(1.0, v) < 0 and (keep_sign or v != 0.0)) else 0x00
    a = abs(v)
    if a == 0.0:
        return sign
    e = max(math.floor(math.log2(a)), -6)                  # subnormals share the 2^-6 binade
    q = a / 2.0 ** (e - 3)                                 # units of the last mantissa bit
    lo = math.floor(q)
    frac = q - lo
    if frac > 0.5 or (frac == 0.5 and (lo % 2 == 1 if tie_even else True)):
        lo += 1
    mag = lo * 2.0 ** (e - 3)
    if mag > 448.0:
        if not saturate:
            return sign | 0x7F                             # NaN
        mag = 448.0
    if mag == 0.0:
        return sign if keep_sign else 0x00
    e2 = max(math.floor(math.log2(mag)), -6)
    m = int(round(mag / 2.0 ** (e2 - 3)))
    if e2 == -6 and m < 8:
        return sign | m                                    # subnormal
    return sign | ((e2 + 7) << 3) | (m - 8)


def _block(vals, emax=8, clamp_lo=-127, **enc):
    amax = max(abs(v) for v in vals)
    s = clamp_lo if amax == 0.0 else max(math.floor(math.log2(amax)) - emax, clamp_lo)
    s = min(s, 127)
    return [_e4m3(v * 2.0 ** -s, **enc) for v in vals], s + 127


def _golden_ok(fn):
    for name, sb, pairs in _golden_blocks():
        vals = [v for v, _ in pairs] + [0.0] * (32 - len(pairs))
        codes, byte = fn(vals)
        if byte != sb or any(codes[i] != c for i, (_, c) in enumerate(pairs)):
            return False
    return True


def _oracle_block(vals):
    codes, sb = oracle.quantize_block(_bf16_bits(vals))
    return list(codes), sb


def test_the_oracle_and_the_restatement_pass_the_golden_blocks():
    assert _golden_ok(_oracle_block)
    assert _golden_ok(_block)


@pytest.mark.parametrize("mutant", [
    dict(emax=7),                  # scale exponent off by one
    dict(emax=9),
    dict(tie_even=False),          # ties rounded away from zero
    dict(saturate=False),          # overflow to NaN instead of 448
    dict(keep_sign=False),         # -0 and negative underflow lose the sign
    dict(clamp_lo=-126),           # wrong lower clamp of the scale exponent
], ids=lambda d: ",".join(f"{k}={v}" for k, v in d.items()))
def test_block_rule_mutants_fail_a_golden_block(mutant):
    assert not _golden_ok(lambda vals: _block(vals, **mutant))


def _fwd_ok(fwd):
    counts = [3, 0, 5, 4]
    offs = wl.offsets_from_counts(counts)
    rng = np.random.default_rng(9)
    M, E, N, K = int(offs[-1]), len(counts), 6, 10
    X, W = rng.standard_normal((M, K)), rng.standard_normal((E, N, K))
    try:
        Y = fwd(X, W, offs)
    except Exception:
        return False
    ref = np.concatenate([X[offs[e]:offs[e + 1]] @ W[e].T for e in range(E)])
    return Y.shape == ref.shape and np.allclose(Y, ref, rtol=1e-12, atol=1e-12)


def _per_expert(op):
    def fwd(X, W, offs):
        return np.concatenate([op(X, W, offs, e) for e in range(W.shape[0])])
    return fwd


@pytest.mark.parametrize("name,mutant", [
    ("dropped_last_k", _per_expert(lambda X, W, o, e: X[o[e]:o[e + 1], :-1] @ W[e][:, :-1].T)),
    ("shifted_boundary", _per_expert(lambda X, W, o, e: X[max(o[e] - 1, 0):max(o[e + 1] - 1, 0)] @ W[e].T)),
    ("wrong_expert", _per_expert(lambda X, W, o, e: X[o[e]:o[e + 1]] @ W[(e + 1) % W.shape[0]].T)),
    ("transposed_weight", _per_expert(lambda X, W, o, e: X[o[e]:o[e + 1]] @ W[e])),
])
def test_gemm_mutants_fail_the_matmul_pin(name, mutant):
    assert _fwd_ok(oracle.gemm_fwd)
    assert not _fwd_ok(mutant), name


def _swizzle(S, offset):
    """Bytes of the logical scale matrix S [R, C] placed by an atom formula
    offset(r, c, pitch) (R a multiple of 128, C a multiple of 4)."""
    R, C = S.shape
    pitch = C // 4
    out = np.zeros(R * C, dtype=np.uint8)
    for r in range(R):
        for c in range(C):
            out[offset(r, c, pitch)] = S[r, c]
    return out


def _atom(inner):
    return lambda r, c, pitch: 512 * ((r // 128) * pitch + c // 4) + inner(r, c)


@pytest.mark.parametrize("name,inner", [
    ("quarter_and_block_swapped", lambda r, c: (r % 32) * 16 + (c % 4) * 4 + (r % 128) // 32),
    ("rows_not_interleaved", lambda r, c: (r % 128) * 4 + c % 4),
    ("quarter_stride_8", lambda r, c: (r % 32) * 16 + ((r % 128) // 32) * 8 % 16 + c % 4),
])
def test_scale_layout_mutants_fail_the_independent_layout(name, inner):
    from tests.test_oracle_layout import _to_blocked
    S = np.random.default_rng(3).integers(0, 255, size=(256, 8)).astype(np.uint8)
    ref = _to_blocked(S)
    assert np.array_equal(_swizzle(S, oracle.sf_offset), ref)         # the oracle's own formula
    bad = _atom(inner)
    try:
        got = _swizzle(S, bad)
    except IndexError:
        return                                                       # not even a layout of the atoms
    assert not np.array_equal(got, ref), name


def _double_rounded_bf16(v):
    """Mutant: round to fp32 first, then to bf16 (two roundings)."""
    import torch
    return torch.tensor(v, dtype=torch.float64).to(torch.float32).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def test_combine_rounding_mutant_rounds_twice():
    """Just above a bf16 tie by less than fp32 can hold: one rounding goes up,
    rounding through fp32 first lands on the tie and goes to even."""
    v = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30, -(1.0 + 2.0 ** -8 + 2.0 ** -30), 3.0 + 2.0 ** -7 + 2.0 ** -29])
    got = oracle.bf16_from_double(v)
    assert got.tolist() == [0x3F81, 0xBF81, 0x4041]
    assert _double_rounded_bf16(v).tolist() != got.tolist()


def test_unstable_dispatch_order_mutant_fails_the_stable_order():
    rng = np.random.default_rng(4)
    idx = np.stack([rng.permutation(6)[:2] for _ in range(50)]).astype(np.int32)
    _, perm, _ = oracle.moe_plan(idx, 6)                          # perm: source token of each grouped row
    flat = idx.reshape(-1)
    assert perm.tolist() == (np.argsort(flat, kind="stable") // 2).tolist()
    unstable = np.lexsort((-np.arange(flat.size), flat)) // 2     # equal experts: later pairs first
    assert unstable.tolist() != perm.tolist()


# ---------------------------------------------------------------- NVFP4
_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e2m1(v, tie_even=True):
    """E2M1 nibble (sign << 3 | magnitude index), nearest with the given tie rule, saturating at 6."""
    sign = 0x8 if math.copysign(1.0, v) < 0 else 0x0
    a = min(abs(v), 6.0)
    best = min(range(8), key=lambda i: abs(_E2M1[i] - a))
    lo = max(i for i in range(8) if _E2M1[i] <= a)
    if lo < 7 and abs(a - _E2M1[lo]) == abs(_E2M1[lo + 1] - a):                # a tie
        best = (lo if lo % 2 == 0 else lo + 1) if tie_even else lo + 1
    return sign | best


def _nvfp4_block(vals, S, div=6.0, tie_even=True):
    f32 = np.float32
    amax = max(abs(v) for v in vals)
    sb = _e4m3(float(f32(f32(amax) * f32(S)) / f32(div)))
    e = (sb >> 3) & 0xF
    sf = (sb & 7) * 2.0 ** -9 if e == 0 else (1 + (sb & 7) / 8) * 2.0 ** (e - 7)
    if sf == 0.0:
        return [0] * len(vals), sb
    return [_e2m1(float(f32(f32(f32(v) * f32(S)) / f32(sf))), tie_even) for v in vals], sb


def _nvfp4_golden_ok(fn):
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_blocks.txt")
    for line in open(path, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, S, sb, pairs = [s.strip() for s in line.split("|")]
        vals = [float(p.split(":")[0]) for p in pairs.split()]
        nibs = [int(p.split(":")[1], 16) for p in pairs.split()]
        codes, got = fn(vals + [0.0] * (16 - len(vals)), float(S))
        if got != int(sb, 16) or codes[:len(nibs)] != nibs:
            return False
    return True


def test_nvfp4_restatement_passes_and_mutants_fail_the_golden_blocks():
    assert _nvfp4_golden_ok(_nvfp4_block)
    assert not _nvfp4_golden_ok(lambda v, S: _nvfp4_block(v, S, div=4.0))           # wrong E2M1 max in sf
    assert not _nvfp4_golden_ok(lambda v, S: _nvfp4_block(v, S, tie_even=False))    # ties away from zero
    assert not _nvfp4_golden_ok(lambda v, S: _nvfp4_block(v, 1.0))                  # tensor scale ignored


# ---------------------------------------------------------------- expert-parallel dispatch plan
def _ep_plan_restated(idx, E, P, owner=None, dedup=True, rec_relative=True, slot_major=False):
    """A loop restatement of the EP send plan with optional planted mistakes:
    owner(e) other than e // (E/P), one record per pair instead of per
    (token, rank), record indices counted from the start of the send buffer
    instead of the destination's first record, or pairs ordered slot-major."""
    T, k = idx.shape
    epr = E // P
    owner = owner or (lambda e: e // epr)
    counts = [0] * (2 * P)
    rec_token, pair_expert, pair_rec = [], [], []
    ret = -np.ones((T, k), dtype=np.int64)
    for p in range(P):
        rec0 = len(rec_token)
        order = [(t, j) for j in range(k) for t in range(T)] if slot_major else \
                [(t, j) for t in range(T) for j in range(k)]
        mine = {}
        for t, j in order:
            e = int(idx[t, j])
            if not (0 <= e < E) or owner(e) != p:
                continue
            if t not in mine or not dedup:
                mine[t] = len(rec_token) - (rec0 if rec_relative else 0)
                rec_token.append(t)
            ret[t, j] = len(pair_expert)
            pair_expert.append(e % epr)
            pair_rec.append(mine[t])
        counts[p] = len(rec_token) - rec0
        counts[P + p] = sum(1 for t, j in order if 0 <= int(idx[t, j]) < E and owner(int(idx[t, j])) == p)
    return counts, rec_token, pair_expert, pair_rec, ret


def _ep_plan_agrees(plan, idx, E, P):
    from tests.test_oracle_ep import brute_plan
    counts, rec_token, pe, prc, ret = brute_plan(idx, E, P)
    c2, rt2, pe2, prc2, ret2 = plan
    return counts == c2 and rec_token == rt2 and pe == pe2 and prc == prc2 and np.array_equal(ret, ret2)


@pytest.mark.parametrize("name,kw", [("owner by modulo", {"owner": "mod"}), ("no dedup", {"dedup": False}),
                                     ("absolute record index", {"rec_relative": False}),
                                     ("slot-major order", {"slot_major": True})])
def test_ep_plan_mutants_fail_the_brute_force_pin(name, kw):
    E, P = 12, 3
    idx = np.array([[0, 1, 5], [11, 4, 3], [7, 8, 2], [6, 9, 10], [1, 0, 4]], dtype=np.int32)
    # the restatement without mistakes and the oracle agree with the pin
    assert _ep_plan_agrees(_ep_plan_restated(idx, E, P), idx, E, P)
    pl = oracle.ep_plan(idx, E, P)
    assert _ep_plan_agrees((pl.counts.tolist(), pl.rec_token.tolist(), pl.pair_expert.tolist(),
                            pl.pair_rec.tolist(), pl.ret_pos), idx, E, P)
    if kw.get("owner") == "mod":
        kw = {"owner": lambda e: e % P}
    assert not _ep_plan_agrees(_ep_plan_restated(idx, E, P, **kw), idx, E, P), name
