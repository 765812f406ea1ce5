"""Pins of the oracle's steps on either side of the linears and of the verify acceptance rule:
fp64 -> bf16 rounding (brute force over the bf16 grid in exact rational arithmetic), RMSNorm and
SwiGLU (hand-worked fixtures, invariants, an independent scalar recomputation) and the
longest-prefix acceptance count (hand-worked fixture, brute force over prefixes, and the
lowest-index tie rule of the head's argmax)."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth


def _rows(path):
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            yield [part.split() for part in line.split("|")]


def _bf16_grid():
    """All finite non-negative bf16 values in increasing order, with their bit patterns."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)
    vals = (bits << 16).view(np.float32).astype(np.float64)
    return vals, bits.astype(np.uint16)


_GRID = _bf16_grid()


def _nearest_bf16(v: float) -> int:
    """Brute force: the bf16 value nearest to v in exact rational arithmetic, ties to the even
    bit pattern; magnitudes at or beyond the midpoint above the largest finite value -> infinity."""
    vals, bits = _GRID
    sign = 0x8000 if math.copysign(1.0, v) < 0 else 0
    a = abs(v)
    top = Fraction(vals[-1]) + (Fraction(vals[-1]) - Fraction(vals[-2])) / 2
    if Fraction(a) >= top:
        return sign | 0x7F80
    i = int(np.searchsorted(vals, a))
    cands = [j for j in (i - 1, i) if 0 <= j < vals.size]
    fa = Fraction(a)
    best = min(cands, key=lambda j: (abs(Fraction(vals[j]) - fa), int(bits[j]) & 1))
    return sign | int(bits[best])


def test_round_bf16_brute_force():
    rng = np.random.default_rng(5)
    vals, _ = _GRID
    xs = list(rng.standard_normal(300) * 2.0 ** rng.integers(-140, 130, 300))
    # midpoints between neighbouring bf16 values (exact in fp64): ties go to the even pattern
    idx = rng.integers(1, vals.size - 1, 200)
    xs += [(vals[i] + vals[i + 1]) / 2 for i in idx] + [-(vals[i] + vals[i + 1]) / 2 for i in idx[:50]]
    xs += [vals[1] / 2, vals[1] * 1.5, vals[127] + vals[1] / 2, 2.0 ** -126 - 2.0 ** -134, 3.0e38, 3.4e38, -3.5e38]
    for x in xs:
        assert int(oracle.round_bf16(x)) == _nearest_bf16(float(x)), x


def test_round_bf16_fixed_points_and_specials():
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    ok = np.isfinite(f)
    got = oracle.round_bf16(f[ok].astype(np.float64))
    assert (got == bits[ok].astype(np.uint16)).all()
    assert int(oracle.round_bf16(float("inf"))) == 0x7F80 and int(oracle.round_bf16(float("-inf"))) == 0xFF80
    assert int(oracle.round_bf16(float("nan"))) & 0x7F80 == 0x7F80


def test_rmsnorm_hand_examples(golden_dir):
    n = 0
    for x, g, eps, out in _rows(os.path.join(golden_dir, "rmsnorm_examples.txt")):
        xv = np.array([float(v) for v in x], np.float32)
        gv = synth.f32_to_bf16_bits(np.array([float(v) for v in g], np.float32))
        got = oracle.rmsnorm(xv, gv, float(eps[0]))[0]
        assert [int(v) for v in got] == [int(h, 16) for h in out], (x, g, eps)
        n += 1
    assert n == 4


def _rmsnorm_scalar(x, gain_bits, eps):
    """The definition recomputed with Python floats: fsum of the squares, then the nearest bf16."""
    K = len(x)
    r = 1.0 / math.sqrt(math.fsum(float(v) * float(v) for v in x) / K + eps)
    g = synth.bf16_bits_to_f32(gain_bits).astype(np.float64)
    return [_nearest_bf16((float(v) * r) * float(gk)) for v, gk in zip(x, g)]


def test_rmsnorm_matches_scalar_recomputation():
    rng = np.random.default_rng(7)
    for K, eps in ((128, 1e-6), (384, 1e-5), (64, 0.0)):
        x = (rng.standard_normal(K) * 3).astype(np.float32)
        gain = synth.f32_to_bf16_bits((1 + 0.1 * rng.standard_normal(K)).astype(np.float32))
        assert [int(v) for v in oracle.rmsnorm(x, gain, eps)[0]] == _rmsnorm_scalar(x, gain, eps)


def test_rmsnorm_invariants():
    rng = np.random.default_rng(8)
    K = 256
    x = rng.standard_normal((3, K)).astype(np.float32)
    ones = np.full(K, 0x3F80, np.uint16)
    base = oracle.rmsnorm(x, ones, 0.0)
    # invariant under a positive power-of-two scaling of the row (exact in fp32 and fp64)
    assert (oracle.rmsnorm(x * np.float32(8.0), ones, 0.0) == base).all()
    # odd in x
    neg = oracle.rmsnorm(-x, ones, 0.0)
    assert ((neg ^ 0x8000) == base).all()
    # unit gain: the output's mean square is 1 up to the bf16 rounding (relative 2^-8 per value)
    ms = (synth.bf16_bits_to_f32(base).astype(np.float64) ** 2).mean(1)
    assert np.abs(ms - 1).max() < 2 * 2.0 ** -8
    # the gain multiplies elementwise: gain 2 doubles every value exactly
    twos = np.full(K, 0x4000, np.uint16)
    assert (synth.bf16_bits_to_f32(oracle.rmsnorm(x, twos, 0.0)) == 2 * synth.bf16_bits_to_f32(base)).all()


def test_swiglu_hand_examples(golden_dir):
    n = 0
    for gu, out in _rows(os.path.join(golden_dir, "swiglu_examples.txt")):
        g, u = float(gu[0]), float(gu[1])
        got = oracle.swiglu(np.array([g, u], np.float32), 1)[0, 0]
        assert int(got) == int(out[0], 16), (g, u)
        n += 1
    assert n == 6


def test_swiglu_matches_scalar_recomputation_and_identity():
    rng = np.random.default_rng(9)
    K = 512
    g = (rng.standard_normal(K) * 4).astype(np.float32)
    u = (rng.standard_normal(K) * 2).astype(np.float32)
    got = oracle.swiglu(np.concatenate([g, u])[None, :], K)[0]
    want = [_nearest_bf16(float(z) / (1.0 + math.exp(-float(z))) * float(w)) for z, w in zip(g, u)]
    assert [int(v) for v in got] == want
    # silu(-z) = silu(z) - z, so with up = 1: out(-z) is the bf16 of out(z) - z before rounding
    ones = np.ones(K, np.float32)
    neg = oracle.swiglu(np.concatenate([-g, ones])[None, :], K)[0]
    want_neg = [_nearest_bf16(float(z) / (1.0 + math.exp(-float(z))) - float(z)) for z in g]
    assert [int(v) for v in neg] == want_neg
    # zero gate or zero up gives zero
    assert (oracle.swiglu(np.concatenate([np.zeros(K, np.float32), u])[None, :], K) & 0x7FFF == 0).all()
    assert (oracle.swiglu(np.concatenate([g, np.zeros(K, np.float32)])[None, :], K) & 0x7FFF == 0).all()


def test_verify_accept_hand_examples(golden_dir):
    n = 0
    for am, dr, out in _rows(os.path.join(golden_dir, "verify_examples.txt")):
        got = oracle.verify_accept([int(v) for v in am], [int(v) for v in dr])
        assert got == (int(out[0]), int(out[1])), (am, dr)
        n += 1
    assert n == 5


def test_verify_accept_brute_force():
    rng = np.random.default_rng(10)
    for _ in range(500):
        k = int(rng.integers(0, 8))
        am = rng.integers(0, 4, k + 1)
        dr = np.where(rng.random(k) < 0.8, am[:k], rng.integers(0, 4, k))
        n = max(j for j in range(k + 1) if (dr[:j] == am[:j]).all())
        assert oracle.verify_accept(am, dr) == (n, int(am[n]))


def test_verify_accept_takes_the_lowest_index_of_an_exact_tie():
    """A head with duplicated rows: the argmax is the lowest of the tied indices, so a draft naming
    the higher duplicate is rejected and the lower one accepted."""
    V, K = 64, 128
    W = synth.head_weights(11, 1, V, K)
    sh = synth.head_scales(11, 1, V)
    q = np.random.default_rng(2).integers(-127, 128, (2, K)).astype(np.int8)
    sx = np.array([0.01, 0.02], np.float32)
    am0, _, _ = oracle.head_i8(W, sh, q, sx)
    w = int(am0[0])
    other = V - 1 if w < V // 2 else 0
    W[other], sh[other] = W[w], sh[w]                # exact tie between w and other
    lo, hi = min(w, other), max(w, other)
    am, _, lg = oracle.head_i8(W, sh, q, sx, want_logits=True)
    assert am[0] == lo and lg[0, hi] == lg[0, lo]
    assert oracle.verify_accept(am, [hi]) == (0, lo)
    assert oracle.verify_accept(am, [lo]) == (1, int(am[1]))
