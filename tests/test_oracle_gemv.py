"""Pins of the oracle's ternary GEMV / GEMM (bf16 activations, fp64 sums): a hand-worked example,
numpy brute force, exhaustive small trit patterns and closed forms."""
import os

import numpy as np
import pytest

import oracle
import synth


def _f16(vals):
    return np.asarray(vals, np.float16).view(np.uint16)


def _bf16(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, np.float32))


def test_hand_example(golden_dir):
    K, xs, rows, ys = 128, {}, {}, {}
    for line in open(os.path.join(golden_dir, "gemv_tiny.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        f = line.split()
        if f[0] == "x":
            xs[int(f[1])] = float(f[2])
        elif f[0] == "row":
            pairs = [(int(f[i]), int(f[i + 1])) for i in range(3, len(f), 2)]
            rows[int(f[1])] = (float(f[2]), pairs)
        elif f[0] == "y":
            ys[int(f[1])] = float(f[2])
    N = len(rows)
    t = np.zeros((N, K), np.int8)
    s = np.zeros(N, np.float32)
    for n, (sc, pairs) in rows.items():
        s[n] = sc
        for k, v in pairs:
            t[n, k] = v
    x = np.zeros(K, np.float32)
    for k, v in xs.items():
        x[k] = v
    y = oracle.gemm_bf16(oracle.pack(t), _f16(s), K, _bf16(x))
    assert y.shape == (1, N)
    for n, v in ys.items():
        assert y[0, n] == v


@pytest.mark.parametrize("N,K,M", [(37, 128, 1), (64, 256, 3), (19, 384, 5), (128, 1024, 2)])
def test_brute_force(N, K, M):
    t = synth.trits(3, N * 7 + K, N, K)
    s = synth.row_scales(3, N, N)
    x = synth.activations(3, K, M, K)
    y = oracle.gemm_bf16(oracle.pack(t), s, K, x)
    ref = (synth.bf16_bits_to_f32(x).astype(np.float64) @ t.astype(np.float64).T) \
        * s.view(np.float16).astype(np.float64)[None, :]
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=0)


def test_exhaustive_patterns():
    # every trit pattern of length 5 in the first columns; x_k = 3^k makes each row's sum the
    # balanced-ternary value of its pattern, so the 243 rows give the 243 integers -121..121
    N, K = 243, 128
    t = np.zeros((N, K), np.int8)
    for n in range(N):
        v = n
        for i in range(5):
            t[n, i] = v % 3 - 1
            v //= 3
    x = np.zeros(K, np.float32)
    x[:5] = [1, 3, 9, 27, 81]
    y = oracle.gemm_bf16(oracle.pack(t), _f16(np.ones(N)), K, _bf16(x))[0]
    expect = t[:, :5].astype(np.float64) @ np.array([1, 3, 9, 27, 81], np.float64)
    assert (y == expect).all()
    assert sorted(y.tolist()) == list(range(-121, 122))


def test_closed_forms():
    K, N = 256, 8
    x = synth.activations(4, 0, 1, K)
    xf = synth.bf16_bits_to_f32(x)[0].astype(np.float64)
    s = synth.row_scales(4, 0, N)
    sf = s.view(np.float16).astype(np.float64)
    # all-zero weights
    assert (oracle.gemm_bf16(oracle.pack(np.zeros((N, K), np.int8)), s, K, x) == 0).all()
    # all +1 weights: s * sum(x)
    y = oracle.gemm_bf16(oracle.pack(np.ones((N, K), np.int8)), s, K, x)[0]
    np.testing.assert_allclose(y, sf * xf.sum(), rtol=1e-14)
    # all -1 weights: -s * sum(x)
    y = oracle.gemm_bf16(oracle.pack(-np.ones((N, K), np.int8)), s, K, x)[0]
    np.testing.assert_allclose(y, -sf * xf.sum(), rtol=1e-14)
    # one nonzero per row picks +-s*x_k
    t = np.zeros((N, K), np.int8)
    ks = [0, 1, 31, 32, 100, 200, 254, 255]
    for n, k in enumerate(ks):
        t[n, k] = 1 if n % 2 else -1
    y = oracle.gemm_bf16(oracle.pack(t), s, K, x)[0]
    for n, k in enumerate(ks):
        assert y[n] == (1 if n % 2 else -1) * sf[n] * xf[k]


def test_unit_vectors_reconstruct_matrix():
    N, K = 12, 128
    t = synth.trits(8, 2, N, K)
    pl = oracle.pack(t)
    ones = _f16(np.ones(N))
    eye = np.eye(K, dtype=np.float32)
    Y = oracle.gemm_bf16(pl, ones, K, _bf16(eye))      # M = K rows of unit vectors
    assert (Y.T == t).all()
