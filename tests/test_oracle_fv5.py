"""Pins of the oracle's five-valued (FV5-style) weights and block-scaled (FV5B-style) head:
hand-worked bit positions and a hand-worked product (tests/golden/fv5_examples.txt), round
trips over every code, numpy brute force of both products, closed forms and the head's
lowest-index tie rule."""
import os

import numpy as np
import pytest

import oracle
import synth

K2 = 512


def _golden(golden_dir):
    for line in open(os.path.join(golden_dir, "fv5_examples.txt")):
        line = line.split("#")[0].strip()
        if line:
            yield [p.split() for p in line.split("|")]


def test_layout_hand_examples(golden_dir):
    n = 0
    for parts in _golden(golden_dir):
        if parts[0] != ["layout"]:
            continue
        k, c = int(parts[1][0]), int(parts[1][1])
        codes = np.zeros((1, K2), np.int8)
        codes[0, k] = c
        planes = oracle.fv5_pack(codes).reshape(3, K2 // 32)
        want = {tuple(int(v) for v in b.split(":")) for b in parts[2]}
        got = {(pl, w, b) for pl in range(3) for w in range(K2 // 32) for b in range(32) if (planes[pl, w] >> b) & 1}
        assert got == want, (k, c)
        n += 1
    assert n == 5


def test_product_hand_example(golden_dir):
    for parts in _golden(golden_dir):
        if parts[0] != ["product"]:
            continue
        v = [int(x) for x in parts[1]]
        codes = np.zeros((1, K2), np.int8)
        q = np.zeros((1, K2), np.int8)
        for i in range(0, len(v), 3):
            codes[0, v[i]], q[0, v[i]] = v[i + 1], v[i + 2]
        s = np.array([float(x) for x in parts[2]], np.float32).reshape(1, 2, 2)
        sx = np.array([float(parts[3][0])], np.float32)
        y = oracle.fv5_gemm_i8(oracle.fv5_pack(codes), s, K2, q, sx)
        assert y[0, 0] == np.float32(float(parts[4][0]))
        return
    raise AssertionError("no product example")


def _codes(rng, N, K):
    return rng.choice(np.array([-2, -1, 0, 1, 2], np.int8), size=(N, K), p=[0.05, 0.14, 0.62, 0.14, 0.05])


def _dense(codes, scales):
    N, K = codes.shape
    s = scales.reshape(N, K // 256, 2).astype(np.float64)
    mag = np.where(np.abs(codes) == 2, 1, 0)
    blk = np.arange(K) // 256
    w = np.sign(codes) * s[np.arange(N)[:, None], blk[None, :], mag]
    return w


def test_k_must_be_whole_groups():
    with pytest.raises(oracle.OracleError):
        oracle.fv5_pack(np.zeros((2, 768), np.int8))


def test_round_trip_every_code():
    rng = np.random.default_rng(1)
    c = _codes(rng, 7, 1024)
    c[0, :5] = [-2, -1, 0, 1, 2]
    planes = oracle.fv5_pack(c)
    assert (oracle.fv5_unpack(planes, 1024) == c).all()
    p3 = planes.reshape(7, 3, 32)
    popc = lambda a: np.unpackbits(a.view(np.uint8)).sum()
    assert popc(p3[:, 0]) == np.count_nonzero(c) and popc(p3[:, 1]) == np.count_nonzero(c < 0)
    assert popc(p3[:, 2]) == np.count_nonzero(np.abs(c) == 2)


def test_gemm_bf16_brute_force_and_closed_forms():
    rng = np.random.default_rng(2)
    N, K, M = 40, 1536, 3
    c = _codes(rng, N, K)
    s = (rng.random((N, K // 256, 2)) * 0.05 + 0.01).astype(np.float32)
    x = synth.activations(2, 1, M, K)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    y = oracle.fv5_gemm_bf16(oracle.fv5_pack(c), s, K, x)
    assert np.allclose(y, xf @ _dense(c, s).T, rtol=1e-12, atol=1e-12)
    # all codes +2: y = sum_b s_hi[b] * (sum of x over block b)
    c2 = np.full((N, K), 2, np.int8)
    y2 = oracle.fv5_gemm_bf16(oracle.fv5_pack(c2), s, K, x)
    bs = xf.reshape(M, K // 256, 256).sum(2)
    assert np.allclose(y2, bs @ s[:, :, 1].astype(np.float64).T, rtol=1e-12)


def test_gemm_i8_brute_force():
    rng = np.random.default_rng(3)
    N, K, M = 33, 1024, 4
    c = _codes(rng, N, K)
    s = (rng.random((N, K // 256, 2)) * 0.05 + 0.01).astype(np.float32)
    q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    sx = (rng.random(M) * 0.1).astype(np.float32)
    y = oracle.fv5_gemm_i8(oracle.fv5_pack(c), s, K, q, sx)
    # independent: exact block sums with numpy int64, fp64 sum in block order, one fp32 rounding
    lo = (np.abs(c) == 1) * np.sign(c)
    hi = (np.abs(c) == 2) * np.sign(c)
    for m in range(M):
        for n in range(N):
            tot = 0.0
            for b in range(K // 256):
                sl = slice(256 * b, 256 * b + 256)
                tot += float(s[n, b, 0]) * int((lo[n, sl].astype(np.int64) * q[m, sl]).sum()) + \
                    float(s[n, b, 1]) * int((hi[n, sl].astype(np.int64) * q[m, sl]).sum())
            assert y[m, n] == np.float32(float(sx[m]) * tot)


def test_head_brute_force_and_ties():
    rng = np.random.default_rng(4)
    V, K, M = 300, 512, 2
    W = rng.integers(-127, 128, (V, K)).astype(np.int8)
    S = (rng.random((V, K // 256)) * 0.02).astype(np.float32)
    x = synth.activations(4, 1, M, K)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    am, lg = oracle.fv5b_head(W, S, x_bf16=x)
    dense = W.astype(np.float64) * np.repeat(S.astype(np.float64), 256, axis=1)
    assert np.allclose(lg, xf @ dense.T, rtol=1e-12, atol=1e-12)
    assert (am == lg.argmax(1)).all()
    # exact tie: the winner duplicated at a higher index keeps the lower index
    w = int(am[0])
    other = V - 1 if w < V // 2 else 0
    W[other], S[other] = W[w], S[w]
    am2, lg2 = oracle.fv5b_head(W, S, x_bf16=x)
    assert am2[0] == min(w, other) and lg2[0, w] == lg2[0, other]
    # int8 mode: fp32(s_x * sum_b s_b A_b)
    q = rng.integers(-127, 128, (M, K)).astype(np.int8)
    sx = np.array([0.01, 0.03], np.float32)
    _, lgq = oracle.fv5b_head(W, S, q=q, sx=sx)
    A = (W.astype(np.int64)[None] * q.astype(np.int64)[:, None, :]).reshape(M, V, K // 256, 256).sum(3)
    for m in range(M):
        for v in range(0, V, 37):
            tot = 0.0
            for b in range(K // 256):
                tot += float(S[v, b]) * float(A[m, v, b])
            assert lgq[m, v] == float(np.float32(float(sx[m]) * tot))
