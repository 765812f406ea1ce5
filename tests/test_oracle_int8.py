"""Pins of the oracle's int8-activation path: hand-worked quantisation (ties to even, zero row),
exact int64 accumulation against numpy, and the fp32 epilogue."""
import os

import numpy as np
import pytest

import oracle
import synth


def _bf16(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, np.float32))


def test_quantize_hand_examples(golden_dir):
    n = 0
    for line in open(os.path.join(golden_dir, "quant_examples.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        xs, sx, qs = line.split("|")
        x = np.array([float(v) for v in xs.split()], np.float32)
        K = 128
        xx = np.zeros(K, np.float32)
        xx[:x.size] = x
        q, s = oracle.quantize_act(_bf16(xx), K)
        assert s[0] == np.float32(float(sx))
        assert q[0, :x.size].tolist() == [int(v) for v in qs.split()]
        assert (q[0, x.size:] == 0).all()
        n += 1
    assert n == 3


def test_quantize_matches_ieee_fp32():
    # an independent fp32 (IEEE, numpy) computation of the same definition on random rows
    K = 512
    x = synth.activations(6, 1, 9, K)
    q, s = oracle.quantize_act(x, K)
    xf = synth.bf16_bits_to_f32(x)
    amax = np.abs(xf).max(1)
    s_ref = amax / np.float32(127.0)
    assert (s == s_ref).all()
    q_ref = np.clip(np.rint(xf / s_ref[:, None]), -127, 127).astype(np.int8)
    assert (q == q_ref).all()
    assert (np.abs(q) == 127).sum(1).min() >= 1                # the absmax element maps to +-127


@pytest.mark.parametrize("N,K,M", [(33, 128, 1), (64, 512, 4), (17, 1024, 16)])
def test_int8_gemm_exact(N, K, M):
    t = synth.trits(12, N + M, N, K)
    s = synth.row_scales(12, N, N)
    x = synth.activations(12, K + M, M, K)
    q, sx = oracle.quantize_act(x, K)
    acc, y = oracle.gemm_i8(oracle.pack(t), s, K, q, sx)
    acc_ref = q.astype(np.int64) @ t.astype(np.int64).T
    assert (acc == acc_ref).all()
    y_ref = (acc_ref.astype(np.float32) * sx[:, None]) * s.view(np.float16).astype(np.float32)[None, :]
    assert (y == y_ref).all()
