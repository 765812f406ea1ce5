"""GPU parity of the M = 1 ternary GEMV (both activation modes) against the CPU oracle, through
the C ABI: small ragged shapes, the single-GEMV configuration (3072 x 1024), the 0.6B and 8B
linear shapes (full output for the smaller ones, sampled rows for the largest), closed forms and
determinism. int8 mode is bit-exact; bf16 mode meets the stated tolerance."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import check_bf16, dev, host, make_matrix

pytestmark = pytest.mark.gpu

SHAPES = [(1, 128), (37, 384), (200, 640), (3072, 1024), (2048, 1024), (1024, 3072), (4096, 4096),
          (6144, 4096), (129, 12288)]


def _run_bf16(W, x):
    y = torch.empty(W.N, dtype=torch.float32, device="cuda")
    tg.tern_gemv(W, tg.TERN_ACT_BF16, dev(x.view(np.int16)), None, y)
    return host(y)


def _run_i8(W, x, K, with_acc=False):
    q = torch.empty(K, dtype=torch.int8, device="cuda")
    sx = torch.empty(1, dtype=torch.float32, device="cuda")
    tg.tern_quantize_act(dev(x.view(np.int16)), 1, K, q, sx)
    y = torch.empty(W.N, dtype=torch.float32, device="cuda")
    acc = torch.full((W.N,), -7, dtype=torch.int32, device="cuda") if with_acc else None
    tg.tern_gemv(W, tg.TERN_ACT_INT8, q, sx, y, acc=acc)
    if with_acc:
        return host(q), host(sx), host(y), host(acc)
    return host(q), host(sx), host(y)


@pytest.mark.parametrize("N,K", SHAPES)
def test_gemv_bf16(N, K):
    W, t, s = make_matrix(41, N * 13 + K, N, K)
    x = synth.activations(41, K, 1, K)
    y = _run_bf16(W, x)
    y_ref = oracle.gemm_bf16(oracle.pack(t), s, K, x)
    check_bf16(y[None, :], y_ref, x, s)


@pytest.mark.parametrize("N,K", SHAPES)
def test_gemv_int8_bit_exact(N, K):
    W, t, s = make_matrix(42, N * 13 + K, N, K)
    x = synth.activations(42, K, 1, K)
    q, sx, y, acc = _run_i8(W, x, K, with_acc=True)
    q_ref, sx_ref = oracle.quantize_act(x, K)
    assert (q == q_ref[0]).all() and sx[0] == sx_ref[0]
    acc_ref, y_ref = oracle.gemm_i8(oracle.pack(t), s, K, q_ref, sx_ref)
    assert (acc == acc_ref[0]).all(), "int32 accumulators"
    assert (y == y_ref[0]).all()


@pytest.mark.parametrize("N,K,sparse", [(24576, 4096, False), (4096, 12288, True), (12288, 4096, True)])
def test_gemv_8b_full_size_sampled(N, K, sparse):
    """Largest 8B launches (fused gate|up, down) with device-generated weights; 96 sampled rows."""
    p = synth.P_SPARSE_FFN if sparse else synth.P_DEFAULT
    W, _, s = make_matrix(43, 7, N, K, p, host_trits=False)
    x = synth.activations(43, 9, 1, K)
    rows = np.sort(np.random.default_rng(N).choice(N, 96, replace=False))
    rows[0], rows[-1] = 0, N - 1
    t_rows = synth.trits(43, 7, N, K, p, rows=rows)
    y = _run_bf16(W, x)
    y_ref = oracle.gemm_bf16(oracle.pack(t_rows), s[rows], K, x)
    check_bf16(y[rows][None, :], y_ref, x, s[rows])
    q, sx, yi = _run_i8(W, x, K)
    _, yi_ref = oracle.gemm_i8(oracle.pack(t_rows), s[rows], K, q[None, :], sx)
    assert (yi[rows] == yi_ref[0]).all()


def test_closed_forms():
    N, K = 300, 1024
    s = synth.row_scales(44, 0, N)
    x = synth.activations(44, 1, 1, K)
    xs = synth.bf16_bits_to_f32(x).astype(np.float64).sum()
    for fill, sign in ((0, 0), (1, 1), (-1, -1)):
        t = np.full((N, K), fill, np.int8)
        W = tg.TernMatrix(dev(oracle.pack(t).view(np.int32)), dev(s.view(np.float16)), N, K)
        y = _run_bf16(W, x)
        ref = sign * xs * s.view(np.float16).astype(np.float64)
        check_bf16(y[None, :], ref[None, :], x, s) if fill else None
        if fill == 0:
            assert (y == 0).all()
    # a zero activation vector gives exact zeros in both modes
    t = synth.trits(44, 2, N, K)
    W = tg.TernMatrix(dev(oracle.pack(t).view(np.int32)), dev(s.view(np.float16)), N, K)
    z = np.zeros((1, K), np.uint16)
    assert (_run_bf16(W, z) == 0).all()
    q, sx, y = _run_i8(W, z, K)
    assert sx[0] == 0 and (q == 0).all() and (y == 0).all()


def test_wide_dynamic_range_bf16():
    N, K = 256, 2048
    W, t, s = make_matrix(45, 3, N, K)
    xf = synth.bf16_bits_to_f32(synth.activations(45, 4, 1, K))
    xf = xf * np.float32(2.0) ** np.random.default_rng(1).integers(-20, 20, K).astype(np.float32)
    x = synth.f32_to_bf16_bits(xf)
    y = _run_bf16(W, x)
    check_bf16(y[None, :], oracle.gemm_bf16(oracle.pack(t), s, K, x), x, s)


def test_deterministic():
    N, K = 4096, 4096
    W, _, _ = make_matrix(46, 5, N, K)
    x = synth.activations(46, 6, 1, K)
    a, b = _run_bf16(W, x), _run_bf16(W, x)
    assert (a.view(np.uint32) == b.view(np.uint32)).all()
