"""GPU parity of the small-M GEMM (speculative-verify batch sizes) against the CPU oracle."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import check_bf16, dev, host, make_matrix

pytestmark = pytest.mark.gpu


def _bf16(W, X, M):
    Y = torch.empty(M * W.N, dtype=torch.float32, device="cuda")
    tg.tern_gemm_small_m(W, M, tg.TERN_ACT_BF16, dev(X.view(np.int16)), None, Y)
    return host(Y).reshape(M, W.N)


def _i8(W, X, M, K):
    q = torch.empty(M * K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    tg.tern_quantize_act(dev(X.view(np.int16)), M, K, q, sx)
    Y = torch.empty(M * W.N, dtype=torch.float32, device="cuda")
    tg.tern_gemm_small_m(W, M, tg.TERN_ACT_INT8, q, sx, Y)
    return host(q).reshape(M, K), host(sx), host(Y).reshape(M, W.N)


@pytest.mark.parametrize("M", [1, 2, 4, 7, 8, 9, 16])
@pytest.mark.parametrize("N,K", [(37, 384), (1000, 1024), (4096, 4096), (1024, 12288)])
def test_small_m(M, N, K):
    W, t, s = make_matrix(51, N + K, N, K)
    X = synth.activations(51, K + M, M, K)
    Y = _bf16(W, X, M)
    check_bf16(Y, oracle.gemm_bf16(oracle.pack(t), s, K, X), X, s)
    q, sx, Yi = _i8(W, X, M, K)
    q_ref, sx_ref = oracle.quantize_act(X, K)
    assert (q == q_ref).all() and (sx == sx_ref).all()
    _, Y_ref = oracle.gemm_i8(oracle.pack(t), s, K, q_ref, sx_ref)
    assert (Yi == Y_ref).all()


@pytest.mark.parametrize("M", [7, 16])
def test_small_m_8b_gate_up_sampled(M):
    N, K = 24576, 4096
    W, _, s = make_matrix(52, 4, N, K, host_trits=False)
    X = synth.activations(52, 5, M, K)
    rows = np.sort(np.random.default_rng(M).choice(N, 64, replace=False))
    t_rows = synth.trits(52, 4, N, K, rows=rows)
    Y = _bf16(W, X, M)
    check_bf16(Y[:, rows], oracle.gemm_bf16(oracle.pack(t_rows), s[rows], K, X), X, s[rows])
