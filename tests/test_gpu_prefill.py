"""GPU parity of the prefill dense contraction (tern_gemm_prefill: tcgen05 MMA, TMEM accumulators)
against the CPU oracle, within the bf16-mode tolerance (relative L2 <= 1e-5 over the outputs and
|err| <= 1e-4 * sum_k |x_k| * scale[n] per output): full outputs at small M, every weight row for
sampled tokens at the 8B prefill size M = 4096, ragged M and N, and argument errors."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import check_bf16, dev, host, make_matrix

pytestmark = pytest.mark.gpu


def _prefill(W, X):
    M = X.shape[0]
    Y = torch.full((M * W.N,), float("nan"), dtype=torch.float32, device="cuda")
    tg.tern_gemm_prefill(W, M, dev(X.view(np.int16)), Y)
    torch.cuda.synchronize()
    assert tg.tern_device_status() == tg.TERN_OK
    return host(Y).reshape(M, W.N)


# The last two shapes give at least 148 tiles of 256 tokens x 256 rows, so they run the two-halves
# kernel (both 128-token halves of a tile share each expanded weight stage) with a ragged M and N.
@pytest.mark.parametrize("N,K,M", [(256, 128, 128), (512, 1024, 200), (300, 640, 130), (1024, 4096, 256),
                                   (256, 12288, 64), (4096, 128, 1), (18944, 128, 300), (18901, 256, 257)])
def test_prefill_full(N, K, M):
    W, t, s = make_matrix(51, N + K, N, K)
    X = synth.activations(51, M + K, M, K)
    Y = _prefill(W, X)
    check_bf16(Y, oracle.gemm_bf16(oracle.pack(t), s, K, X), X, s)


@pytest.mark.parametrize("proj", ["q", "k", "o", "gate", "down"])
def test_prefill_8b_shapes_sampled_tokens(proj):
    """M = 4096 tokens through an 8B linear shape; 64 sampled tokens (the first and the last among
    them) checked against every row."""
    N, K = {p: (n, k) for p, n, k in synth.linear_shapes("8b")}[proj]
    M = 4096
    W, t, s = make_matrix(52, 7000 + N + K, N, K, host_trits=False)
    X = synth.activations(52, N + K, M, K)
    Y = _prefill(W, X)
    toks = np.sort(np.random.default_rng(N + K).choice(M, 64, replace=False))
    toks[0], toks[-1] = 0, M - 1
    tr = synth.trits(52, 7000 + N + K, N, K)
    check_bf16(Y[toks], oracle.gemm_bf16(oracle.pack(tr), s, K, X[toks]), X[toks], s)


def test_prefill_matches_gemv_rows():
    """Every token row of the prefill equals the M = 1 GEMV of that token within the tolerance."""
    N, K, M = 768, 1024, 9
    W, t, s = make_matrix(53, 1, N, K)
    X = synth.activations(53, 2, M, K)
    Y = _prefill(W, X)
    for m in range(M):
        y = torch.empty(N, dtype=torch.float32, device="cuda")
        tg.tern_gemv(W, tg.TERN_ACT_BF16, dev(X[m].view(np.int16)), None, y)
        check_bf16(Y[m][None, :], host(y).astype(np.float64)[None, :], X[m][None, :], s)


def test_prefill_argument_errors():
    W = tg.TernMatrix.empty(256, 128)
    X = torch.zeros(128 * 4, dtype=torch.int16, device="cuda")
    Y = torch.zeros(256 * 4, dtype=torch.float32, device="cuda")
    with pytest.raises(tg.TernError):
        tg.tern_gemm_prefill(W, 0, X, Y)                      # M < 1
    with pytest.raises(tg.TernError):
        tg.tern_gemm_prefill(W, 4, X[1:], Y)                  # misaligned X
