"""GPU parity of the int8 output head with fused scale and argmax against the CPU oracle:
logits, argmax (int8 mode bit-exact; bf16 mode equal or within the near-tie bound), exact ties
and the full 151,936-row vocabulary."""
import functools

import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import PER_OUT, dev, host

pytestmark = pytest.mark.gpu


def _head(W, sh, X, M, mode, want_logits=True):
    V, K = W.shape
    ws = torch.zeros(tg.i8_head_workspace_bytes(V, M), dtype=torch.uint8, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    mv = torch.empty(M, dtype=torch.float32, device="cuda")
    lg = torch.empty(M * V, dtype=torch.float32, device="cuda") if want_logits else None
    Wd, shd = dev(W), dev(sh.view(np.float16))
    if mode == "bf16":
        tg.i8_head_gemv_argmax(Wd, shd, V, K, M, tg.TERN_ACT_BF16, dev(X.view(np.int16)), None, am, mv, lg, ws)
        q = sx = None
    else:
        q = torch.empty(M * K, dtype=torch.int8, device="cuda")
        sx = torch.empty(M, dtype=torch.float32, device="cuda")
        tg.tern_quantize_act(dev(X.view(np.int16)), M, K, q, sx)
        tg.i8_head_gemv_argmax(Wd, shd, V, K, M, tg.TERN_ACT_INT8, q, sx, am, mv, lg, ws)
    torch.cuda.synchronize()
    assert (host(ws) == 0).all(), "workspace must be left zero-filled"
    return (host(am), host(mv), host(lg).reshape(M, V) if lg is not None else None,
            None if q is None else (host(q).reshape(M, K), host(sx)))


def _check_bf16(am, mv, lg, X, W, sh):
    am_ref, mv_ref, lg_ref = oracle.head_bf16(W, sh, X, want_logits=True)
    absx = np.abs(synth.bf16_bits_to_f32(X).astype(np.float64)).sum(1)
    shf = sh.view(np.float16).astype(np.float64)
    bound = PER_OUT * absx[:, None] * 127.0 * shf[None, :]
    err = lg.astype(np.float64) - lg_ref
    assert np.linalg.norm(err) / np.linalg.norm(lg_ref) <= 1e-5
    assert (np.abs(err) <= bound).all()
    for m in range(X.shape[0]):
        # equal index, or the oracle logit at the GPU's index within the per-output bound of the max
        if am[m] != am_ref[m]:
            assert mv_ref[m] - lg_ref[m, am[m]] <= bound[m, am[m]], (m, am[m], am_ref[m])
        assert lg[m, am[m]] == mv[m]


@pytest.mark.parametrize("M", [1, 2, 7, 16])
@pytest.mark.parametrize("V,K", [(1000, 1024), (517, 4096), (4099, 128)])
def test_head(V, K, M):
    W = synth.head_weights(61, V + K, V, K)
    sh = synth.head_scales(61, V + K, V)
    X = synth.activations(61, M, M, K)
    am, mv, lg, _ = _head(W, sh, X, M, "bf16")
    _check_bf16(am, mv, lg, X, W, sh)
    am, mv, lg, (q, sx) = _head(W, sh, X, M, "int8")
    am_ref, mv_ref, lg_ref = oracle.head_i8(W, sh, q, sx, want_logits=True)
    assert (lg == lg_ref).all()
    assert (am == am_ref).all() and (mv == mv_ref).all()


@pytest.mark.parametrize("mode", ["bf16", "int8"])
def test_head_exact_ties_lowest_index(mode):
    V, K, M = 3000, 1024, 3
    W = synth.head_weights(62, 1, V, K)
    sh = synth.head_scales(62, 1, V)
    X = synth.activations(62, 2, M, K)
    # duplicate the oracle's winning row at a lower and a higher index: exact tie, lowest wins
    am0, _, _ = oracle.head_bf16(W, sh, X)
    for m in range(M):
        w = am0[m]
        for r in (5 + m, V - 1 - m):
            W[r] = W[w]
            sh[r] = sh[w]
    am, mv, lg, qs = _head(W, sh, X, M, mode)
    if mode == "int8":
        am_ref, _, lg_ref = oracle.head_i8(W, sh, qs[0], qs[1], want_logits=True)
        assert (am == am_ref).all()
    for m in range(M):
        best = lg[m].max()
        assert am[m] == np.flatnonzero(lg[m] == best)[0]


@functools.lru_cache(maxsize=2)
def _full_head(K):
    V = 151936
    return synth.head_weights(63, 252, V, K), synth.head_scales(63, 252, V)


@pytest.mark.parametrize("mode", ["bf16", "int8"])
@pytest.mark.parametrize("K,M", [(4096, 1), (4096, 7), (1024, 1)])
def test_head_full_vocab(mode, K, M):
    V = 151936
    W, sh = _full_head(K)
    X = synth.activations(63, 3, M, K)
    am, mv, lg, qs = _head(W, sh, X, M, mode)
    if mode == "bf16":
        _check_bf16(am, mv, lg, X, W, sh)
    else:
        am_ref, mv_ref, lg_ref = oracle.head_i8(W, sh, qs[0], qs[1], want_logits=True)
        assert (lg == lg_ref).all() and (am == am_ref).all() and (mv == mv_ref).all()
    # without logits the argmax is the same
    am2, mv2, _, _ = _head(W, sh, X, M, mode, want_logits=False)
    assert (am2 == am).all() and (mv2 == mv).all()
