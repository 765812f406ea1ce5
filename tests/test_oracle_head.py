"""Pins of the oracle's int8 output head with greedy argmax: numpy logits, planted maxima,
exact ties (lowest index wins) and the last index."""
import numpy as np
import pytest

import oracle
import synth


def _bf16(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, np.float32))


def test_logits_match_numpy():
    V, K, M = 300, 256, 3
    W = synth.head_weights(2, 252, V, K)
    sh = synth.head_scales(2, 252, V)
    x = synth.activations(2, 99, M, K)
    am, mv, lg = oracle.head_bf16(W, sh, x, want_logits=True)
    ref = (synth.bf16_bits_to_f32(x).astype(np.float64) @ W.astype(np.float64).T) \
        * sh.view(np.float16).astype(np.float64)[None, :]
    np.testing.assert_allclose(lg, ref, rtol=1e-13)
    assert (am == ref.argmax(1)).all()
    assert (mv == ref.max(1)).all()


@pytest.mark.parametrize("mode", ["bf16", "int8"])
def test_planted_max_and_ties(mode):
    V, K = 257, 128
    W = synth.head_weights(3, 1, V, K)
    W[W == 127] = 126
    sh = np.full(V, np.float16(1.0)).view(np.uint16)
    x = np.abs(synth.bf16_bits_to_f32(synth.activations(3, 2, 3, K))) + np.float32(0.5)
    # row 0 of x: single planted max at v = 77; row 1: exact tie between 10 and 200 (lowest wins);
    # row 2: max at the last index
    Wp = W.copy()
    Wp[77] = 127
    Wp[10] = 127
    Wp[200] = 127
    Wp[V - 1] = 127
    xb = _bf16(x)
    xb[0] = _bf16(x[0])
    # row 0 and row 1 see the planted rows; to separate them give row 0 a sign pattern that
    # favours 77 only: negate x where row 77 would otherwise tie
    Wp[10, 0] = -127
    Wp[200, 0] = -127
    Wp[V - 1, 0] = -127
    if mode == "bf16":
        am, _, lg = oracle.head_bf16(Wp, sh, xb, want_logits=True)
    else:
        q, sx = oracle.quantize_act(xb, K)
        am, _, lg = oracle.head_i8(Wp, sh, q, sx, want_logits=True)
    assert am[0] == 77
    # rows 10, 200 and V-1 are identical, so their logits tie exactly in every row
    assert (lg[:, 10] == lg[:, 200]).all() and (lg[:, 10] == lg[:, V - 1]).all()
    for m in range(3):
        best = lg[m].max()
        assert am[m] == np.flatnonzero(lg[m] == best)[0]


def test_last_index_wins_alone():
    V, K = 64, 128
    W = np.zeros((V, K), np.int8)
    W[V - 1] = 1
    sh = np.full(V, np.float16(0.5)).view(np.uint16)
    x = _bf16(np.ones((1, K)))
    am, mv, _ = oracle.head_bf16(W, sh, x)
    assert am[0] == V - 1 and mv[0] == 64.0
    q, sx = oracle.quantize_act(x, K)
    am, mv, _ = oracle.head_i8(W, sh, q, sx)
    assert am[0] == V - 1
    assert mv[0] == np.float32(np.float32(128 * 127) * sx[0]) * np.float32(0.5)


def test_int8_head_exact_acc():
    V, K, M = 200, 384, 4
    W = synth.head_weights(4, 7, V, K)
    sh = synth.head_scales(4, 7, V)
    x = synth.activations(4, 8, M, K)
    q, sx = oracle.quantize_act(x, K)
    am, mv, lg = oracle.head_i8(W, sh, q, sx, want_logits=True)
    acc = q.astype(np.int64) @ W.astype(np.int64).T
    ref = (acc.astype(np.float32) * sx[:, None]) * sh.view(np.float16).astype(np.float32)[None, :]
    assert (lg == ref).all()
    assert (am == ref.argmax(1)).all()
