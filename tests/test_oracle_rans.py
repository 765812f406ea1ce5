"""Pins of the oracle's order-0 rANS transport: hand-worked rows (tests/golden/rans_examples.txt),
the frequency quantisation rule on hand-worked counts, round trips on random and degenerate
tensors, the coded size against the order-0 entropy of each tensor, and invalid streams."""
import math
import os

import numpy as np
import pytest

import oracle
import synth


def _rows(path):
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            yield [part.split() for part in line.split("|")]


def test_hand_worked_rows(golden_dir):
    n = 0
    for freq, trits, stream in _rows(os.path.join(golden_dir, "rans_examples.txt")):
        f = np.array([int(v) for v in freq], np.uint16)
        t = np.array([[int(v) for v in trits]], np.int8)
        _, row_end, payload = oracle.rans_encode(t, f)
        assert payload.tobytes().hex() == "".join(stream).lower()
        assert row_end.tolist() == [len(stream)]
        back, ok = oracle.rans_decode(f, row_end, payload, 1, t.shape[1])
        assert ok and (back == t).all()
        n += 1
    assert n == 2


@pytest.mark.parametrize("counts,want", [
    ((6263, 1868, 1869), (2566, 765, 765)),      # floor(4096 c / 10000) = 2565, 765, 765; the +1 to t = 0
    ((100, 0, 0), (4094, 1, 1)),                 # absent symbols keep frequency 1
    ((1, 1, 1), (1366, 1365, 1365)),             # a three-way tie: the rest goes to t = 0
    ((0, 5, 5), (1, 2047, 2048)),               # 1 + 2048 + 2048 = 4097: one taken from the first of the tie
])
def test_frequency_rule(counts, want):
    t = np.concatenate([np.zeros(counts[0], np.int8), np.ones(counts[1], np.int8), -np.ones(counts[2], np.int8)])
    assert tuple(int(v) for v in oracle.rans_freqs(t)) == want


def _entropy_bits(t):
    n = t.size
    return -sum(c * math.log2(c / n) for c in (np.count_nonzero(t == 0), np.count_nonzero(t == 1),
                                                np.count_nonzero(t == -1)) if c)


@pytest.mark.parametrize("N,K,p", [(37, 128, synth.P_DEFAULT), (64, 4096, synth.P_DEFAULT),
                                   (16, 12288, synth.P_SPARSE_FFN), (5, 640, synth.P_DEFAULT)])
def test_round_trip_and_rate(N, K, p):
    t = synth.trits(21, N + K, N, K, p)
    f, row_end, payload = oracle.rans_encode(t)
    back, ok = oracle.rans_decode(f, row_end, payload, N, K)
    assert ok and (back == t).all()
    # the stream costs the tensor's order-0 entropy H (no coder of these frequencies can do better)
    # plus, per row, the 32-bit final state, of which up to 8 bits carry message (the state ends in
    # [2^23, 2^31)), and the loss of 12-bit frequencies (a few thousandths of a bit per trit)
    bits = 8 * payload.size
    H = _entropy_bits(t)
    assert H + 24 * N - 1 <= bits <= H * 1.002 + 32 * N


def test_degenerate_tensors():
    for t in (np.zeros((3, 256), np.int8), np.ones((2, 128), np.int8), -np.ones((1, 384), np.int8),
              np.tile(np.array([1, -1, 0, 0], np.int8), (4, 32))):
        f, row_end, payload = oracle.rans_encode(t)
        back, ok = oracle.rans_decode(f, row_end, payload, *t.shape)
        assert ok and (back == t).all()


def test_invalid_streams_are_reported():
    t = synth.trits(22, 1, 8, 1024)
    f, row_end, payload = oracle.rans_encode(t)
    bad = payload.copy()
    bad[row_end[2] - 1] ^= 0x5A                                    # corrupt the end of row 3
    assert not oracle.rans_decode(f, row_end, bad, 8, 1024)[1]
    short = row_end.copy()
    short[4] -= 1                                                  # a row claims one byte less
    assert not oracle.rans_decode(f, short, payload, 8, 1024)[1]
    assert not oracle.rans_decode(np.array([4096, 1, 1], np.uint16), row_end, payload, 8, 1024)[1]
