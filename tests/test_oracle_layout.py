"""Pins of the oracle's packed layout (pack / unpack / occupancy) against hand-worked examples,
round trips and invariants. The layout is this library's own definition (include/tern.h)."""
import os

import numpy as np
import pytest

import oracle
import synth


def _layout_examples(golden_dir):
    rows = []
    for line in open(os.path.join(golden_dir, "layout_examples.txt")):
        line = line.split("#")[0].strip()
        if line:
            k, t, w, m, s = line.split()
            rows.append((int(k), int(t), int(w), int(m, 16), int(s, 16)))
    return rows


def test_single_trit_examples(golden_dir):
    ex = _layout_examples(golden_dir)
    assert len(ex) >= 10
    for k, t, w, mhex, shex in ex:
        trits = np.zeros((1, 128), np.int8)
        trits[0, k] = t
        pl = oracle.pack(trits)
        assert pl.shape == (1, 8)
        mask, sign = pl[0, :4], pl[0, 4:]
        expect_mask = np.zeros(4, np.uint32); expect_mask[w] = mhex
        expect_sign = np.zeros(4, np.uint32); expect_sign[w] = shex
        assert (mask == expect_mask).all(), (k, t, [hex(v) for v in mask])
        assert (sign == expect_sign).all(), (k, t, [hex(v) for v in sign])


def test_every_bit_used_once():
    # each of the 32 columns of a word owns a distinct mask bit and a distinct sign bit
    masks, signs = set(), set()
    for k in range(32):
        trits = np.zeros((1, 128), np.int8)
        trits[0, k] = -1
        pl = oracle.pack(trits)
        masks.add(int(pl[0, 0])); signs.add(int(pl[0, 4]))
    assert len(masks) == 32 and len(signs) == 32
    assert all(bin(v).count("1") == 1 for v in masks | signs)


@pytest.mark.parametrize("N,K", [(1, 128), (7, 256), (33, 384), (16, 1024)])
def test_roundtrip(N, K):
    t = synth.trits(11, N + K, N, K)
    pl = oracle.pack(t)
    assert pl.nbytes == N * K // 4                      # 2 bits per trit
    assert (oracle.unpack(pl, K) == t).all()


def test_canonical_sign():
    # sign bits only where the mask bit is set: sign word is a subset of the mask word rotated by 1
    t = synth.trits(5, 3, 64, 512)
    pl = oracle.pack(t).reshape(64, 2, 16)
    m, s = pl[:, 0, :].astype(np.uint64), pl[:, 1, :].astype(np.uint64)
    rot = ((m << np.uint64(1)) | (m >> np.uint64(31))) & np.uint64(0xFFFFFFFF)
    assert ((s & ~rot) == 0).all()
    # a row of zeros packs to zeros
    assert (oracle.pack(np.zeros((2, 128), np.int8)) == 0).all()


def test_invalid_trit_rejected():
    t = np.zeros((2, 128), np.int8)
    t[1, 77] = 2
    with pytest.raises(oracle.OracleError, match="index 205"):
        oracle.pack(t)


def test_occupancy_counts():
    t = synth.trits(9, 1, 40, 256)
    occ = oracle.occupancy(oracle.pack(t), 256)
    assert (occ[:, 0] == (t == 0).sum(1)).all()
    assert (occ[:, 1] == (t == 1).sum(1)).all()
    assert (occ[:, 2] == (t == -1).sum(1)).all()
