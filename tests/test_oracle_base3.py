"""Pins of the oracle's base-3 transport codec: hand-worked bytes, exhaustive decode of all
byte values, invalid bytes, padding and round trips."""
import os

import numpy as np
import pytest

import oracle
import synth


def test_hand_examples(golden_dir):
    n = 0
    for line in open(os.path.join(golden_dir, "base3_examples.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        b, *ts = (int(v) for v in line.split())
        trits = np.array([ts + [0] * 123], np.int8)         # K = 128, rest zero
        enc = oracle.base3_encode(trits)
        assert enc.shape == (1, 26)
        assert enc[0, 0] == b
        assert (enc[0, 1:25] == 121).all()                  # all-zero groups encode as 121
        dec = oracle.base3_decode(enc, 1, 128)
        assert (dec == trits).all()
        n += 1
    assert n >= 10


def test_all_valid_bytes_bijective():
    data = np.arange(243, dtype=np.uint8).reshape(1, 243)
    # a row of K = 1215 trits (= 243 * 5) is not a multiple of 128; decode the codec directly on
    # K = 1280 rows padded with zero groups instead
    K = 1280
    row = np.full((1, 256), 121, np.uint8)
    row[0, :243] = data
    dec = oracle.base3_decode(row, 1, K)
    digits = dec[0, :1215].reshape(243, 5).astype(np.int64) + 1
    assert digits.min() >= 0 and digits.max() <= 2
    value = digits @ np.array([1, 3, 9, 27, 81])
    assert (value == np.arange(243)).all()
    assert (oracle.base3_encode(dec)[0, :243] == data[0]).all()


@pytest.mark.parametrize("bad", [243, 250, 255])
def test_invalid_byte(bad):
    row = np.full((2, 26), 121, np.uint8)
    row[1, 3] = bad
    with pytest.raises(oracle.OracleError, match="index 29"):
        oracle.base3_decode(row, 2, 128)


def test_padding_and_roundtrip():
    K = 384                                              # 77 bytes per row, one padding trit
    t = synth.trits(21, 4, 50, K)
    enc = oracle.base3_encode(t)
    assert enc.shape == (50, (K + 4) // 5)
    last = enc[:, -1].astype(np.int64)
    assert ((last // 81) % 3 == 1).all()                 # padding digit is t = 0
    assert (oracle.base3_decode(enc, 50, K) == t).all()
    # padding digits are ignored on decode
    enc2 = enc.copy()
    enc2[:, -1] = (enc2[:, -1].astype(np.int64) % 81 + 2 * 81).astype(np.uint8)
    assert (oracle.base3_decode(enc2, 50, K) == t).all()


def test_transport_size_8b():
    total = 0
    for _, N, K in synth.linear_shapes("8b"):
        total += N * oracle.base3_row_bytes(K)
    assert total * 36 == 1_390_215_168
