"""GPU parity of the loader kernels against the CPU oracle: packing (byte-exact), base-3
transport in both directions (bit-exact), error flags, occupancy, and the device twin of the
input generator."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", [(1, 128), (37, 384), (64, 4096), (3, 12288), (130, 1024)])
def test_pack_trits_bit_exact(N, K):
    t = synth.trits(31, N + K, N, K)
    planes = torch.empty(N * K // 16, dtype=torch.int32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_pack(tg.TERN_SRC_INT8_TRITS, dev(t), N, K, planes, flag)
    assert tg.tern_read_flag(flag) == 0
    assert (host(planes).view(np.uint32).reshape(N, K // 16) == oracle.pack(t)).all()


@pytest.mark.parametrize("N,K", [(1, 128), (37, 384), (20, 4096), (5, 12288), (9, 1024)])
def test_base3_both_directions_bit_exact(N, K):
    t = synth.trits(32, N * 3 + K, N, K)
    enc_ref = oracle.base3_encode(t)
    enc = torch.empty(N * oracle.base3_row_bytes(K), dtype=torch.uint8, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_base3_encode(dev(t), N, K, enc, flag)
    assert tg.tern_read_flag(flag) == 0
    assert (host(enc).reshape(enc_ref.shape) == enc_ref).all()
    planes = torch.empty(N * K // 16, dtype=torch.int32, device="cuda")
    tg.tern_pack(tg.TERN_SRC_BASE3, dev(enc_ref), N, K, planes, flag)
    assert tg.tern_read_flag(flag) == 0
    assert (host(planes).view(np.uint32).reshape(N, K // 16) == oracle.pack(t)).all()


def test_all_243_bytes():
    K = 1280
    row = np.full((1, 256), 121, np.uint8)
    row[0, :243] = np.arange(243)
    planes = torch.empty(K // 16, dtype=torch.int32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_pack(tg.TERN_SRC_BASE3, dev(row), 1, K, planes, flag)
    assert tg.tern_read_flag(flag) == 0
    ref = oracle.pack(oracle.base3_decode(row, 1, K))
    assert (host(planes).view(np.uint32).reshape(1, -1) == ref).all()


def test_invalid_inputs_set_flag():
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    planes = torch.empty(2 * 128 // 16, dtype=torch.int32, device="cuda")
    t = np.zeros((2, 128), np.int8)
    t[1, 50] = 3
    tg.tern_pack(tg.TERN_SRC_INT8_TRITS, dev(t), 2, 128, planes, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_EBADCODE
    row = np.full((2, 26), 121, np.uint8)
    row[0, 7] = 250
    tg.tern_pack(tg.TERN_SRC_BASE3, dev(row), 2, 128, planes, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_EBADCODE
    enc = torch.empty(2 * 26, dtype=torch.uint8, device="cuda")
    tg.tern_base3_encode(dev(t), 2, 128, enc, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_EBADCODE
    # the flag is cleared by the next call
    tg.tern_pack(tg.TERN_SRC_INT8_TRITS, dev(np.zeros((2, 128), np.int8)), 2, 128, planes, flag)
    assert tg.tern_read_flag(flag) == 0


def test_occupancy():
    N, K = 77, 4096
    t = synth.trits(33, 1, N, K)
    pl = dev(oracle.pack(t).view(np.int32))
    W = tg.TernMatrix(pl, torch.zeros(N, dtype=torch.float16, device="cuda"), N, K)
    counts = torch.empty(N * 3, dtype=torch.int64, device="cuda")
    tg.tern_occupancy(W, counts)
    assert (host(counts).reshape(N, 3) == oracle.occupancy(oracle.pack(t), K)).all()


def test_device_generator_matches_host():
    import synth.cuda as sc
    N, K = 64, 1024
    d = torch.empty(N * K, dtype=torch.int8, device="cuda")
    sc.trits_into(d, 5, 17, K, synth.P_SPARSE_FFN, row0=100)
    assert (host(d).reshape(N, K) == synth.trits(5, 17, 200, K, synth.P_SPARSE_FFN, rows=np.arange(100, 164))).all()
    h = torch.empty(N * K, dtype=torch.int8, device="cuda")
    sc.head_into(h, 5, 252, K)
    assert (host(h).reshape(N, K) == synth.head_weights(5, 252, N, K)).all()


def test_8b_transport_full_size():
    """All 6,945,767,424 trits of the 8B geometry: GPU encode -> GPU unpack must equal the GPU
    pack of the same trits on every word, and sampled rows of every tensor equal the oracle."""
    import synth.cuda as sc
    seed = synth.DEFAULT_SEED
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(0)
    total = 0
    for layer in range(synth.GEOMETRY["8b"]["layers"]):
        for proj, N, K in synth.linear_shapes("8b"):
            tid = synth.tensor_id(layer, proj)
            p = synth.trit_probs("8b", layer, proj)
            t = torch.empty(N * K, dtype=torch.int8, device="cuda")
            sc.trits_into(t, seed, tid, K, p)
            enc = torch.empty(N * oracle.base3_row_bytes(K), dtype=torch.uint8, device="cuda")
            tg.tern_base3_encode(t, N, K, enc, flag)
            a = torch.empty(N * K // 16, dtype=torch.int32, device="cuda")
            b = torch.empty_like(a)
            tg.tern_pack(tg.TERN_SRC_INT8_TRITS, t, N, K, a, flag)
            tg.tern_pack(tg.TERN_SRC_BASE3, enc, N, K, b, flag)
            assert torch.equal(a, b), (layer, proj)
            if layer in (0, 2, 35) or proj == "down":
                rows = np.sort(rng.choice(N, 3, replace=False))
                ref = oracle.pack(synth.trits(seed, tid, N, K, p, rows=rows))
                got = host(a).view(np.uint32).reshape(N, K // 16)[rows]
                assert (got == ref).all(), (layer, proj)
            total += N * K
            del t, enc, a, b
    assert tg.tern_read_flag(flag) == 0
    assert total == 6_945_767_424


def test_base3_batch_bit_exact_and_flag():
    """tern_pack_batch over ragged base-3 items equals the oracle per item (odd byte counts, so the
    transport buffers end inside a word); a bad byte in one item sets the flag."""
    shapes = [(1, 128), (37, 384), (20, 4096), (5, 12288), (9, 1024), (3, 640)]
    items, refs, flag = [], [], torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, (N, K) in enumerate(shapes):
        t = synth.trits(34, 50 + i, N, K)
        enc = dev(oracle.base3_encode(t).reshape(-1))
        planes = torch.full((N * K // 16,), -1, dtype=torch.int32, device="cuda")
        items.append((enc, N, K, planes))
        refs.append(oracle.pack(t))
    tg.tern_pack_batch(tg.TERN_SRC_BASE3, items, flag)
    assert tg.tern_read_flag(flag) == 0
    for (enc, N, K, planes), ref in zip(items, refs):
        assert (host(planes).view(np.uint32).reshape(N, K // 16) == ref).all(), (N, K)
    bad = items[3][0].clone()
    bad[7] = 243
    tg.tern_pack_batch(tg.TERN_SRC_BASE3, [items[0], (bad, 5, 12288, items[3][3])], flag)
    assert tg.tern_read_flag(flag) == tg.TERN_EBADCODE
    tg.tern_pack_batch(tg.TERN_SRC_BASE3, items[:2], flag)          # the next call clears the flag
    assert tg.tern_read_flag(flag) == 0


def test_int8_batch_bit_exact_and_flag():
    """tern_pack_batch over ragged int8-trit items (one persistent launch; units of 16 rows x 128
    words, so N % 16 != 0 and K / 32 % 128 != 0 leave partial units) equals the oracle per item;
    a byte outside {0, 1, 0xFF} in one item sets the flag, and the next call clears it."""
    shapes = [(1, 128), (37, 384), (20, 4096), (5, 12288), (17, 1024), (300, 640), (33, 8192)]
    items, refs, flag = [], [], torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, (N, K) in enumerate(shapes):
        t = synth.trits(35, 60 + i, N, K)
        planes = torch.full((N * K // 16,), -1, dtype=torch.int32, device="cuda")
        items.append((dev(t.reshape(-1)), N, K, planes))
        refs.append(oracle.pack(t))
    tg.tern_pack_batch(tg.TERN_SRC_INT8_TRITS, items, flag)
    assert tg.tern_read_flag(flag) == 0
    for (src, N, K, planes), ref in zip(items, refs):
        assert (host(planes).view(np.uint32).reshape(N, K // 16) == ref).all(), (N, K)
    bad = items[5][0].clone()
    bad[300 * 640 - 1] = 2                                          # the last byte of the last row
    tg.tern_pack_batch(tg.TERN_SRC_INT8_TRITS, [items[0], (bad, 300, 640, items[5][3])], flag)
    assert tg.tern_read_flag(flag) == tg.TERN_EBADCODE
    tg.tern_pack_batch(tg.TERN_SRC_INT8_TRITS, items[:2], flag)     # the next call clears the flag
    assert tg.tern_read_flag(flag) == 0
