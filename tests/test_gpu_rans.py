"""GPU parity of the order-0 rANS transport: the device encoder byte for byte against the CPU
oracle (frequency table, row ends, payload), the device decoder bit for bit against the oracle's
packing of the same trits (several tensors in one launch, ragged and sparse shapes, degenerate
tensors, a full 8B layer), and invalid transports reported through the flag."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import dev, host

pytestmark = pytest.mark.gpu


def _encode_gpu(t_dev, N, K):
    freq = torch.empty(3, dtype=torch.int16, device="cuda")
    row_end = torch.empty(N, dtype=torch.int32, device="cuda")
    payload = torch.empty(tg.tern_rans_payload_bound(N, K), dtype=torch.uint8, device="cuda")
    ws = torch.empty(tg.tern_rans_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_rans_encode(t_dev, N, K, freq, row_end, payload, ws, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_OK
    n = int(host(row_end).view(np.uint32)[-1])
    return freq, row_end, payload[:n].clone()


SHAPES = [(37, 128, synth.P_DEFAULT), (300, 1024, synth.P_DEFAULT), (129, 4096, synth.P_SPARSE_FFN),
          (64, 12288, synth.P_DEFAULT), (5, 640, synth.P_DEFAULT)]


@pytest.mark.parametrize("N,K,p", SHAPES)
def test_encode_matches_oracle_bytes(N, K, p):
    t = synth.trits(31, N + K, N, K, p)
    freq, row_end, payload = _encode_gpu(dev(t), N, K)
    f_ref, re_ref, pl_ref = oracle.rans_encode(t)
    assert (host(freq).view(np.uint16) == f_ref).all()
    assert (host(row_end).view(np.uint32) == re_ref).all()
    assert (host(payload) == pl_ref).all()


def test_decode_list_matches_oracle_planes():
    entries, refs = [], []
    for i, (N, K, p) in enumerate(SHAPES):
        t = synth.trits(32, i, N, K, p)
        f, re, pl = oracle.rans_encode(t)
        planes = torch.full((N * K // 16,), -1, dtype=torch.int32, device="cuda")
        entries.append((dev(f.view(np.int16)), dev(re.view(np.int32)), dev(pl), N, K, planes))
        refs.append(oracle.pack(t))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_rans_decode(entries, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_OK
    for e, r in zip(entries, refs):
        assert (host(e[5]).view(np.uint32).reshape(r.shape) == r).all()


def test_degenerate_and_round_trip():
    for t in (np.zeros((3, 256), np.int8), np.ones((2, 128), np.int8), -np.ones((4, 384), np.int8),
              np.tile(np.array([1, -1, 0, 0], np.int8), (8, 64))):
        N, K = t.shape
        freq, row_end, payload = _encode_gpu(dev(t), N, K)
        planes = torch.empty(N * K // 16, dtype=torch.int32, device="cuda")
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        tg.tern_rans_decode([(freq, row_end, payload, N, K, planes)], flag)
        assert tg.tern_read_flag(flag) == tg.TERN_OK
        assert (host(planes).view(np.uint32).reshape(N, K // 16) == oracle.pack(t)).all()


def test_full_8b_layer_round_trip():
    """The seven tensors of one 8B layer: encoded on the device, decoded in one launch, bit-exact
    against tern_pack of the same trits; the stream is within 1% of the order-0 bound."""
    import synth.cuda as sc
    entries, packed, total_bits, total_H = [], [], 0, 0.0
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    for proj, N, K in synth.linear_shapes("8b"):
        t = torch.empty(N * K, dtype=torch.int8, device="cuda")
        sc.trits_into(t, synth.DEFAULT_SEED, synth.tensor_id(2, proj), K, synth.trit_probs("8b", 2, proj))
        ref = torch.empty(N * K // 16, dtype=torch.int32, device="cuda")
        tg.tern_pack(tg.TERN_SRC_INT8_TRITS, t, N, K, ref, flag)
        assert tg.tern_read_flag(flag) == tg.TERN_OK
        freq, row_end, payload = _encode_gpu(t, N, K)
        counts = torch.stack([(t == 0).sum(), (t == 1).sum(), (t == -1).sum()]).double().cpu().numpy()
        total_H += float(-(counts * np.log2(counts / counts.sum())).sum())
        total_bits += 8 * payload.numel()
        entries.append((freq, row_end, payload, N, K, torch.empty_like(ref)))
        packed.append(ref)
        del t
    tg.tern_rans_decode(entries, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_OK
    for e, ref in zip(entries, packed):
        assert torch.equal(e[5], ref)
    assert total_bits <= 1.01 * total_H


def test_invalid_transports_set_the_flag():
    N, K = 16, 1024
    t = synth.trits(33, 1, N, K)
    f, re, pl = oracle.rans_encode(t)
    planes = torch.empty(N * K // 16, dtype=torch.int32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad = pl.copy()
    bad[re[3] - 2] ^= 0x33
    for fr, r, p in ((f, re, bad), (f, np.where(np.arange(N) == 5, re + 1, re).astype(np.uint32), pl),
                     (np.array([4000, 100, 100], np.uint16), re, pl),
                     (f, np.where(np.arange(N) == N - 1, re[-1] + 4096, re).astype(np.uint32), pl)):
        tg.tern_rans_decode([(dev(fr.view(np.int16)), dev(r.view(np.int32)), dev(p), N, K, planes)], flag)
        assert tg.tern_read_flag(flag) == tg.TERN_EBADCODE
    # a valid call afterwards is clean again
    tg.tern_rans_decode([(dev(f.view(np.int16)), dev(re.view(np.int32)), dev(pl), N, K, planes)], flag)
    assert tg.tern_read_flag(flag) == tg.TERN_OK
    assert (host(planes).view(np.uint32).reshape(N, K // 16) == oracle.pack(t)).all()
