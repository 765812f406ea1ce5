"""The seeded input generator: published statistics of the weights, exact geometry totals from
the pages, and row-wise regeneration."""
import json
import math
import os

import numpy as np
import pytest

import synth


def test_geometry_totals(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "geometry.json")))
    for model in ("8b", "0.6b"):
        ref, geo = g[model], synth.GEOMETRY[model]
        for key, gk in (("layers", "layers"), ("hidden", "d"), ("ffn", "ffn"), ("q_heads", "q_heads"),
                        ("kv_heads", "kv_heads"), ("head_dim", "head_dim"), ("vocab", "vocab")):
            assert geo[gk] == ref[key], (model, key)
    # 8B: 36 layers x 7 linears = 6,945,767,424 ternary weights in 2,604,662,784 container bytes (3.0 bpw)
    L = synth.GEOMETRY["8b"]["layers"]
    trits8 = L * sum(N * K for _, N, K in synth.linear_shapes("8b"))
    assert trits8 == g["8b"]["ternary_trits"]
    assert g["8b"]["ternary_container_bytes"] * 8 == 3 * trits8
    # parameters = ternary + int8 vocabulary table(s) + fp32 norm gains
    d, V = synth.GEOMETRY["8b"]["d"], synth.GEOMETRY["8b"]["vocab"]
    assert 2 * V * d == g["8b"]["int8_vocab_params"]
    norms8 = L * (2 * d + 2 * 128) + d
    assert norms8 == g["8b"]["norm_gains"]
    assert trits8 + 2 * V * d + norms8 == g["8b"]["params"]
    L6, d6 = synth.GEOMETRY["0.6b"]["layers"], synth.GEOMETRY["0.6b"]["d"]
    trits6 = L6 * sum(N * K for _, N, K in synth.linear_shapes("0.6b"))
    assert V * d6 == g["0.6b"]["int8_vocab_params"]
    norms6 = L6 * (2 * d6 + 2 * 128) + d6
    assert trits6 + V * d6 + norms6 == g["0.6b"]["params"]


def test_thresholds_exact():
    t0, t1 = synth.thresholds(("0.6263", "0.1868"))
    assert t0 == 6263 * 2**64 // 10000
    assert t1 == (6263 + 1868) * 2**64 // 10000


def _binom_ok(count, n, p, sigmas=5.0):
    return abs(count - n * p) <= sigmas * math.sqrt(n * p * (1 - p))


def test_trit_distribution():
    n_rows, K = 256, 4096
    t = synth.trits(synth.DEFAULT_SEED, 7, n_rows, K)
    n = t.size
    assert _binom_ok((t == 0).sum(), n, 0.6263)
    assert _binom_ok((t == 1).sum(), n, 0.1868)
    assert _binom_ok((t == -1).sum(), n, 0.1869)
    ts = synth.trits(synth.DEFAULT_SEED, 8, n_rows, K, synth.P_SPARSE_FFN)
    assert _binom_ok((ts == 0).sum(), n, 0.71)
    assert _binom_ok((ts == 1).sum(), n, 0.145) and _binom_ok((ts == -1).sum(), n, 0.145)


def test_sparse_tensors_are_the_published_ones():
    sparse = [(l, p) for l in range(36) for p in synth.PROJ if synth.trit_probs("8b", l, p) != synth.P_DEFAULT]
    assert sparse == [(1, "gate"), (1, "down"), (2, "gate"), (2, "down"), (3, "gate"), (3, "down")]
    assert all(synth.trit_probs("0.6b", l, p) == synth.P_DEFAULT for l in range(28) for p in synth.PROJ)


def test_rows_regenerate_independently():
    full = synth.trits(1, 5, 40, 256)
    rows = np.array([0, 3, 39, 17])
    assert (synth.trits(1, 5, 40, 256, rows=rows) == full[rows]).all()
    hw = synth.head_weights(1, 252, 40, 128)
    assert (synth.head_weights(1, 252, 40, 128, rows=rows) == hw[rows]).all()


def test_scales_and_activations():
    s = synth.row_scales(1, 2, 10000).view(np.float16).astype(np.float64)
    assert s.min() >= 0.0099 and s.max() <= 0.0501
    x = synth.bf16_bits_to_f32(synth.activations(1, 2, 4, 4096)).astype(np.float64)
    assert abs(x.mean()) < 0.05 and abs(x.std() - 1.0) < 0.03
    hw = synth.head_weights(1, 3, 64, 1024)
    assert hw.min() == -127 and hw.max() == 127
    assert abs(hw.astype(np.float64).mean()) < 1.0


def test_splitmix_reference_values():
    # SplitMix64 seeded with 0: the first outputs of the published generator
    z = synth.uniform_u64(0, np.arange(3, dtype=np.uint64))
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
