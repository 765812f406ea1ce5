"""GPU parity of the five-valued (FV5-style) weights and the block-scaled (FV5B-style) int8 head
against the CPU oracle: the packed planes bit for bit, the product in both activation modes (int8:
the fp64 block sum rounded once, bit for bit but for values within 1e-12 of an fp32 rounding
midpoint, where the device's split-K order may round the other way; bf16: the per-output bound
with the row's largest scale and relative L2), the head's logits and argmax (lowest index on exact
ties), several K slices per row, ragged N, M up to the limits, and invalid codes."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import PER_OUT, REL_L2, dev, host

pytestmark = pytest.mark.gpu


def _codes(seed, N, K):
    rng = np.random.default_rng(seed)
    return rng.choice(np.array([-2, -1, 0, 1, 2], np.int8), size=(N, K), p=[0.06, 0.13, 0.62, 0.13, 0.06])


def _scales(seed, N, K):
    rng = np.random.default_rng(seed + 1)
    lo = (0.01 + 0.04 * rng.random((N, K // 256))).astype(np.float32)
    return np.stack([lo, (lo * (2 + rng.random((N, K // 256)))).astype(np.float32)], axis=2)


def _matrix(seed, N, K):
    c = _codes(seed, N, K)
    s = _scales(seed, N, K)
    planes = torch.empty(N * 3 * K // 32, dtype=torch.int32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_fv5_pack(dev(c), N, K, planes, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_OK
    return tg.Fv5Matrix(planes, dev(s), N, K), c, s


def _near_f32_midpoint(v):
    """True where the fp64 value v is within 1e-12 (relative) of a midpoint between fp32 neighbours."""
    f = v.astype(np.float32).astype(np.float64)
    up = np.nextafter(v.astype(np.float32), np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(v.astype(np.float32), np.float32(-np.inf)).astype(np.float64)
    mids = np.stack([(f + up) / 2, (f + dn) / 2])
    return (np.abs(mids - v[None]) <= 1e-12 * np.abs(v[None])).any(0)


@pytest.mark.parametrize("N,K", [(37, 512), (300, 1024), (129, 4096), (64, 12288)])
def test_pack_matches_oracle(N, K):
    W, c, s = _matrix(5 + N, N, K)
    assert (host(W.planes).view(np.uint32).reshape(N, -1) == oracle.fv5_pack(c)).all()


@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("N,K", [(37, 512), (300, 1024), (1024, 4096), (200, 12288), (4096, 4096)])
def test_gemm_bf16(N, K, M):
    W, c, s = _matrix(11 + M, N, K)
    X = synth.activations(12, M, M, K)
    Y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
    tg.tern_fv5_gemm(W, M, tg.TERN_ACT_BF16, dev(X.view(np.int16)), None, Y)
    y = host(Y).reshape(M, N).astype(np.float64)
    ref = oracle.fv5_gemm_bf16(oracle.fv5_pack(c), s, K, X)
    err = y - ref
    absx = np.abs(synth.bf16_bits_to_f32(X).astype(np.float64)).sum(1)
    smax = s.reshape(N, -1).max(1).astype(np.float64)
    assert (np.abs(err) <= PER_OUT * absx[:, None] * smax[None, :]).all()
    assert np.linalg.norm(err) / np.linalg.norm(ref) <= REL_L2


@pytest.mark.parametrize("M", [1, 3, 8, 16])
@pytest.mark.parametrize("N,K", [(37, 512), (300, 1024), (1024, 4096), (200, 12288)])
def test_gemm_int8(N, K, M):
    W, c, s = _matrix(21 + M, N, K)
    X = synth.activations(22, M, M, K)
    q = torch.empty(M * K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    tg.tern_quantize_act(dev(X.view(np.int16)), M, K, q, sx)
    Y = torch.empty(M * N, dtype=torch.float32, device="cuda")
    tg.tern_fv5_gemm(W, M, tg.TERN_ACT_INT8, q, sx, Y)
    y = host(Y).reshape(M, N)
    qh, sxh = host(q).reshape(M, K), host(sx)
    ref = oracle.fv5_gemm_i8(oracle.fv5_pack(c), s, K, qh, sxh)
    # the exact value, for the midpoint test: exact block sums and scales in fp64 (Python floats)
    diff = y != ref
    if diff.any():
        lo = (np.abs(c) == 1) * np.sign(c)
        hi = (np.abs(c) == 2) * np.sign(c)
        for m, n in zip(*np.nonzero(diff)):
            tot = sum(float(s[n, b, 0]) * float((lo[n, 256 * b:256 * b + 256].astype(np.int64) * qh[m, 256 * b:256 * b + 256]).sum())
                      + float(s[n, b, 1]) * float((hi[n, 256 * b:256 * b + 256].astype(np.int64) * qh[m, 256 * b:256 * b + 256]).sum())
                      for b in range(K // 256))
            v = np.array([float(sxh[m]) * tot])
            assert _near_f32_midpoint(v)[0], (m, n, y[m, n], ref[m, n])
            assert abs(float(y[m, n]) - float(ref[m, n])) <= float(np.spacing(np.float32(ref[m, n])))


@pytest.mark.parametrize("mode", ["bf16", "int8"])
@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("V,K", [(1000, 1024), (517, 4096)])
def test_fv5b_head(V, K, M, mode):
    rng = np.random.default_rng(V + K + M)
    W = rng.integers(-127, 128, (V, K)).astype(np.int8)
    S = (rng.random((V, K // 256)) * 0.02 + 0.001).astype(np.float32)
    X = synth.activations(31, M, M, K)
    ws = torch.zeros(tg.i8_head_workspace_bytes(V, M), dtype=torch.uint8, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    mv = torch.empty(M, dtype=torch.float32, device="cuda")
    lg = torch.empty(M * V, dtype=torch.float32, device="cuda")
    if mode == "bf16":
        tg.fv5b_head_gemv_argmax(dev(W), dev(S), V, K, M, tg.TERN_ACT_BF16, dev(X.view(np.int16)), None, am, mv, lg, ws)
        am_ref, lg_ref = oracle.fv5b_head(W, S, x_bf16=X)
    else:
        q = torch.empty(M * K, dtype=torch.int8, device="cuda")
        sx = torch.empty(M, dtype=torch.float32, device="cuda")
        tg.tern_quantize_act(dev(X.view(np.int16)), M, K, q, sx)
        tg.fv5b_head_gemv_argmax(dev(W), dev(S), V, K, M, tg.TERN_ACT_INT8, q, sx, am, mv, lg, ws)
        am_ref, lg_ref = oracle.fv5b_head(W, S, q=host(q).reshape(M, K), sx=host(sx))
    torch.cuda.synchronize()
    assert (host(ws) == 0).all()
    a, m, l = host(am), host(mv), host(lg).reshape(M, V).astype(np.float64)
    absx = np.abs(synth.bf16_bits_to_f32(X).astype(np.float64)).sum(1)
    bound = PER_OUT * 127.0 * absx[:, None] * S.max(1).astype(np.float64)[None, :]
    err = l - lg_ref
    if mode == "int8":
        # one rounding of the fp64 block sum: equal, or one ulp at a rounding midpoint
        assert (np.abs(err) <= np.abs(np.spacing(lg_ref.astype(np.float32))).astype(np.float64)).all()
        assert (err != 0).mean() < 1e-3
    assert (np.abs(err) <= bound).all() and np.linalg.norm(err) / np.linalg.norm(lg_ref) <= REL_L2
    for r in range(M):
        if a[r] != am_ref[r]:
            assert lg_ref[r, am_ref[r]] - lg_ref[r, a[r]] <= bound[r, a[r]]
        assert l[r, a[r]] == m[r]


def test_fv5b_head_exact_tie_lowest_index():
    V, K, M = 2000, 1024, 2
    rng = np.random.default_rng(7)
    W = rng.integers(-127, 128, (V, K)).astype(np.int8)
    S = (rng.random((V, K // 256)) * 0.02 + 0.001).astype(np.float32)
    X = synth.activations(32, 1, M, K)
    q_ref, sx_ref = oracle.quantize_act(X, K)
    am0, _ = oracle.fv5b_head(W, S, q=q_ref, sx=sx_ref)
    w = int(am0[0])
    other = V - 1 if w < V // 2 else 0
    W[other], S[other] = W[w], S[w]
    ws = torch.zeros(tg.i8_head_workspace_bytes(V, M), dtype=torch.uint8, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    mv = torch.empty(M, dtype=torch.float32, device="cuda")
    tg.fv5b_head_gemv_argmax(dev(W), dev(S), V, K, M, tg.TERN_ACT_INT8, dev(q_ref), dev(sx_ref), am, mv, None, ws)
    torch.cuda.synchronize()
    assert host(am)[0] == min(w, other)


def test_fv5_invalid_codes_and_arguments():
    N, K = 16, 512
    c = _codes(40, N, K)
    c[3, 7] = 3
    planes = torch.empty(N * 3 * K // 32, dtype=torch.int32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_fv5_pack(dev(c), N, K, planes, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_EBADCODE
    with pytest.raises(tg.TernError):
        tg.tern_fv5_pack(dev(c[:, :256]), N, 256, planes, flag)          # K % 512 != 0
    W, _, _ = _matrix(41, N, K)
    x = torch.zeros(9 * K, dtype=torch.int16, device="cuda")
    y = torch.zeros(9 * N, dtype=torch.float32, device="cuda")
    with pytest.raises(tg.TernError):
        tg.tern_fv5_gemm(W, 9, tg.TERN_ACT_BF16, x, None, y)             # bf16 mode M <= 8


BATCH_SHAPES = [(37, 512), (300, 1024), (1024, 4096), (200, 12288), (129, 4096), (4096, 4096)]
_rs = np.random.default_rng(7)
BATCH_SETS = {
    # ragged shapes, K up to 12288: tiles split between two warps of a CTA
    "ragged": BATCH_SHAPES,
    # one 16-row tile over K = 12288: its 24 chunks cut among all eight warps of one CTA, each part
    # taking the partial sums of the one before
    "one_tile": [(16, 12288)],
    # many small items of mixed K
    "many_items": [(int(_rs.integers(1, 49)), 512 * int(_rs.integers(1, 9))) for _ in range(120)],
    # one long item, then 150 one-tile items: a range's share of the chunks holds more than the
    # 32 items a CTA stages, so ranges close at that limit
    "item_limit": [(200000, 512)] + [(1 + i % 16, 512) for i in range(150)],
    # K = 12288 items of a few tiles: in bf16 mode a second one would outgrow a CTA's staging
    # budget, so ranges close at each item
    "staging_budget": [(40 + 8 * i, 12288) for i in range(12)],
}


@pytest.mark.parametrize("mode", ["bf16", "int8"])
@pytest.mark.parametrize("shapes", sorted(BATCH_SETS))
def test_gemv_batch_matches_oracle(mode, shapes):
    """tern_fv5_gemv_batch: a list of shapes in one launch against the oracle: int8 mode bit for bit
    (the block sums are added in block order, as the oracle adds them, also where a tile's blocks
    are split among warps), bf16 mode within the per-output bound; twice on the same outputs, with
    no device-side wait giving up."""
    act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
    shape_list = BATCH_SETS[shapes]
    entries, refs, bounds = [], [], []
    for i, (N, K) in enumerate(shape_list):
        W, c, s = _matrix(41 + i, N, K)
        X = synth.activations(42 + i, 1, 1, K)
        y = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
        if mode == "bf16":
            entries.append((W, dev(X.view(np.int16)), None, y))
            refs.append(oracle.fv5_gemm_bf16(oracle.fv5_pack(c), s, K, X)[0])
            absx = np.abs(synth.bf16_bits_to_f32(X).astype(np.float64)).sum()
            bounds.append(PER_OUT * absx * s.reshape(N, -1).max(1).astype(np.float64))
        else:
            q = torch.empty(K, dtype=torch.int8, device="cuda")
            sx = torch.empty(1, dtype=torch.float32, device="cuda")
            tg.tern_quantize_act(dev(X.view(np.int16)), 1, K, q, sx)
            entries.append((W, q, sx, y))
            refs.append(oracle.fv5_gemm_i8(oracle.fv5_pack(c), s, K, host(q).reshape(1, K), host(sx))[0])
    for _ in range(2):
        for (_, _, _, y) in entries:
            y.fill_(float("nan"))
        tg.tern_fv5_gemv_batch(entries, act)
        torch.cuda.synchronize()
        assert tg.tern_device_status() == tg.TERN_OK
        for i, (W, _, _, y) in enumerate(entries):
            got = host(y)
            if mode == "int8":
                assert (got.view(np.uint32) == refs[i].astype(np.float32).view(np.uint32)).all(), shape_list[i]
            else:
                err = got.astype(np.float64) - refs[i]
                assert (np.abs(err) <= bounds[i]).all(), shape_list[i]
                assert np.linalg.norm(err) / np.linalg.norm(refs[i]) <= REL_L2


def test_gemv_batch_equals_single_entry_bf16():
    """bf16 mode: each item equals tern_fv5_gemm at M = 1 on K values one 512-weight slice long (a
    single K slice there too, so the fp64 order is the same)."""
    entries, singles = [], []
    for i, N in enumerate([64, 300, 1000]):
        W, c, s = _matrix(61 + i, N, 512)
        X = dev(synth.activations(62 + i, 1, 1, 512).view(np.int16))
        y = torch.empty(N, dtype=torch.float32, device="cuda")
        y1 = torch.empty(N, dtype=torch.float32, device="cuda")
        tg.tern_fv5_gemm(W, 1, tg.TERN_ACT_BF16, X, None, y1)
        entries.append((W, X, None, y))
        singles.append(y1)
    tg.tern_fv5_gemv_batch(entries, tg.TERN_ACT_BF16)
    torch.cuda.synchronize()
    for (_, _, _, y), y1 in zip(entries, singles):
        assert (host(y).view(np.uint32) == host(y1).view(np.uint32)).all()


def test_gemv_batch_argument_errors():
    W, c, s = _matrix(71, 64, 512)
    x = torch.zeros(512, dtype=torch.int16, device="cuda")
    y = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(tg.TernError):                 # int8 mode needs x_scale
        tg.tern_fv5_gemv_batch([(W, x, None, y)], tg.TERN_ACT_INT8)
    with pytest.raises(tg.TernError):                 # empty list
        tg.tern_fv5_gemv_batch([], tg.TERN_ACT_BF16)
