"""GPU parity of the batched M = 1 GEMV (one prep launch + one persistent streaming launch for a
whole list of matrices) against the CPU oracle, and its agreement with the single-GEMV path."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import check_bf16, dev, host, make_matrix

pytestmark = pytest.mark.gpu

SHAPES = [(37, 384), (200, 640), (1, 128), (3072, 1024), (2048, 1024), (1024, 3072), (6144, 4096),
          (4096, 4096), (129, 12288), (4096, 12288), (24576, 4096)]


def _build(seed, shapes, act):
    items, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W, t, s = make_matrix(seed, 100 + i, N, K, host_trits=N * K <= 4096 * 4096)
        x = synth.activations(seed, 200 + i, 1, K)
        xd = dev(x.view(np.int16))
        if act == tg.TERN_ACT_INT8:
            q = torch.empty(K, dtype=torch.int8, device="cuda")
            sx = torch.empty(1, dtype=torch.float32, device="cuda")
            tg.tern_quantize_act(xd, 1, K, q, sx)
            xin, sxin = q, sx
        else:
            xin, sxin = xd, None
        y = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
        items.append((W, xin, sxin, y))
        refs.append((t, s, x, i))
    return items, refs


def _rows(N, seed):
    if N <= 4096:
        return np.arange(N)
    r = np.sort(np.random.default_rng(seed).choice(N, 64, replace=False))
    r[0], r[-1] = 0, N - 1
    return r


@pytest.mark.parametrize("mode", ["bf16", "int8"])
def test_batch_matches_oracle(mode):
    act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
    items, refs = _build(71, SHAPES, act)
    batch = tg.GemvBatch(items, act)
    batch()
    torch.cuda.synchronize()
    assert tg.tern_device_status() == tg.TERN_OK
    for (W, xin, sxin, y), (t, s, x, i) in zip(items, refs):
        N, K = W.N, W.K
        rows = _rows(N, i)
        tr = t[rows] if t is not None else synth.trits(71, 100 + i, N, K, rows=rows)
        yy = host(y)[rows]
        if mode == "bf16":
            check_bf16(yy[None, :], oracle.gemm_bf16(oracle.pack(tr), s[rows], K, x), x, s[rows])
        else:
            q, sx = host(xin), host(sxin)
            _, y_ref = oracle.gemm_i8(oracle.pack(tr), s[rows], K, q[None, :], sx)
            assert (yy == y_ref[0]).all(), (N, K)


def test_batch_int8_equals_single_and_is_deterministic():
    items, _ = _build(72, [(6144, 4096), (4096, 12288), (1000, 1024)], tg.TERN_ACT_INT8)
    batch = tg.GemvBatch(items, tg.TERN_ACT_INT8)
    batch()
    first = [host(y).copy() for (_, _, _, y) in items]
    batch(flags=tg.TERN_FLAG_PDL)
    for (W, q, sx, y), a in zip(items, first):
        b = host(y)
        assert (a.view(np.uint32) == b.view(np.uint32)).all()
        y1 = torch.empty_like(y)
        tg.tern_gemv(W, tg.TERN_ACT_INT8, q, sx, y1)
        assert (host(y1).view(np.uint32) == b.view(np.uint32)).all()


def test_batch_full_8b_layer_sampled():
    """One 8B layer as its four fused launches (q|k|v, o, gate|up, down) in one batch, bf16."""
    import bench
    lins = [bench.build_linear("8b", 2, projs) for _, projs in synth.FUSED_GROUPS]
    items, xs = [], []
    for i, lin in enumerate(lins):
        x = synth.activations(73, i, 1, lin.K)
        xs.append(x)
        items.append((lin.W, dev(x.view(np.int16)), None, torch.empty(lin.N, dtype=torch.float32, device="cuda")))
    tg.GemvBatch(items, tg.TERN_ACT_BF16)()
    shapes = {p: (N, K) for p, N, K in synth.linear_shapes("8b")}
    for (grp, projs), lin, (W, xd, _, y), x in zip(synth.FUSED_GROUPS, lins, items, xs):
        r0 = 0
        for pj in projs:
            n = shapes[pj][0]
            rows = np.sort(np.random.default_rng(n).choice(n, 24, replace=False))
            tid = synth.tensor_id(2, pj)
            p = synth.trit_probs("8b", 2, pj)
            t = synth.trits(synth.DEFAULT_SEED, tid, n, lin.K, p, rows=rows)
            s = synth.row_scales(synth.DEFAULT_SEED, tid, n)[rows]
            ref = oracle.gemm_bf16(oracle.pack(t), s, lin.K, x)
            check_bf16(host(y)[r0 + rows][None, :], ref, x, s)
            r0 += n


def test_batch_argument_errors():
    W = tg.TernMatrix.empty(64, 128)
    x = torch.zeros(128, dtype=torch.int16, device="cuda")
    y = torch.zeros(64, dtype=torch.float32, device="cuda")
    assert tg.tern_gemv_batch_workspace_bytes([(W, x, None, y)], tg.TERN_ACT_BF16) > 0
    big = tg.TernMatrix.empty(16, 12288 + 128)
    assert tg.tern_gemv_batch_workspace_bytes([(big, x, None, y)], tg.TERN_ACT_BF16) == 0
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(tg.TernError):
        tg.tern_gemv_batch([(W, x, None, y)], tg.TERN_ACT_BF16, ws)        # workspace too small
    with pytest.raises(tg.TernError):
        tg.tern_gemv_batch([(W, x, None, y)], tg.TERN_ACT_INT8, ws)        # int8 needs s_x


def _build_m(seed, shapes, M, act):
    items, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W, t, s = make_matrix(seed, 300 + i, N, K, host_trits=N * K <= 4096 * 4096)
        X = synth.activations(seed, 400 + i, M, K)
        Xd = dev(X.view(np.int16))
        if act == tg.TERN_ACT_INT8:
            q = torch.empty(M * K, dtype=torch.int8, device="cuda")
            sx = torch.empty(M, dtype=torch.float32, device="cuda")
            tg.tern_quantize_act(Xd, M, K, q, sx)
            xin, sxin = q, sx
        else:
            xin, sxin = Xd, None
        Y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
        items.append((W, xin, sxin, Y))
        refs.append((t, s, X, i))
    return items, refs


SHAPES_M = [(37, 384), (200, 640), (3072, 1024), (1024, 3072), (4096, 12288), (24576, 4096)]


@pytest.mark.parametrize("M", [2, 3, 4, 5, 6, 7, 8, 9, 16])
@pytest.mark.parametrize("mode", ["bf16", "int8"])
def test_gemm_batch_small_m_matches_oracle(mode, M):
    """Every token row of every item: int8 bit-exact, bf16 within the tolerance (sampled rows of
    the large matrices); rows of Y beyond N and tokens beyond M are never written."""
    act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
    items, refs = _build_m(81 + M, SHAPES_M, M, act)
    tg.GemvBatch(items, act, M=M)()
    torch.cuda.synchronize()
    assert tg.tern_device_status() == tg.TERN_OK
    for (W, xin, sxin, Y), (t, s, X, i) in zip(items, refs):
        N, K = W.N, W.K
        rows = _rows(N, i)
        tr = t[rows] if t is not None else synth.trits(81 + M, 300 + i, N, K, rows=rows)
        yy = host(Y).reshape(M, N)[:, rows]
        if mode == "bf16":
            check_bf16(yy, oracle.gemm_bf16(oracle.pack(tr), s[rows], K, X), X, s[rows])
        else:
            q, sx = host(xin).reshape(M, K), host(sxin)
            _, y_ref = oracle.gemm_i8(oracle.pack(tr), s[rows], K, q, sx)
            assert (yy == y_ref).all(), (N, K, M)


@pytest.mark.parametrize("mode,M", [("bf16", M) for M in (2, 3, 4, 5, 6, 7, 8)] + [("int8", M) for M in (2, 5, 7, 8, 9, 12, 16)])
def test_gemm_batch_tensor_core_equals_mma_sync(mode, M):
    """The tcgen05 kernels (TERN_FLAG_TCGEN05) and the mma.sync kernels (the default at these sizes)
    give the same bits for every output: every sum is an exact integer and the final roundings are
    the same. Ragged N (37, 200, 1000 rows: partial row blocks and boxes), K = 128 and 640 (partial
    512-trit parts), and lists whose row blocks are split between CTAs. The tcgen05 result is the
    reference; the mma.sync kernels run four times against it (split-block scratch left clean
    between runs), the last two with PDL, then tcgen05 once more."""
    act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
    shapes = SHAPES_M + [(1000, 128), (6144, 4096)]
    items, _ = _build_m(95 + M, shapes, M, act)
    batch = tg.GemvBatch(items, act, M=M)
    batch(flags=tg.TERN_FLAG_TCGEN05)
    torch.cuda.synchronize()
    assert tg.tern_device_status() == tg.TERN_OK
    want = [host(Y).copy() for (_, _, _, Y) in items]
    for flags in (0, 0, tg.TERN_FLAG_PDL, tg.TERN_FLAG_PDL, tg.TERN_FLAG_TCGEN05 | tg.TERN_FLAG_PDL):
        for (_, _, _, Y) in items:
            Y.fill_(float("nan"))
        batch(flags=flags)
        torch.cuda.synchronize()
        assert tg.tern_device_status() == tg.TERN_OK
        for (W, _, _, Y), a in zip(items, want):
            assert (host(Y).view(np.uint32) == a.view(np.uint32)).all(), (mode, M, W.N, W.K, flags)


def _on_grid(X: np.ndarray) -> np.ndarray:
    """bf16 activations with every nonzero |x| >= 2^-12 (tiny values moved to +-2^-12): far above the
    fixed-point grid 2^(E-30) of the four-limb encoding for these rows (absmax < 2^5), so the device
    sums are the exact sums and the result equals the oracle's single rounding bit for bit."""
    X = X.copy()
    mag = X & 0x7FFF
    tiny = (mag != 0) & (mag < 0x3980)
    X[tiny] = (X[tiny] & 0x8000) | 0x3980
    return X


@pytest.mark.parametrize("flags", [0, 2])
@pytest.mark.parametrize("M", [5, 6, 8, 16])
def test_gemm_batch_bf16_tensor_core_exact(M, flags):
    """bf16 lists of 5..16 rows, on the default kernels (mma.sync up to 8 rows, tcgen05 above) and on
    tcgen05 (flags = TERN_FLAG_TCGEN05). On activations with no element below the limb grid every
    output equals the oracle's bit for bit (exact integer sums, the same final rounding), twice in a
    row, on ragged and split shapes."""
    shapes = [(200, 640), (1000, 128), (4096, 12288), (24576, 4096), (6144, 4096)]
    items, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W, t, s = make_matrix(131 + M, 300 + i, N, K, host_trits=False)
        X = _on_grid(synth.activations(131 + M, 400 + i, M, K))
        Y = torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")
        items.append((W, dev(X.view(np.int16)), None, Y))
        refs.append((s, X, i))
    batch = tg.GemvBatch(items, tg.TERN_ACT_BF16, M=M)
    assert flags in (0, tg.TERN_FLAG_TCGEN05)
    for _ in range(2):
        for (_, _, _, Y) in items:
            Y.fill_(float("nan"))
        batch(flags=flags)
        torch.cuda.synchronize()
        assert tg.tern_device_status() == tg.TERN_OK
        for (W, _, _, Y), (s, X, i) in zip(items, refs):
            N, K = W.N, W.K
            rows = _rows(N, i)
            tr = synth.trits(131 + M, 300 + i, N, K, rows=rows)
            want = oracle.gemm_bf16(oracle.pack(tr), s[rows], K, X)
            got = host(Y).reshape(M, N)[:, rows]
            assert (got.astype(np.float32).view(np.uint32) == np.asarray(want, np.float32).view(np.uint32)).all(), (M, N, K)


def test_gemm_batch_int8_equals_small_m_entry():
    """The batched small-M path and tern_gemm_small_m agree bit for bit in int8 mode."""
    M = 7
    items, _ = _build_m(90, [(6144, 4096), (4096, 12288)], M, tg.TERN_ACT_INT8)
    tg.GemvBatch(items, tg.TERN_ACT_INT8, M=M)()
    for W, q, sx, Y in items:
        Y1 = torch.empty_like(Y)
        tg.tern_gemm_small_m(W, M, tg.TERN_ACT_INT8, q, sx, Y1)
        assert (host(Y1).view(np.uint32) == host(Y).view(np.uint32)).all()
