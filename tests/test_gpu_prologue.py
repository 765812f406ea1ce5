"""GPU parity of the activation prologues (RMSNorm, SwiGLU, fp32 cast, bf16 passthrough) and of
their fusion into the batched launch's operand preparation:
  * tern_act_prologue against the CPU oracle, bit for bit (a value within 1e-12 of a bf16 rounding
    midpoint may round either way: the oracle and the kernel sum the squares in different orders);
  * tern_gemm_batch_pro against the two-step device path (prologue, then tern_quantize_act in int8
    mode, then tern_gemm_batch), bit for bit, including the prepared activation and s_x it returns;
  * the fused product against the oracle: int8 mode bit-exact, bf16 mode within the tolerance."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import check_bf16, dev, host, make_matrix

pytestmark = pytest.mark.gpu

KINDS = {"bf16": tg.TERN_PRO_BF16, "cast": tg.TERN_PRO_CAST, "rmsnorm": tg.TERN_PRO_RMSNORM,
         "swiglu": tg.TERN_PRO_SWIGLU}


def _source(kind, M, K, seed, gain_scale=1.0):
    """(src numpy, gain bf16 bits or None, eps, oracle bf16 bits [M][K], exact fp64 values [M][K])."""
    rng = np.random.default_rng(seed)
    if kind == "bf16":
        x = synth.activations(seed, 1, M, K)
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        return x, None, 0.0, x.copy(), xf
    if kind == "swiglu":
        gu = (rng.standard_normal((M, 2 * K)) * 3).astype(np.float32)
        g, u = gu[:, :K].astype(np.float64), gu[:, K:].astype(np.float64)
        return gu, None, 0.0, oracle.swiglu(gu, K), g / (1 + np.exp(-g)) * u
    x = (rng.standard_normal((M, K)) * 2.0 ** rng.integers(-6, 7, (M, 1))).astype(np.float32)
    if kind == "cast":
        return x, None, 0.0, oracle.round_bf16(x.astype(np.float64)), x.astype(np.float64)
    gain = synth.f32_to_bf16_bits(((1 + 0.2 * rng.standard_normal(K)) * gain_scale).astype(np.float32))
    eps = 1e-6
    xd = x.astype(np.float64)
    r = 1.0 / np.sqrt((xd * xd).sum(1, keepdims=True) / K + eps)
    exact = xd * r * synth.bf16_bits_to_f32(gain).astype(np.float64)[None, :]
    return x, gain, eps, oracle.rmsnorm(x, gain, eps), exact


def _near_midpoint(v):
    """True where |v| lies within 1e-12 (relative) of a midpoint between neighbouring bf16 values."""
    a = np.abs(v)
    lo = synth.bf16_bits_to_f32(oracle.round_bf16(a)).astype(np.float64)
    step = np.where(a >= 2.0 ** -126, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-300))) - 7), 2.0 ** -133)
    mids = np.stack([lo - step / 2, lo + step / 2])
    return (np.abs(mids - a[None]) <= 1e-12 * a[None]).any(0)


def _assert_bits(got, want, exact):
    diff = got != want
    assert not (diff & ~_near_midpoint(exact)).any(), f"{int(diff.sum())} values differ"


@pytest.mark.parametrize("K", [128, 4096, 12288])
@pytest.mark.parametrize("kind", list(KINDS))
def test_standalone_prologue_matches_oracle(kind, K):
    M = 3
    src, gain, eps, want, exact = _source(kind, M, K, 7 + K)
    out = torch.empty(M * K, dtype=torch.int16, device="cuda")
    tg.tern_act_prologue(KINDS[kind], dev(src.view(np.int16) if kind == "bf16" else src),
                         None if gain is None else dev(gain.view(np.int16)), eps, M, K, out)
    _assert_bits(host(out).view(np.uint16).reshape(M, K), want, exact)


@pytest.mark.parametrize("gain_scale", [2.0 ** -125, 2.0 ** 126])
def test_rmsnorm_prologue_subnormal_and_overflow(gain_scale):
    """Gains of 2^-125 put the outputs into bf16's subnormal range; gains of 2^126 push the larger
    normalised values (|x| r > 2) past bf16's largest value, to infinity: the one-step fp64 -> bf16
    rounding on the device matches the oracle there too."""
    M, K = 2, 1024
    src, gain, eps, want, exact = _source("rmsnorm", M, K, 11, gain_scale)
    out = torch.empty(M * K, dtype=torch.int16, device="cuda")
    tg.tern_act_prologue(tg.TERN_PRO_RMSNORM, dev(src), dev(gain.view(np.int16)), eps, M, K, out)
    got = host(out).view(np.uint16).reshape(M, K)
    _assert_bits(got, want, exact)
    if gain_scale < 1:
        assert ((got & 0x7F80) == 0).any() and (got & 0x7FFF).any()          # subnormal values occur
    else:
        assert ((got & 0x7FFF) == 0x7F80).any()                             # infinities occur


def _batch(kind, mode, M, shapes, seed):
    """Items with prologues and the matching two-step inputs."""
    act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
    fused, plain, pros, refs = [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W, t, s = make_matrix(seed, 50 + i, N, K)
        src, gain, eps, want, exact = _source(kind, M, K, seed + 100 * i)
        srcd = dev(src.view(np.int16) if kind == "bf16" else src)
        gaind = None if gain is None else dev(gain.view(np.int16))
        # two-step path: the prologue alone, then (int8) the quantiser, then the plain batch
        xb = torch.empty(M * K, dtype=torch.int16, device="cuda")
        tg.tern_act_prologue(KINDS[kind], srcd, gaind, eps, M, K, xb)
        if act == tg.TERN_ACT_INT8:
            q = torch.empty(M * K, dtype=torch.int8, device="cuda")
            sx = torch.empty(M, dtype=torch.float32, device="cuda")
            tg.tern_quantize_act(xb, M, K, q, sx)
            plain.append((W, q, sx, torch.empty(M * N, dtype=torch.float32, device="cuda")))
            xo = torch.full((M * K,), 99, dtype=torch.int8, device="cuda")
            sxo = torch.full((M,), float("nan"), dtype=torch.float32, device="cuda")
        else:
            plain.append((W, xb, None, torch.empty(M * N, dtype=torch.float32, device="cuda")))
            xo = torch.full((M * K,), -1, dtype=torch.int16, device="cuda")
            sxo = None
        fused.append((W, xo, sxo, torch.full((M * N,), float("nan"), dtype=torch.float32, device="cuda")))
        pros.append((KINDS[kind], srcd, gaind, eps))
        refs.append((t, s, want, exact, srcd, gaind))
    return act, fused, plain, pros, refs


@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("mode", ["bf16", "int8"])
@pytest.mark.parametrize("kind", list(KINDS))
def test_fused_prologue_equals_two_step_and_oracle(kind, mode, M):
    """M = 1 and int8 M = 4 run the mma.sync lists, bf16 M = 4 and both modes at M = 8 the tcgen05
    lists (whose operand preparation computes the prologue itself)."""
    shapes = [(640, 4096), (300, 1024), (256, 12288)]
    act, fused, plain, pros, refs = _batch(kind, mode, M, shapes, 31)
    tg.GemvBatch(plain, act, M=M)()
    tg.GemvBatch(fused, act, M=M, prologues=pros)()
    torch.cuda.synchronize()
    assert tg.tern_device_status() == tg.TERN_OK
    for (W, xo, sxo, Y), (_, xp, sxp, Yp), (t, s, want, exact, _, _) in zip(fused, plain, refs):
        N, K = W.N, W.K
        assert (host(Y).view(np.uint32) == host(Yp).view(np.uint32)).all(), (kind, mode, N, K)
        assert (host(xo) == host(xp)).all()                     # the prepared activation it returns
        xb = host(xp).view(np.uint16).reshape(M, K) if mode == "bf16" else None
        if mode == "int8":
            assert (host(sxo).view(np.uint32) == host(sxp).view(np.uint32)).all()
            # the oracle's prologue row, quantised by the oracle: q and s_x equal, y bit-exact
            q_ref, sx_ref = oracle.quantize_act(want, K)
            assert (q_ref == host(xp).reshape(M, K)).all() and (sx_ref == host(sxp)).all()
            _, y_ref = oracle.gemm_i8(oracle.pack(t), s, K, q_ref, sx_ref)
            assert (host(Y).reshape(M, N) == y_ref).all()
        else:
            _assert_bits(xb, want, exact)
            check_bf16(host(Y).reshape(M, N), oracle.gemm_bf16(oracle.pack(t), s, K, xb), xb, s)


def test_fused_prologue_mixed_with_plain_items():
    """A batch mixing a plain item and prologue items (the layer-input patterns: RMSNorm before
    q|k|v, SwiGLU before down) gives the same bits as running each through the plain path."""
    M = 2
    act = tg.TERN_ACT_BF16
    a_act, a_f, a_p, a_pro, _ = _batch("rmsnorm", "bf16", M, [(512, 1024)], 41)
    b_act, b_f, b_p, b_pro, _ = _batch("swiglu", "bf16", M, [(384, 3072)], 42)
    W, t, s = make_matrix(43, 9, 200, 1024)
    X = dev(synth.activations(43, 1, M, 1024).view(np.int16))
    plain_item = (W, X, None, torch.empty(M * 200, dtype=torch.float32, device="cuda"))
    tg.GemvBatch(a_p + b_p + [plain_item], act, M=M)()
    ref = [host(e[3]).copy() for e in a_p + b_p + [plain_item]]
    mixed = [a_f[0], b_f[0], (W, X, None, torch.empty(M * 200, dtype=torch.float32, device="cuda"))]
    tg.GemvBatch(mixed, act, M=M, prologues=[a_pro[0], b_pro[0], None])()
    torch.cuda.synchronize()
    for e, r in zip(mixed, ref):
        assert (host(e[3]).view(np.uint32) == r.view(np.uint32)).all()


def test_prologue_argument_errors():
    M, K = 2, 256
    src = torch.zeros(M * K, dtype=torch.float32, device="cuda")
    out = torch.zeros(M * K, dtype=torch.int16, device="cuda")
    with pytest.raises(tg.TernError):
        tg.tern_act_prologue(tg.TERN_PRO_RMSNORM, src, None, 1e-6, M, K, out)       # RMSNorm needs a gain
    with pytest.raises(tg.TernError):
        tg.tern_act_prologue(tg.TERN_PRO_NONE, src, None, 0.0, M, K, out)           # no transform
    with pytest.raises(tg.TernError):
        tg.tern_act_prologue(tg.TERN_PRO_CAST, src, None, 0.0, M, 100, out)         # K % 128 != 0
    g = torch.ones(K, dtype=torch.int16, device="cuda")
    with pytest.raises(tg.TernError):
        tg.tern_act_prologue(tg.TERN_PRO_RMSNORM, src, g, -1.0, M, K, out)          # negative eps
    W = tg.TernMatrix.empty(64, K)
    y = torch.zeros(M * 64, dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(tg.TernError):                                               # int8 needs s_x out
        tg.tern_gemm_batch_pro([(W, None, None, y)], [(tg.TERN_PRO_CAST, src, None, 0.0)], M,
                               tg.TERN_ACT_INT8, ws)
    with pytest.raises(tg.TernError):                                               # unknown kind
        tg.tern_gemm_batch_pro([(W, None, None, y)], [(9, src, None, 0.0)], M, tg.TERN_ACT_BF16, ws)
