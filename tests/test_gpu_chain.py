"""GPU parity of the dependent decode chain (tern_chain_plan / tern_chain_run): two layers of the
0.6B geometry as eight linears whose activations come from earlier linears' outputs (RMSNorm
before q|k|v and gate|up, a cast of the q part before o, the SwiGLU of the interleaved gate|up
output before down), in one cooperative launch. Every item is checked bit for bit against the
two-step device path on the chain's own source outputs (tern_act_prologue, then tern_quantize_act
in int8 mode, then tern_gemm_batch), the fused SwiGLU output against the standalone SwiGLU
prologue, the last output against the oracle, and a second run against the first."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import check_bf16, dev, host

pytestmark = pytest.mark.gpu

D, Q, FF = 1024, 2048, 3072          # 0.6B: d, q width (attention output), FFN width


def _pack(t, s):
    N, K = t.shape
    W = tg.TernMatrix.empty(N, K)
    W.scale.copy_(dev(s.view(np.float16)))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_pack(tg.TERN_SRC_INT8_TRITS, dev(t), N, K, W.planes, flag)
    assert tg.tern_read_flag(flag) == tg.TERN_OK
    return W


def _interleave(a, b):
    """Rows of a and b interleaved in groups of eight: a 0..7, b 0..7, a 8..15, ..."""
    n = a.shape[0]
    out = np.empty((2 * n,) + a.shape[1:], a.dtype)
    out.reshape(n // 8, 2, 8, *a.shape[1:])[:, 0] = a.reshape(n // 8, 8, *a.shape[1:])
    out.reshape(n // 8, 2, 8, *a.shape[1:])[:, 1] = b.reshape(n // 8, 8, *b.shape[1:])
    return out


def _build(seed, layers=2):
    mats, items, ys, hs, sxs, specs = [], [], [], [], [], []
    h0 = dev(synth.residual(seed, 0, 1, D).reshape(-1))
    gains = [dev(synth.norm_gains(seed, i, D).view(np.int16)) for i in range(2 * layers)]
    for layer in range(layers):
        tid = 100 * layer
        qkv_t = synth.trits(seed, tid + 1, Q + 2 * D, D)
        o_t = synth.trits(seed, tid + 2, D, Q)
        g_t, u_t = synth.trits(seed, tid + 3, FF, D), synth.trits(seed, tid + 4, FF, D)
        d_t = synth.trits(seed, tid + 5, D, FF)
        sc = lambda k, n: synth.row_scales(seed, tid + k, n)
        gu_t = _interleave(g_t, u_t)
        gu_s = _interleave(sc(3, FF), sc(4, FF))
        for name, t, s in (("qkv", qkv_t, sc(1, Q + 2 * D)), ("o", o_t, sc(2, D)), ("gu", gu_t, gu_s),
                           ("down", d_t, sc(5, D))):
            mats.append((name, _pack(t, s), t, s))
    for i, (name, W, t, s) in enumerate(mats):
        layer = i // 4
        y = torch.full((W.N,), float("nan"), dtype=torch.float32, device="cuda")
        h = torch.full((W.N // 2,), -1, dtype=torch.int16, device="cuda") if name == "gu" else None
        sx = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
        ys.append(y); hs.append(h); sxs.append(sx)
        if name == "qkv":
            src_item = i - 1 if i else -1
            spec = dict(kind=tg.TERN_PRO_RMSNORM, src_item=src_item, src=None if i else h0, gain=gains[2 * layer],
                        eps=1e-6)
        elif name == "o":
            spec = dict(kind=tg.TERN_PRO_CAST, src_item=i - 1)
        elif name == "gu":
            spec = dict(kind=tg.TERN_PRO_RMSNORM, src_item=i - 1, gain=gains[2 * layer + 1], eps=1e-6, swiglu_out=True,
                        h=h)
        else:
            spec = dict(kind=tg.TERN_PRO_BF16, src_item=i - 1, src_h=True)
        specs.append(spec)
        items.append(tg.ChainItem(W, y=y, x_scale=sx, **spec))
    return mats, items, ys, hs, sxs, specs, h0


def _two_step(W, kind, src, gain, eps, K, act):
    xb = torch.empty(K, dtype=torch.int16, device="cuda")
    if kind == tg.TERN_PRO_BF16:
        xb.copy_(src[:K])
    else:
        tg.tern_act_prologue(kind, src, gain, eps, 1, K, xb)
    y = torch.empty(W.N, dtype=torch.float32, device="cuda")
    if act == tg.TERN_ACT_INT8:
        q = torch.empty(K, dtype=torch.int8, device="cuda")
        sx = torch.empty(1, dtype=torch.float32, device="cuda")
        tg.tern_quantize_act(xb, 1, K, q, sx)
        tg.GemvBatch([(W, q, sx, y)], act)()
        return y, xb, sx
    tg.GemvBatch([(W, xb, None, y)], act)()
    return y, xb, None


@pytest.mark.parametrize("mode", ["bf16", "int8"])
def test_chain_equals_two_step_path(mode):
    act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
    mats, items, ys, hs, sxs, specs, h0 = _build(51)
    chain = tg.Chain(items, act)
    chain()
    torch.cuda.synchronize()
    assert tg.tern_device_status() == tg.TERN_OK
    first = [host(y).copy() for y in ys]
    for i, ((name, W, t, s), spec) in enumerate(zip(mats, specs)):
        K = W.K
        if spec.get("src_h"):
            src = hs[spec["src_item"]]
        elif spec["src_item"] >= 0:
            src = ys[spec["src_item"]]
        else:
            src = spec["src"]
        y_ref, xb, sx_ref = _two_step(W, spec["kind"], src, spec.get("gain"), spec.get("eps", 0.0), K, act)
        torch.cuda.synchronize()
        assert (host(ys[i]).view(np.uint32) == host(y_ref).view(np.uint32)).all(), (mode, i, name)
        if act == tg.TERN_ACT_INT8:
            assert host(sxs[i]).view(np.uint32)[0] == host(sx_ref).view(np.uint32)[0], (i, name)
        if name == "gu":
            # the fused SwiGLU equals the standalone prologue on the de-interleaved gate|up output
            yg = host(ys[i]).reshape(-1, 2, 8)
            gu = np.concatenate([yg[:, 0].reshape(-1), yg[:, 1].reshape(-1)])
            want = torch.empty(FF, dtype=torch.int16, device="cuda")
            tg.tern_act_prologue(tg.TERN_PRO_SWIGLU, dev(gu), None, 0.0, 1, FF, want)
            assert (host(hs[i]) == host(want)).all()
        if i == len(mats) - 1 and mode == "bf16":
            x = host(xb).view(np.uint16)[None, :]
            check_bf16(host(ys[i])[None, :], oracle.gemm_bf16(oracle.pack(t), s, K, x), x, s)
    # a second run of the same workspace gives the same bits (counters and scratch left clean)
    chain()
    torch.cuda.synchronize()
    assert tg.tern_device_status() == tg.TERN_OK
    for y, a in zip(ys, first):
        assert (host(y).view(np.uint32) == a.view(np.uint32)).all()


def test_chain_argument_errors():
    W = tg.TernMatrix.empty(64, 128)
    y = torch.zeros(64, dtype=torch.float32, device="cuda")
    x = torch.zeros(128, dtype=torch.int16, device="cuda")
    with pytest.raises(tg.TernError):                   # a source item must come earlier
        tg.Chain([tg.ChainItem(W, tg.TERN_PRO_CAST, y, src_item=0)], tg.TERN_ACT_BF16)
    with pytest.raises(tg.TernError):                   # src_h needs a SwiGLU item
        tg.Chain([tg.ChainItem(W, tg.TERN_PRO_BF16, y, src=x),
                  tg.ChainItem(W, tg.TERN_PRO_BF16, y, src_item=0, src_h=True)], tg.TERN_ACT_BF16)
    with pytest.raises(tg.TernError):                   # RMSNorm needs a gain
        tg.Chain([tg.ChainItem(W, tg.TERN_PRO_RMSNORM, y, src=y)], tg.TERN_ACT_BF16)


def test_chain_runs_read_only_their_own_outputs():
    """Each run of one workspace reads only the outputs of that run: two entry vectors A and B run
    as A, B, A, B give the first two runs' bits again (a linear that read a stale source would
    mix the runs)."""
    mats, items, ys, hs, sxs, specs, h0 = _build(52)
    chain = tg.Chain(items, tg.TERN_ACT_BF16)
    a = h0.clone()
    b = dev(synth.residual(53, 0, 1, D).reshape(-1))
    runs = []
    for src in (a, b, a, b):
        h0.copy_(src)
        chain()
        torch.cuda.synchronize()
        assert tg.tern_device_status() == tg.TERN_OK
        runs.append([host(y).view(np.uint32).copy() for y in ys] + [host(hs[2]).copy()])
    for i in range(len(runs[0])):
        assert (runs[0][i] == runs[2][i]).all() and (runs[1][i] == runs[3][i]).all(), i
        assert not (runs[0][i] == runs[1][i]).all(), i
