"""GPU check of i8_head_gemv_argmax_noalloc, the head entry point for callers that cannot allocate
device memory (code that runs where cudaMalloc is unavailable or forbidden, e.g. inside another
library's fixed memory budget): its scratch is one library-internal device array instead of a
caller workspace.

Two calls in a row through the C ABI, each compared with the CPU oracle and with
i8_head_gemv_argmax on the same inputs (int8 mode bit-exact; bf16 mode within the packed path's
tolerance: relative L2 <= 1e-5 and |err| <= 1e-4 * sum|x| * 127 * scale per logit, argmax equal or
a near tie). Device free memory is the same before and after the calls, and an invalid call
enqueues nothing. The file name sorts last so that pytest collects it after every other test."""

import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import PER_OUT, REL_L2, dev, host

pytestmark = pytest.mark.gpu


def _inputs(seed, V, K, M, mode):
    W_host = synth.head_weights(seed, V + K, V, K)
    sh_bits = synth.head_scales(seed, V + K, V)
    X = synth.activations(seed, M, M, K)
    W, sh, xd = dev(W_host), dev(sh_bits.view(np.float16)), dev(X.view(np.int16))
    if mode == "bf16":
        return W, W_host, sh, sh_bits, X, tg.TERN_ACT_BF16, xd, None
    q = torch.empty(M * K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    tg.tern_quantize_act(xd, M, K, q, sx)
    return W, W_host, sh, sh_bits, X, tg.TERN_ACT_INT8, q, sx


def _outs(M, V):
    return (torch.full((M,), -1, dtype=torch.int32, device="cuda"),
            torch.full((M,), float("nan"), dtype=torch.float32, device="cuda"),
            torch.full((M * V,), float("nan"), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("mode", ["int8", "bf16"])
@pytest.mark.parametrize("V,K,M", [(4099, 1024, 1), (1000, 4096, 7), (517, 128, 16)])
def test_noalloc_matches_oracle_and_workspace_entry_twice(V, K, M, mode):
    W, W_host, sh, sh_bits, X, act, xin, sx = _inputs(91, V, K, M, mode)
    ws = torch.zeros(tg.i8_head_workspace_bytes(V, M), dtype=torch.uint8, device="cuda")
    am0, mv0, lg0 = _outs(M, V)
    tg.i8_head_gemv_argmax(W, sh, V, K, M, act, xin, sx, am0, mv0, lg0, ws)
    ref_am, ref_mv, ref_lg = host(am0), host(mv0), host(lg0).reshape(M, V).astype(np.float64)
    absx = np.abs(synth.bf16_bits_to_f32(X).astype(np.float64)).sum(1)
    bound = PER_OUT * absx[:, None] * 127.0 * sh_bits.view(np.float16).astype(np.float64)[None, :]
    if mode == "int8":
        o_am, o_mv, o_lg = oracle.head_i8(W_host, sh_bits, host(xin).reshape(M, K), host(sx), want_logits=True)
    else:
        o_am, o_mv, o_lg = oracle.head_bf16(W_host, sh_bits, X, want_logits=True)
    outs = [_outs(M, V) for _ in range(2)]
    torch.cuda.synchronize()
    for call in range(2):
        am, mv, lg = outs[call]
        tg.i8_head_gemv_argmax_noalloc(W, sh, V, K, M, act, xin, sx, am, mv, lg)
        torch.cuda.synchronize()
        assert tg.tern_device_status() == tg.TERN_OK
        a, m, l = host(am), host(mv), host(lg).reshape(M, V)
        if mode == "int8":
            # the oracle's int64 sums and the workspace entry, bit for bit
            assert (a == o_am).all() and (m == o_mv).all() and (l == o_lg).all(), call
            assert (a == ref_am).all(), call
            assert (m.view(np.uint32) == ref_mv.view(np.uint32)).all(), call
            assert (l.view(np.uint32) == host(lg0).reshape(M, V).view(np.uint32)).all(), call
        else:
            for ref in (o_lg, ref_lg):
                err = l.astype(np.float64) - ref
                assert np.linalg.norm(err) / np.linalg.norm(ref) <= REL_L2, call
                assert (np.abs(err) <= bound).all(), call
            for r in range(M):
                if a[r] != o_am[r]:             # only a near tie may pick another index
                    assert o_mv[r] - o_lg[r, a[r]] <= bound[r, a[r]], (call, r)
                assert l[r, a[r]] == m[r], (call, r)


def test_noalloc_allocates_no_device_memory():
    """After a first call (which looks up the scratch address on this device), further calls leave
    the device's free memory unchanged: the entry point allocates nothing."""
    V, K, M = 2048, 1024, 4
    W, _, sh, _, _, act, xin, sx = _inputs(92, V, K, M, "bf16")
    am, mv, lg = _outs(M, V)
    tg.i8_head_gemv_argmax_noalloc(W, sh, V, K, M, act, xin, sx, am, mv, lg)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        tg.i8_head_gemv_argmax_noalloc(W, sh, V, K, M, act, xin, sx, am, mv, lg)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert tg.tern_device_status() == tg.TERN_OK


def test_noalloc_invalid_call_enqueues_nothing():
    """A call with a null weight pointer returns TERN_EINVAL and writes nothing; the next valid call
    still matches the workspace entry point."""
    V, K, M = 1000, 1024, 2
    W, _, sh, _, _, act, xin, sx = _inputs(93, V, K, M, "int8")
    am, mv, lg = _outs(M, V)
    st = tg.lib().i8_head_gemv_argmax_noalloc(None, tg._ptr(sh), V, K, M, act, tg._ptr(xin), tg._ptr(sx),
                                              tg._ptr(am), tg._ptr(mv), tg._ptr(lg), tg._stream(None))
    assert st == tg.TERN_EINVAL
    torch.cuda.synchronize()
    assert (host(am) == -1).all() and np.isnan(host(mv)).all() and np.isnan(host(lg)).all()
    tg.i8_head_gemv_argmax_noalloc(W, sh, V, K, M, act, xin, sx, am, mv, lg)
    ws = torch.zeros(tg.i8_head_workspace_bytes(V, M), dtype=torch.uint8, device="cuda")
    am1, mv1, lg1 = _outs(M, V)
    tg.i8_head_gemv_argmax(W, sh, V, K, M, act, xin, sx, am1, mv1, lg1, ws)
    torch.cuda.synchronize()
    assert (host(am) == host(am1)).all() and (host(lg).view(np.uint32) == host(lg1).view(np.uint32)).all()


def test_noalloc_rejects_m_above_scratch():
    V, K = 64, 128
    W = torch.zeros(V * K, dtype=torch.int8, device="cuda")
    sh = torch.ones(V, dtype=torch.float16, device="cuda")
    M = tg.TERN_HEAD_NOALLOC_MAX_M + 1
    x = torch.zeros(M * K, dtype=torch.int16, device="cuda")
    am, mv, lg = _outs(M, V)
    with pytest.raises(tg.TernError) as e:
        tg.i8_head_gemv_argmax_noalloc(W, sh, V, K, M, tg.TERN_ACT_BF16, x, None, am, mv, lg)
    assert e.value.status == tg.TERN_ESHAPE
    torch.cuda.synchronize()
    assert (host(am) == -1).all()                # nothing was launched
