"""GPU parity of the speculative-verify round: the int8 head over the k + 1 rows of a verify pass
with the acceptance count computed in the same launch (i8_head_verify), and the acceptance rule
alone (tern_verify_accept), against the CPU oracle's head argmax and acceptance count: every draft
accepted, the first rejected, a rejection in the middle, k = 0, and exact ties (the lowest index
wins, so a draft naming the higher duplicate is rejected)."""
import numpy as np
import pytest
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth
from gpu_util import PER_OUT, dev, host

pytestmark = pytest.mark.gpu


def _run(W, sh, X, draft, mode):
    V, K = W.shape
    M = X.shape[0]
    ws = torch.zeros(tg.i8_head_workspace_bytes(V, M), dtype=torch.uint8, device="cuda")
    am = torch.full((M,), -1, dtype=torch.int32, device="cuda")
    mv = torch.empty(M, dtype=torch.float32, device="cuda")
    acc = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    xd = dev(X.view(np.int16))
    d = dev(np.asarray(draft, np.int32)) if len(draft) else None
    if mode == "int8":
        q = torch.empty(M * K, dtype=torch.int8, device="cuda")
        sx = torch.empty(M, dtype=torch.float32, device="cuda")
        tg.tern_quantize_act(xd, M, K, q, sx)
        tg.i8_head_verify(dev(W), dev(sh.view(np.float16)), V, K, M, tg.TERN_ACT_INT8, q, sx, d, am, mv, acc, ws)
        qs = (host(q).reshape(M, K), host(sx))
    else:
        tg.i8_head_verify(dev(W), dev(sh.view(np.float16)), V, K, M, tg.TERN_ACT_BF16, xd, None, d, am, mv, acc, ws)
        qs = None
    torch.cuda.synchronize()
    assert (host(ws) == 0).all()
    return host(am), host(mv), tuple(int(v) for v in host(acc)), qs


def _drafts(am, k, case, rng):
    if case == "all":
        return list(am[:k])
    d = list(am[:k])
    j = 0 if case == "first" else int(rng.integers(1, k)) if k > 1 else 0
    if k:
        d[j] = int(am[j]) + 1
    return d


@pytest.mark.parametrize("case", ["all", "first", "middle"])
@pytest.mark.parametrize("k", [0, 1, 3, 6, 15])
@pytest.mark.parametrize("mode", ["int8", "bf16"])
def test_verify_round_matches_oracle(mode, k, case):
    V, K, M = 5000, 4096, k + 1
    rng = np.random.default_rng(100 * k + len(case))
    W = synth.head_weights(71, k, V, K)
    sh = synth.head_scales(71, k, V)
    X = synth.activations(71, 100 + k, M, K)
    # the oracle's greedy tokens decide the drafts
    if mode == "int8":
        q_ref, sx_ref = oracle.quantize_act(X, K)
        am_ref, mv_ref, _ = oracle.head_i8(W, sh, q_ref, sx_ref)
    else:
        am_ref, mv_ref, lg_ref = oracle.head_bf16(W, sh, X, want_logits=True)
    draft = _drafts(am_ref, k, case, rng)
    am, mv, acc, qs = _run(W, sh, X, draft, mode)
    if mode == "int8":
        assert (am == am_ref).all() and (mv == mv_ref).all()
    else:
        absx = np.abs(synth.bf16_bits_to_f32(X).astype(np.float64)).sum(1)
        for m in range(M):
            if am[m] != am_ref[m]:                    # a near tie only
                bound = PER_OUT * absx[m] * 127.0 * float(sh.view(np.float16)[am[m]])
                assert mv_ref[m] - lg_ref[m, am[m]] <= bound
    # the device count follows the rule on the device's own argmax, and equals the oracle's
    assert acc == oracle.verify_accept(am, draft)
    if (am == am_ref).all():
        assert acc == oracle.verify_accept(am_ref, draft)
        want_n = {"all": k, "first": 0, "middle": None}[case]
        if want_n is not None and k:
            assert acc[0] == want_n


def test_verify_round_exact_tie_takes_lowest_index():
    V, K, M = 3000, 1024, 3
    W = synth.head_weights(72, 1, V, K)
    sh = synth.head_scales(72, 1, V)
    X = synth.activations(72, 2, M, K)
    q, sx = oracle.quantize_act(X, K)
    am0, _, _ = oracle.head_i8(W, sh, q, sx)
    w = int(am0[0])
    other = V - 1 if w < V // 2 else 0
    W[other], sh[other] = W[w], sh[w]
    lo, hi = min(w, other), max(w, other)
    am_ref, _, _ = oracle.head_i8(W, sh, q, sx)
    assert am_ref[0] == lo
    am, _, acc, _ = _run(W, sh, X, [hi, int(am_ref[1])], "int8")
    assert am[0] == lo and acc == (0, lo)
    am, _, acc, _ = _run(W, sh, X, [lo, int(am_ref[1])], "int8")
    assert acc == oracle.verify_accept(am_ref, [lo, int(am_ref[1])]) == (2, int(am_ref[2]))


def test_verify_accept_standalone():
    rng = np.random.default_rng(3)
    acc = torch.empty(2, dtype=torch.int32, device="cuda")
    for _ in range(40):
        k = int(rng.integers(0, 16))
        am = rng.integers(0, 5, k + 1).astype(np.int32)
        dr = np.where(rng.random(k) < 0.85, am[:k], rng.integers(0, 5, k)).astype(np.int32)
        tg.tern_verify_accept(dev(am), dev(dr) if k else None, k, acc)
        torch.cuda.synchronize()
        assert tuple(int(v) for v in host(acc)) == oracle.verify_accept(am, dr)


def test_verify_argument_errors():
    V, K, M = 64, 128, 3
    W = torch.zeros(V * K, dtype=torch.int8, device="cuda")
    sh = torch.ones(V, dtype=torch.float16, device="cuda")
    x = torch.zeros(M * K, dtype=torch.int16, device="cuda")
    am = torch.empty(M, dtype=torch.int32, device="cuda")
    mv = torch.empty(M, dtype=torch.float32, device="cuda")
    acc = torch.empty(2, dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(tg.TernError):                     # M > 1 needs the drafts
        tg.i8_head_verify(W, sh, V, K, M, tg.TERN_ACT_BF16, x, None, None, am, mv, acc, ws)
    with pytest.raises(tg.TernError):                     # no accept output
        tg.i8_head_verify(W, sh, V, K, M, tg.TERN_ACT_BF16, x, None, am, am, mv, None, ws)
    with pytest.raises(tg.TernError):
        tg.tern_verify_accept(am, None, 2, acc)           # k > 0 needs the drafts
