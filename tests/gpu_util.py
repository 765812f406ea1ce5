"""Helpers shared by the GPU parity tests: device transfer, packing through the C ABI, and the
bf16-mode tolerance of the packed-ternary path (relative L2 error <= 1e-5 over the output and
|err| <= 1e-4 * sum_k |x_k| * scale for every output)."""
from __future__ import annotations

import numpy as np
import torch

import bit_gemv_tern_b200 as tg
import oracle
import synth

REL_L2 = 1e-5
PER_OUT = 1e-4


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def pack_gpu(trits: torch.Tensor, scale_f16: torch.Tensor, N: int, K: int) -> tg.TernMatrix:
    W = tg.TernMatrix.empty(N, K)
    W.scale.copy_(scale_f16.view(torch.float16) if scale_f16.dtype != torch.float16 else scale_f16)
    W._c.scale_f16 = W.scale.data_ptr()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_pack(tg.TERN_SRC_INT8_TRITS, trits, N, K, W.planes, flag)
    assert tg.tern_read_flag(flag) == 0
    return W


def make_matrix(seed: int, tid: int, N: int, K: int, p=synth.P_DEFAULT, host_trits: bool = True):
    """(TernMatrix on the GPU, host trits or None, host fp16 scale bits)."""
    s = synth.row_scales(seed, tid, N)
    if host_trits:
        t = synth.trits(seed, tid, N, K, p)
        td = dev(t)
    else:
        import synth.cuda as sc
        td = torch.empty(N * K, dtype=torch.int8, device="cuda")
        sc.trits_into(td, seed, tid, K, p)
        t = None
    W = pack_gpu(td, dev(s.view(np.float16)), N, K)
    del td
    return W, t, s


def check_bf16(y: np.ndarray, y_ref: np.ndarray, x_bf16: np.ndarray, scale_f16: np.ndarray,
               rel_l2=True) -> None:
    """y, y_ref: [M, N]; x_bf16: [M, K] bits; scale_f16: [N] bits (or for sampled rows, the rows' scales).
    The per-output bound is always checked. rel_l2: True checks relative L2 <= 1e-5; a float checks
    it against that limit instead; False skips it (for inputs whose every output is made of
    activations far below the absmax -- a single nonzero weight per row against sub-grid values --
    the relative L2 error is not bounded by any fixed-precision arithmetic, while the per-output
    bound still holds for every input)."""
    y = np.asarray(y, np.float64)
    err = y - y_ref
    absx = np.abs(synth.bf16_bits_to_f32(x_bf16).astype(np.float64)).sum(1)       # [M]
    sc = scale_f16.view(np.float16).astype(np.float64)                             # [N]
    bound = PER_OUT * absx[:, None] * sc[None, :]
    assert (np.abs(err) <= bound).all(), f"max |err|/bound = {(np.abs(err) / bound).max():.3e}"
    rel = np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-300)
    if rel_l2 is not False:
        limit = REL_L2 if rel_l2 is True else float(rel_l2)
        assert rel <= limit, f"rel-L2 {rel:.3e} > {limit} (max |err|/bound {(np.abs(err) / bound).max():.3e})"
