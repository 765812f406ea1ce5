"""CPU oracle for the packed-ternary path: numpy-facing wrappers over oracle/tern_oracle.c.

TEST INFRASTRUCTURE. Only tests/, the smoke check in __graft_entry__ and the CPU-baseline leg of
bench.py may import this package. The product (bit_gemv_tern_b200) never imports it and shares
no code with it. See tern_oracle.c for the definitions, the layout and the sources on the pages.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]; L.orc_half_to_double.restype = ctypes.c_double
        L.orc_bf16_to_float.argtypes = [ctypes.c_uint16]; L.orc_bf16_to_float.restype = ctypes.c_float
        L.orc_packed_words.argtypes = [i32, i32]; L.orc_packed_words.restype = i64
        L.orc_pack.argtypes = [vp, i32, i32, vp]; L.orc_pack.restype = i64
        L.orc_unpack.argtypes = [vp, i32, i32, vp]; L.orc_unpack.restype = None
        L.orc_occupancy.argtypes = [vp, i32, i32, vp]; L.orc_occupancy.restype = None
        L.orc_base3_row_bytes.argtypes = [i32]; L.orc_base3_row_bytes.restype = i32
        L.orc_base3_encode.argtypes = [vp, i32, i32, vp]; L.orc_base3_encode.restype = i64
        L.orc_base3_decode.argtypes = [vp, i32, i32, vp]; L.orc_base3_decode.restype = i64
        L.orc_gemm_bf16.argtypes = [vp, vp, i32, i32, i32, vp, vp, i32]; L.orc_gemm_bf16.restype = None
        L.orc_quantize_act.argtypes = [vp, i32, i32, vp, vp]; L.orc_quantize_act.restype = None
        L.orc_gemm_i8.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, i32]; L.orc_gemm_i8.restype = None
        L.orc_head_bf16.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, i32]; L.orc_head_bf16.restype = None
        L.orc_head_i8.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, i32]; L.orc_head_i8.restype = None
        L.orc_round_bf16.argtypes = [ctypes.c_double]; L.orc_round_bf16.restype = ctypes.c_uint16
        L.orc_rmsnorm.argtypes = [vp, i32, i32, vp, ctypes.c_double, vp]; L.orc_rmsnorm.restype = None
        L.orc_swiglu.argtypes = [vp, i32, i32, vp]; L.orc_swiglu.restype = None
        L.orc_verify_accept.argtypes = [vp, vp, i32, vp, vp]; L.orc_verify_accept.restype = None
        L.orc_rans_freqs.argtypes = [vp, i64, vp]; L.orc_rans_freqs.restype = None
        L.orc_rans_encode.argtypes = [vp, i32, i32, vp, vp, vp, i64]; L.orc_rans_encode.restype = i64
        L.orc_rans_decode.argtypes = [vp, vp, i32, i32, vp, vp]; L.orc_rans_decode.restype = i32
        L.orc_fv5_pack.argtypes = [vp, i32, i32, vp]; L.orc_fv5_pack.restype = i64
        L.orc_fv5_unpack.argtypes = [vp, i32, i32, vp]; L.orc_fv5_unpack.restype = None
        L.orc_fv5_gemm_bf16.argtypes = [vp, vp, i32, i32, i32, vp, vp, i32]; L.orc_fv5_gemm_bf16.restype = None
        L.orc_fv5_gemm_i8.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, i32]; L.orc_fv5_gemm_i8.restype = None
        L.orc_fv5b_head.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, vp]; L.orc_fv5b_head.restype = None
        _LIB = L
    return _LIB


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    return os.cpu_count() or 1


class OracleError(ValueError):
    pass


def half_to_double(h: int) -> float:
    return lib().orc_half_to_double(int(h))


def bf16_to_float(b: int) -> float:
    return lib().orc_bf16_to_float(int(b))


def pack(trits: np.ndarray) -> np.ndarray:
    """int8[N, K] trits -> uint32[N, K/16] planes (mask words then sign words per row)."""
    t = _c(trits, np.int8)
    N, K = t.shape
    if K % 128:
        raise OracleError("K must be a multiple of 128")
    planes = np.empty((N, K // 16), dtype=np.uint32)
    bad = lib().orc_pack(_p(t), N, K, _p(planes))
    if bad >= 0:
        raise OracleError(f"invalid trit at flat index {bad}")
    return planes


def unpack(planes: np.ndarray, K: int) -> np.ndarray:
    pl = _c(planes, np.uint32)
    N = pl.size // (K // 16)
    out = np.empty((N, K), dtype=np.int8)
    lib().orc_unpack(_p(pl), N, K, _p(out))
    return out


def occupancy(planes: np.ndarray, K: int) -> np.ndarray:
    """int64[N, 3]: zeros, +1s, -1s per row."""
    pl = _c(planes, np.uint32)
    N = pl.size // (K // 16)
    out = np.empty((N, 3), dtype=np.int64)
    lib().orc_occupancy(_p(pl), N, K, _p(out))
    return out


def base3_row_bytes(K: int) -> int:
    return lib().orc_base3_row_bytes(K)


def base3_encode(trits: np.ndarray) -> np.ndarray:
    t = _c(trits, np.int8)
    N, K = t.shape
    out = np.empty((N, base3_row_bytes(K)), dtype=np.uint8)
    bad = lib().orc_base3_encode(_p(t), N, K, _p(out))
    if bad >= 0:
        raise OracleError(f"invalid trit at flat index {bad}")
    return out


def base3_decode(data: np.ndarray, N: int, K: int) -> np.ndarray:
    b = _c(data, np.uint8)
    if b.size != N * base3_row_bytes(K):
        raise OracleError("transport size does not match N x ceil(K/5)")
    out = np.zeros((N, K), dtype=np.int8)
    bad = lib().orc_base3_decode(_p(b), N, K, _p(out))
    if bad >= 0:
        raise OracleError(f"invalid base-3 byte at flat index {bad}")
    return out


def gemm_bf16(planes: np.ndarray, scale_f16: np.ndarray, K: int, x_bf16: np.ndarray,
              nthreads: int | None = None) -> np.ndarray:
    """fp64 Y[M, N] = scale[n] * sum_k t[n, k] * x[m, k]; x as bf16 bit patterns [M, K] (or [K])."""
    pl = _c(planes, np.uint32)
    N = pl.size // (K // 16)
    x = _c(x_bf16, np.uint16).reshape(-1, K)
    M = x.shape[0]
    s = _c(scale_f16, np.uint16)
    assert s.size == N
    y = np.empty((M, N), dtype=np.float64)
    lib().orc_gemm_bf16(_p(pl), _p(s), N, K, M, _p(x), _p(y), nthreads or default_threads())
    return y


def quantize_act(x_bf16: np.ndarray, K: int) -> tuple[np.ndarray, np.ndarray]:
    x = _c(x_bf16, np.uint16).reshape(-1, K)
    M = x.shape[0]
    q = np.empty((M, K), dtype=np.int8)
    sx = np.empty(M, dtype=np.float32)
    lib().orc_quantize_act(_p(x), M, K, _p(q), _p(sx))
    return q, sx


def gemm_i8(planes: np.ndarray, scale_f16: np.ndarray, K: int, q: np.ndarray, sx: np.ndarray,
            nthreads: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """int8 mode: (acc int64[M, N], y float32[M, N]) with y = ((float)acc * s_x) * scale."""
    pl = _c(planes, np.uint32)
    N = pl.size // (K // 16)
    qq = _c(q, np.int8).reshape(-1, K)
    M = qq.shape[0]
    s = _c(scale_f16, np.uint16)
    sxx = _c(sx, np.float32).reshape(M)
    acc = np.empty((M, N), dtype=np.int64)
    y = np.empty((M, N), dtype=np.float32)
    lib().orc_gemm_i8(_p(pl), _p(s), N, K, M, _p(qq), _p(sxx), _p(acc), _p(y), nthreads or default_threads())
    return acc, y


def head_bf16(W: np.ndarray, sh_f16: np.ndarray, x_bf16: np.ndarray, want_logits: bool = False,
              nthreads: int | None = None):
    """Returns (argmax int32[M], maxval float64[M], logits float64[M, V] or None)."""
    w = _c(W, np.int8)
    V, K = w.shape
    x = _c(x_bf16, np.uint16).reshape(-1, K)
    M = x.shape[0]
    sh = _c(sh_f16, np.uint16)
    am = np.empty(M, dtype=np.int32)
    mv = np.empty(M, dtype=np.float64)
    lg = np.empty((M, V), dtype=np.float64) if want_logits else None
    lib().orc_head_bf16(_p(w), _p(sh), V, K, M, _p(x), _p(lg), _p(am), _p(mv), nthreads or default_threads())
    return am, mv, lg


def head_i8(W: np.ndarray, sh_f16: np.ndarray, q: np.ndarray, sx: np.ndarray, want_logits: bool = False,
            nthreads: int | None = None):
    """Returns (argmax int32[M], maxval float32[M], logits float32[M, V] or None)."""
    w = _c(W, np.int8)
    V, K = w.shape
    qq = _c(q, np.int8).reshape(-1, K)
    M = qq.shape[0]
    sh = _c(sh_f16, np.uint16)
    sxx = _c(sx, np.float32).reshape(M)
    am = np.empty(M, dtype=np.int32)
    mv = np.empty(M, dtype=np.float32)
    lg = np.empty((M, V), dtype=np.float32) if want_logits else None
    lib().orc_head_i8(_p(w), _p(sh), V, K, M, _p(qq), _p(sxx), _p(lg), _p(am), _p(mv), nthreads or default_threads())
    return am, mv, lg


def round_bf16(v) -> np.ndarray:
    """fp64 values -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    a = np.asarray(v, dtype=np.float64)
    f = lib().orc_round_bf16
    return np.array([f(float(x)) for x in a.reshape(-1)], dtype=np.uint16).reshape(a.shape)


def rmsnorm(x_f32: np.ndarray, gain_bf16: np.ndarray, eps: float) -> np.ndarray:
    """bf16 bits [M, K] of RMSNorm(x) * gain per row (fp64, one rounding); x fp32 [M, K] or [K]."""
    K = np.asarray(gain_bf16).size
    x = _c(x_f32, np.float32).reshape(-1, K)
    M = x.shape[0]
    g = _c(gain_bf16, np.uint16)
    out = np.empty((M, K), dtype=np.uint16)
    lib().orc_rmsnorm(_p(x), M, K, _p(g), float(eps), _p(out))
    return out


def swiglu(gu_f32: np.ndarray, K: int) -> np.ndarray:
    """bf16 bits [M, K] of silu(gate) * up per row; gu fp32 [M, 2K] (gate first, then up)."""
    gu = _c(gu_f32, np.float32).reshape(-1, 2 * K)
    M = gu.shape[0]
    out = np.empty((M, K), dtype=np.uint16)
    lib().orc_swiglu(_p(gu), M, K, _p(out))
    return out


def verify_accept(argmax, draft) -> tuple[int, int]:
    """(accepted drafts n, next token argmax[n]) for argmax [k+1] and draft [k]."""
    am = _c(argmax, np.int32).reshape(-1)
    dr = _c(draft, np.int32).reshape(-1)
    k = dr.size
    if am.size != k + 1:
        raise OracleError("argmax needs k + 1 entries")
    n = np.zeros(1, np.int32)
    nt = np.zeros(1, np.int32)
    lib().orc_verify_accept(_p(am), _p(dr) if k else _p(np.zeros(1, np.int32)), k, _p(n), _p(nt))
    return int(n[0]), int(nt[0])


def rans_freqs(trits: np.ndarray) -> np.ndarray:
    """Quantised frequencies (uint16[3], order t = 0, +1, -1, sum 4096) of a tensor's trits."""
    t = _c(trits, np.int8).reshape(-1)
    f = np.empty(3, np.uint16)
    lib().orc_rans_freqs(_p(t), t.size, _p(f))
    return f


def rans_encode(trits: np.ndarray, freq: np.ndarray | None = None):
    """Order-0 rANS transport of an int8 [N, K] trit tensor: (freq uint16[3], row_end uint32[N],
    payload uint8[...]). freq defaults to the tensor's own quantised frequencies."""
    t = _c(trits, np.int8)
    N, K = t.shape
    f = rans_freqs(t) if freq is None else _c(freq, np.uint16)
    row_end = np.empty(N, np.uint32)
    cap = N * (2 * K + 8)
    out = np.empty(cap, np.uint8)
    n = lib().orc_rans_encode(_p(t), N, K, _p(f), _p(row_end), _p(out), cap)
    if n < 0:
        raise OracleError("rans_encode: not a trit tensor")
    return f, row_end, out[:n].copy()


def rans_decode(freq: np.ndarray, row_end: np.ndarray, payload: np.ndarray, N: int, K: int):
    """(trits int8[N, K], ok): ok is False if any row's stream is invalid."""
    t = np.empty((N, K), np.int8)
    pl, re, f = _c(payload, np.uint8), _c(row_end, np.uint32), _c(freq, np.uint16)
    st = lib().orc_rans_decode(_p(pl), _p(re), N, K, _p(f), _p(t))
    return t, st == 0


def fv5_pack(codes: np.ndarray) -> np.ndarray:
    """Five-valued codes int8 [N, K] (values -2..2, K % 256 == 0) -> planes uint32 [N, 3K/32]."""
    c = _c(codes, np.int8)
    N, K = c.shape
    if K % 512:
        raise OracleError("fv5_pack: K must be a multiple of 512")
    planes = np.empty((N, 3 * K // 32), np.uint32)
    if lib().orc_fv5_pack(_p(c), N, K, _p(planes)) != 0:
        raise OracleError("fv5_pack: code outside -2..2")
    return planes


def fv5_unpack(planes: np.ndarray, K: int) -> np.ndarray:
    pl = _c(planes, np.uint32)
    N = pl.size // (3 * K // 32)
    out = np.empty((N, K), np.int8)
    lib().orc_fv5_unpack(_p(pl), N, K, _p(out))
    return out


def fv5_gemm_bf16(planes, scales, K: int, x_bf16, nthreads: int | None = None) -> np.ndarray:
    """fp64 Y[M, N] of the five-valued weights (scales fp32 [N, K/256, 2]) times bf16 x [M, K]."""
    pl = _c(planes, np.uint32)
    N = pl.size // (3 * K // 32)
    x = _c(x_bf16, np.uint16).reshape(-1, K)
    sc = _c(scales, np.float32)
    y = np.empty((x.shape[0], N), np.float64)
    lib().orc_fv5_gemm_bf16(_p(pl), _p(sc), N, K, x.shape[0], _p(x), _p(y), nthreads or default_threads())
    return y


def fv5_gemm_i8(planes, scales, K: int, q, sx, nthreads: int | None = None) -> np.ndarray:
    pl = _c(planes, np.uint32)
    N = pl.size // (3 * K // 32)
    qq = _c(q, np.int8).reshape(-1, K)
    sc, sxx = _c(scales, np.float32), _c(sx, np.float32)
    y = np.empty((qq.shape[0], N), np.float32)
    lib().orc_fv5_gemm_i8(_p(pl), _p(sc), N, K, qq.shape[0], _p(qq), _p(sxx), _p(y), nthreads or default_threads())
    return y


def fv5b_head(W, S, x_bf16=None, q=None, sx=None):
    """(argmax int32[M], logits float64[M, V]) of the block-scaled int8 head; bf16 x or int8 q + s_x."""
    w = _c(W, np.int8)
    V, K = w.shape
    if q is not None:
        qq = _c(q, np.int8).reshape(-1, K)
        M, X, Q, SX = qq.shape[0], None, qq, _c(sx, np.float32)
    else:
        X = _c(x_bf16, np.uint16).reshape(-1, K)
        M, Q, SX = X.shape[0], None, None
    ss = _c(S, np.float32)
    lg = np.empty((M, V), np.float64)
    am = np.empty(M, np.int32)
    lib().orc_fv5b_head(_p(w), _p(ss), V, K, M, _p(X), _p(Q), _p(SX), _p(lg), _p(am))
    return am, lg
