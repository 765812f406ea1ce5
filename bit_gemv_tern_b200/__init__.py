"""bit_gemv_tern_b200: packed-ternary linear layers and the int8 output head on NVIDIA B200.

A thin ctypes binding over libterngemv.so, whose C ABI is declared in include/tern.h. Every
function here only marshals arguments: device memory comes from torch tensors (data_ptr), the
stream from torch's current stream, and every step of the computation runs in the library's
sm_100a kernels. There is no CPU path; if the shared library is missing, importing the functions
raises.

The functions keep the C names (tern_pack, tern_gemv, tern_gemm_small_m, tern_gemm_prefill,
i8_head_gemv_argmax, ...), take torch tensors, check the returned tern_status and raise
TernError on anything but TERN_OK.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "TernError", "TernMatrix", "lib", "library_path",
    "TERN_ACT_BF16", "TERN_ACT_INT8", "TERN_SRC_INT8_TRITS", "TERN_SRC_BASE3", "TERN_FLAG_PDL", "TERN_FLAG_TCGEN05",
    "tern_packed_bytes", "tern_base3_bytes", "tern_pack", "tern_pack_batch", "tern_base3_encode", "tern_occupancy",
    "tern_quantize_act", "tern_gemv", "tern_gemm_small_m", "tern_gemm_prefill",
    "i8_head_workspace_bytes", "i8_head_gemv_argmax", "i8_head_gemv_argmax_noalloc",
    "TERN_HEAD_NOALLOC_MAX_M", "tern_read_flag", "tern_device_status",
    "GemvBatch", "tern_gemv_batch", "tern_gemv_batch_workspace_bytes", "tern_gemm_batch",
    "tern_gemm_batch_workspace_bytes", "tern_gemm_batch_pro", "tern_act_prologue",
    "i8_head_verify", "tern_verify_accept",
    "ChainItem", "Chain",
    "Fv5Matrix", "tern_fv5_packed_bytes", "tern_fv5_pack", "tern_fv5_gemm", "tern_fv5_gemv_batch",
    "fv5b_head_gemv_argmax",
    "tern_rans_payload_bound", "tern_rans_workspace_bytes", "tern_rans_encode", "tern_rans_decode",
    "TERN_PRO_NONE", "TERN_PRO_BF16", "TERN_PRO_CAST", "TERN_PRO_RMSNORM", "TERN_PRO_SWIGLU",
    "tern_status_string",
]

TERN_OK, TERN_EINVAL, TERN_ESHAPE, TERN_EBADCODE, TERN_ECUDA, TERN_ETIMEOUT = range(6)
TERN_ACT_BF16, TERN_ACT_INT8 = 0, 1
TERN_SRC_INT8_TRITS, TERN_SRC_BASE3 = 0, 1
TERN_FLAG_PDL = 1
TERN_FLAG_TCGEN05 = 2
TERN_HEAD_NOALLOC_MAX_M = 16
TERN_PRO_NONE, TERN_PRO_BF16, TERN_PRO_CAST, TERN_PRO_RMSNORM, TERN_PRO_SWIGLU = range(5)

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libterngemv.so")
_LIB = None


class TernError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {tern_status_string(status)}")


class _Matrix(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("planes", ctypes.c_void_p), ("scale_f16", ctypes.c_void_p)]


def lib() -> ctypes.CDLL:
    """Load libterngemv.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(library_path):
            raise RuntimeError(f"{library_path} is missing: build it with `python bit_gemv_tern_b200/build.py`")
        L = ctypes.CDLL(library_path)
        vp, i32, u32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
        mp = ctypes.POINTER(_Matrix)
        sig = {
            "tern_status_string": ([i32], ctypes.c_char_p),
            "tern_packed_bytes": ([i32, i32], sz),
            "tern_base3_bytes": ([i32, i32], sz),
            "tern_pack": ([i32, vp, i32, i32, vp, vp, vp], i32),
            "tern_base3_encode": ([vp, i32, i32, vp, vp, vp], i32),
            "tern_pack_batch": ([i32, vp, i32, vp, vp], i32),
            "tern_occupancy": ([mp, vp, vp], i32),
            "tern_quantize_act": ([vp, i32, i32, vp, vp, vp], i32),
            "tern_gemv": ([mp, i32, vp, vp, vp, vp, vp], i32),
            "tern_gemv_ex": ([mp, i32, vp, vp, vp, vp, u32, vp], i32),
            "tern_gemm_small_m": ([mp, i32, i32, vp, vp, vp, vp], i32),
            "tern_gemm_small_m_ex": ([mp, i32, i32, vp, vp, vp, u32, vp], i32),
            "tern_gemm_prefill": ([mp, i32, vp, vp, vp], i32),
            "i8_head_workspace_bytes": ([i32, i32], sz),
            "i8_head_gemv_argmax": ([vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "i8_head_gemv_argmax_ex": ([vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, u32, vp], i32),
            "i8_head_gemv_argmax_noalloc": ([vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp], i32),
            "tern_read_flag": ([vp, vp], i32),
            "tern_device_status": ([vp], i32),
            "tern_gemv_batch_workspace_bytes": ([vp, i32, i32], sz),
            "tern_gemv_batch": ([vp, i32, i32, vp, sz, u32, vp], i32),
            "tern_gemm_batch_workspace_bytes": ([vp, i32, i32, i32], sz),
            "tern_gemm_batch": ([vp, i32, i32, i32, vp, sz, u32, vp], i32),
            "tern_gemm_batch_pro": ([vp, vp, i32, i32, i32, vp, sz, u32, vp], i32),
            "tern_act_prologue": ([vp, i32, i32, vp, vp], i32),
            "i8_head_verify": ([vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "tern_verify_accept": ([vp, vp, i32, vp, vp], i32),
            "tern_chain_workspace_bytes": ([vp, i32, i32], sz),
            "tern_chain_plan": ([vp, i32, i32, vp, sz, vp], i32),
            "tern_chain_run": ([vp, vp], i32),
            "tern_fv5_packed_bytes": ([i32, i32], sz),
            "tern_fv5_pack": ([vp, i32, i32, vp, vp, vp], i32),
            "tern_fv5_gemm": ([vp, i32, i32, vp, vp, vp, vp], i32),
            "tern_fv5_gemv_batch": ([vp, i32, i32, vp], i32),
            "fv5b_head_gemv_argmax": ([vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp], i32),
            "tern_rans_payload_bound": ([i32, i32], sz),
            "tern_rans_workspace_bytes": ([i32, i32], sz),
            "tern_rans_encode": ([vp, i32, i32, vp, vp, vp, sz, vp, sz, vp, vp], i32),
            "tern_rans_decode": ([vp, i32, vp, vp], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def tern_status_string(status: int) -> str:
    return lib().tern_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != TERN_OK:
        raise TernError(status, what)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


class _Item(ctypes.Structure):
    _fields_ = [("W", _Matrix), ("x_dev", ctypes.c_void_p), ("x_scale_dev", ctypes.c_void_p),
                ("y_dev", ctypes.c_void_p)]


class _Prologue(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("eps", ctypes.c_float), ("src_dev", ctypes.c_void_p),
                ("gain_dev", ctypes.c_void_p)]


def _prologues(pros):
    """pros: list of None or (kind, src tensor, gain tensor or None, eps)."""
    arr = (_Prologue * len(pros))()
    for i, pr in enumerate(pros):
        if pr is None:
            arr[i].kind = TERN_PRO_NONE
            continue
        kind, src, gain, eps = pr
        arr[i].kind, arr[i].src_dev, arr[i].gain_dev, arr[i].eps = int(kind), _ptr(src), _ptr(gain), float(eps)
    return arr


class TernMatrix:
    """A packed ternary matrix: planes (int32/uint32 tensor of N*K/16 words) and fp16 scales."""

    def __init__(self, planes, scale_f16, N: int, K: int):
        self.planes, self.scale, self.N, self.K = planes, scale_f16, int(N), int(K)
        self._c = _Matrix(self.N, self.K, _ptr(planes), _ptr(scale_f16))

    def ref(self):
        return ctypes.byref(self._c)

    @staticmethod
    def empty(N: int, K: int, device="cuda"):
        import torch
        planes = torch.empty(N * K // 16, dtype=torch.int32, device=device)
        scale = torch.empty(N, dtype=torch.float16, device=device)
        return TernMatrix(planes, scale, N, K)


def tern_packed_bytes(N: int, K: int) -> int:
    return int(lib().tern_packed_bytes(N, K))


def tern_base3_bytes(N: int, K: int) -> int:
    return int(lib().tern_base3_bytes(N, K))


def tern_pack(src_kind: int, src, N: int, K: int, planes, err_flag, stream=None) -> None:
    """Pack dense int8 trits (src_kind=TERN_SRC_INT8_TRITS) or the base-3 transport
    (TERN_SRC_BASE3) into planes; invalid input values set err_flag (see tern_read_flag)."""
    _check(lib().tern_pack(src_kind, _ptr(src), N, K, _ptr(planes), _ptr(err_flag), _stream(stream)), "tern_pack")


class _PackItem(ctypes.Structure):
    _fields_ = [("src_dev", ctypes.c_void_p), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("planes_dev", ctypes.c_void_p)]


def tern_pack_batch(src_kind: int, entries, err_flag, stream=None) -> None:
    """tern_pack over a list of (src, N, K, planes) in one call (one flag clear, one launch)."""
    arr = (_PackItem * len(entries))()
    for i, (src, N, K, planes) in enumerate(entries):
        arr[i].src_dev, arr[i].N, arr[i].K, arr[i].planes_dev = _ptr(src), int(N), int(K), _ptr(planes)
    _check(lib().tern_pack_batch(src_kind, arr, len(entries), _ptr(err_flag), _stream(stream)), "tern_pack_batch")


def tern_base3_encode(trits, N: int, K: int, out, err_flag, stream=None) -> None:
    _check(lib().tern_base3_encode(_ptr(trits), N, K, _ptr(out), _ptr(err_flag), _stream(stream)),
           "tern_base3_encode")


def tern_occupancy(W: TernMatrix, counts, stream=None) -> None:
    _check(lib().tern_occupancy(W.ref(), _ptr(counts), _stream(stream)), "tern_occupancy")


def tern_quantize_act(x_bf16, M: int, K: int, q, s_x, stream=None) -> None:
    _check(lib().tern_quantize_act(_ptr(x_bf16), M, K, _ptr(q), _ptr(s_x), _stream(stream)), "tern_quantize_act")


def tern_gemv(W: TernMatrix, act: int, x, x_scale, y, flags: int = 0, stream=None, acc=None) -> None:
    """acc: optional int32 tensor of N elements; int8 mode writes the exact sums sum_k t*q there."""
    _check(lib().tern_gemv_ex(W.ref(), act, _ptr(x), _ptr(x_scale), _ptr(y), _ptr(acc), flags, _stream(stream)),
           "tern_gemv")


def tern_gemm_small_m(W: TernMatrix, M: int, act: int, X, x_scale, Y, flags: int = 0, stream=None) -> None:
    _check(lib().tern_gemm_small_m_ex(W.ref(), M, act, _ptr(X), _ptr(x_scale), _ptr(Y), flags, _stream(stream)),
           "tern_gemm_small_m")


def tern_gemm_prefill(W: TernMatrix, M: int, X_bf16, Y, stream=None) -> None:
    _check(lib().tern_gemm_prefill(W.ref(), M, _ptr(X_bf16), _ptr(Y), _stream(stream)), "tern_gemm_prefill")


def i8_head_workspace_bytes(V: int, M: int) -> int:
    return int(lib().i8_head_workspace_bytes(V, M))


def i8_head_gemv_argmax(W, scale_f16, V: int, K: int, M: int, act: int, X, x_scale, argmax, maxval,
                        logits, workspace, flags: int = 0, stream=None) -> None:
    """workspace: a zero-filled uint8 CUDA tensor of at least i8_head_workspace_bytes(V, M) bytes."""
    _check(lib().i8_head_gemv_argmax_ex(_ptr(W), _ptr(scale_f16), V, K, M, act, _ptr(X), _ptr(x_scale),
                                        _ptr(argmax), _ptr(maxval), _ptr(logits), _ptr(workspace),
                                        int(workspace.numel() * workspace.element_size()), flags,
                                        _stream(stream)), "i8_head_gemv_argmax")


def i8_head_gemv_argmax_noalloc(W, scale_f16, V: int, K: int, M: int, act: int, X, x_scale, argmax, maxval,
                                logits, stream=None) -> None:
    """i8_head_gemv_argmax with the library's internal per-device scratch instead of a caller
    workspace (M <= TERN_HEAD_NOALLOC_MAX_M; calls that overlap in time race)."""
    _check(lib().i8_head_gemv_argmax_noalloc(_ptr(W), _ptr(scale_f16), V, K, M, act, _ptr(X), _ptr(x_scale),
                                             _ptr(argmax), _ptr(maxval), _ptr(logits), _stream(stream)),
           "i8_head_gemv_argmax_noalloc")


def i8_head_verify(W, scale_f16, V: int, K: int, M: int, act: int, X, x_scale, draft, argmax, maxval, accept,
                   workspace, stream=None) -> None:
    """The head over the k + 1 = M verify rows plus the on-device acceptance count: accept[0] = accepted
    drafts n, accept[1] = the target's token argmax[n]."""
    _check(lib().i8_head_verify(_ptr(W), _ptr(scale_f16), V, K, M, act, _ptr(X), _ptr(x_scale), _ptr(draft),
                                _ptr(argmax), _ptr(maxval), _ptr(accept), _ptr(workspace),
                                int(workspace.numel() * workspace.element_size()), _stream(stream)), "i8_head_verify")


def tern_verify_accept(argmax, draft, k: int, accept, stream=None) -> None:
    _check(lib().tern_verify_accept(_ptr(argmax), _ptr(draft), k, _ptr(accept), _stream(stream)), "tern_verify_accept")


class _ChainItem(ctypes.Structure):
    _fields_ = [("W", _Matrix), ("kind", ctypes.c_int32), ("src_item", ctypes.c_int32), ("src_h", ctypes.c_int32),
                ("swiglu_out", ctypes.c_int32), ("eps", ctypes.c_float), ("src_dev", ctypes.c_void_p),
                ("gain_dev", ctypes.c_void_p), ("y_dev", ctypes.c_void_p), ("h_dev", ctypes.c_void_p),
                ("x_scale_dev", ctypes.c_void_p)]


class _ChainHandle(ctypes.Structure):
    _fields_ = [("workspace_dev", ctypes.c_void_p), ("count", ctypes.c_int32), ("mode", ctypes.c_int32),
                ("grid", ctypes.c_int32), ("stages", ctypes.c_int32), ("seg_parts", ctypes.c_int32),
                ("smem_bytes", ctypes.c_size_t)]


class ChainItem:
    """One linear of a dependent chain (see tern_chain_item in include/tern.h)."""

    def __init__(self, W: TernMatrix, kind: int, y, src_item: int = -1, src=None, gain=None, eps: float = 0.0,
                 src_h: bool = False, swiglu_out: bool = False, h=None, x_scale=None):
        self.W, self.kind, self.y, self.src_item, self.src, self.gain = W, kind, y, src_item, src, gain
        self.eps, self.src_h, self.swiglu_out, self.h, self.x_scale = eps, src_h, swiglu_out, h, x_scale


class Chain:
    """A planned chain: its workspace and host handle; call() runs it (one cooperative launch)."""

    def __init__(self, items, act: int, device="cuda"):
        import torch
        self.items = list(items)
        arr = (_ChainItem * len(self.items))()
        for i, it in enumerate(self.items):
            a = arr[i]
            a.W = it.W._c
            a.kind, a.src_item, a.src_h, a.swiglu_out = int(it.kind), int(it.src_item), int(it.src_h), int(it.swiglu_out)
            a.eps = float(it.eps)
            a.src_dev, a.gain_dev, a.y_dev = _ptr(it.src), _ptr(it.gain), _ptr(it.y)
            a.h_dev, a.x_scale_dev = _ptr(it.h), _ptr(it.x_scale)
        self._arr = arr
        n = int(lib().tern_chain_workspace_bytes(arr, len(self.items), act))
        if n == 0:
            raise TernError(TERN_ESHAPE, "tern_chain_workspace_bytes")
        self.workspace = torch.empty(n + 64, dtype=torch.uint8, device=device)
        base = self.workspace.data_ptr()
        off = (-base) % 64
        self.handle = _ChainHandle()
        _check(lib().tern_chain_plan(arr, len(self.items), act, base + off, n, ctypes.byref(self.handle)),
               "tern_chain_plan")

    def __call__(self, stream=None) -> None:
        _check(lib().tern_chain_run(ctypes.byref(self.handle), _stream(stream)), "tern_chain_run")


class _Fv5Matrix(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("planes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class Fv5Matrix:
    """Five-valued weights: planes (int32 tensor of N*3K/32 words) and fp32 scales [N, K/256, 2]."""

    def __init__(self, planes, scales, N: int, K: int):
        self.planes, self.scales, self.N, self.K = planes, scales, int(N), int(K)
        self._c = _Fv5Matrix(self.N, self.K, _ptr(planes), _ptr(scales))

    def ref(self):
        return ctypes.byref(self._c)


def tern_fv5_packed_bytes(N: int, K: int) -> int:
    return int(lib().tern_fv5_packed_bytes(N, K))


def tern_fv5_pack(codes, N: int, K: int, planes, err_flag, stream=None) -> None:
    _check(lib().tern_fv5_pack(_ptr(codes), N, K, _ptr(planes), _ptr(err_flag), _stream(stream)), "tern_fv5_pack")


def tern_fv5_gemm(W: Fv5Matrix, M: int, act: int, X, x_scale, Y, stream=None) -> None:
    _check(lib().tern_fv5_gemm(W.ref(), M, act, _ptr(X), _ptr(x_scale), _ptr(Y), _stream(stream)), "tern_fv5_gemm")


class _Fv5BatchItem(ctypes.Structure):
    _fields_ = [("W", _Fv5Matrix), ("x", ctypes.c_void_p), ("x_scale", ctypes.c_void_p), ("y", ctypes.c_void_p)]


def tern_fv5_gemv_batch(entries, act: int, stream=None) -> None:
    """entries: list of (Fv5Matrix, x, x_scale or None, y) at M = 1, run in one launch."""
    arr = (_Fv5BatchItem * len(entries))()
    for i, (W, x, sx, y) in enumerate(entries):
        arr[i] = _Fv5BatchItem(W._c, _ptr(x), _ptr(sx), _ptr(y))
    _check(lib().tern_fv5_gemv_batch(arr, len(entries), act, _stream(stream)), "tern_fv5_gemv_batch")


def fv5b_head_gemv_argmax(W, block_scale, V: int, K: int, M: int, act: int, X, x_scale, argmax, maxval, logits,
                          workspace, stream=None) -> None:
    _check(lib().fv5b_head_gemv_argmax(_ptr(W), _ptr(block_scale), V, K, M, act, _ptr(X), _ptr(x_scale),
                                       _ptr(argmax), _ptr(maxval), _ptr(logits), _ptr(workspace),
                                       int(workspace.numel() * workspace.element_size()), _stream(stream)),
           "fv5b_head_gemv_argmax")


class _RansItem(ctypes.Structure):
    _fields_ = [("freq_dev", ctypes.c_void_p), ("row_end_dev", ctypes.c_void_p), ("payload_dev", ctypes.c_void_p),
                ("payload_bytes", ctypes.c_size_t), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("planes_dev", ctypes.c_void_p)]


def tern_rans_payload_bound(N: int, K: int) -> int:
    return int(lib().tern_rans_payload_bound(N, K))


def tern_rans_workspace_bytes(N: int, K: int) -> int:
    return int(lib().tern_rans_workspace_bytes(N, K))


def tern_rans_encode(trits, N: int, K: int, freq, row_end, payload, workspace, err_flag, stream=None) -> None:
    """int8 trits [N*K] -> order-0 rANS transport: freq (3 x int16), row_end (N x int32), payload (uint8)."""
    _check(lib().tern_rans_encode(_ptr(trits), N, K, _ptr(freq), _ptr(row_end), _ptr(payload),
                                  int(payload.numel() * payload.element_size()), _ptr(workspace),
                                  int(workspace.numel() * workspace.element_size()), _ptr(err_flag),
                                  _stream(stream)), "tern_rans_encode")


def tern_rans_decode(entries, err_flag, stream=None) -> None:
    """entries: list of (freq, row_end, payload, N, K, planes); one launch for all."""
    arr = (_RansItem * len(entries))()
    for i, (freq, row_end, payload, N, K, planes) in enumerate(entries):
        arr[i].freq_dev, arr[i].row_end_dev, arr[i].payload_dev = _ptr(freq), _ptr(row_end), _ptr(payload)
        arr[i].payload_bytes = int(payload.numel() * payload.element_size())
        arr[i].N, arr[i].K, arr[i].planes_dev = int(N), int(K), _ptr(planes)
    _check(lib().tern_rans_decode(arr, len(entries), _ptr(err_flag), _stream(stream)), "tern_rans_decode")


def tern_read_flag(err_flag, stream=None) -> int:
    """Synchronise the stream and return TERN_OK or TERN_EBADCODE from a device error flag."""
    st = lib().tern_read_flag(_ptr(err_flag), _stream(stream))
    if st not in (TERN_OK, TERN_EBADCODE):
        raise TernError(st, "tern_read_flag")
    return st


def tern_device_status(stream=None) -> int:
    """Synchronise and return TERN_OK, or TERN_ETIMEOUT if a kernel gave up a bounded wait."""
    return int(lib().tern_device_status(_stream(stream)))


def _items(entries):
    arr = (_Item * len(entries))()
    for i, (W, x, x_scale, y) in enumerate(entries):
        arr[i].W = W._c
        arr[i].x_dev = _ptr(x)
        arr[i].x_scale_dev = _ptr(x_scale)
        arr[i].y_dev = _ptr(y)
    return arr


def tern_gemv_batch_workspace_bytes(entries, act: int) -> int:
    """entries: list of (TernMatrix, x, x_scale or None, y)."""
    arr = _items(entries)
    return int(lib().tern_gemv_batch_workspace_bytes(arr, len(entries), act))


def tern_gemv_batch(entries, act: int, workspace, flags: int = 0, stream=None) -> None:
    arr = _items(entries)
    _check(lib().tern_gemv_batch(arr, len(entries), act, _ptr(workspace),
                                 int(workspace.numel() * workspace.element_size()), flags, _stream(stream)),
           "tern_gemv_batch")


def tern_gemm_batch_workspace_bytes(entries, M: int, act: int) -> int:
    """entries: list of (TernMatrix, X [M][K], x_scale [M] or None, Y [M][N])."""
    arr = _items(entries)
    return int(lib().tern_gemm_batch_workspace_bytes(arr, len(entries), M, act))


def tern_gemm_batch(entries, M: int, act: int, workspace, flags: int = 0, stream=None) -> None:
    arr = _items(entries)
    _check(lib().tern_gemm_batch(arr, len(entries), M, act, _ptr(workspace),
                                 int(workspace.numel() * workspace.element_size()), flags, _stream(stream)),
           "tern_gemm_batch")


def tern_gemm_batch_pro(entries, prologues, M: int, act: int, workspace, flags: int = 0, stream=None) -> None:
    """tern_gemm_batch with a prologue per entry: prologues[i] is None or (kind, src, gain, eps); for a
    prologue entry, X is an optional output (or None) and x_scale (int8 mode) the output s_x."""
    arr, pro = _items(entries), _prologues(prologues)
    _check(lib().tern_gemm_batch_pro(arr, pro, len(entries), M, act, _ptr(workspace),
                                     int(workspace.numel() * workspace.element_size()), flags, _stream(stream)),
           "tern_gemm_batch_pro")


def tern_act_prologue(kind: int, src, gain, eps: float, M: int, K: int, out, stream=None) -> None:
    """The prologue alone: M rows of K bf16 activations (bit patterns) into out."""
    pro = _prologues([(kind, src, gain, eps)])
    _check(lib().tern_act_prologue(pro, M, K, _ptr(out), _stream(stream)), "tern_act_prologue")


class GemvBatch:
    """A fixed list of GEMVs (M = 1) or small-M GEMMs with its descriptor array and workspace,
    launched repeatedly (e.g. inside a captured CUDA graph). entries: list of (TernMatrix, X,
    x_scale or None, Y) with X [M][K] and Y [M][N]; prologues: optional list (one per entry) of
    None or (kind, src, gain, eps), see tern_gemm_batch_pro."""

    def __init__(self, entries, act: int, M: int = 1, device="cuda", prologues=None):
        import torch
        self.entries, self.act, self.M = list(entries), act, int(M)
        self._arr = _items(self.entries)
        self._pro = _prologues(prologues) if prologues is not None else None
        nbytes = int(lib().tern_gemm_batch_workspace_bytes(self._arr, len(self.entries), self.M, act))
        if nbytes == 0:
            raise TernError(TERN_ESHAPE, "tern_gemm_batch_workspace_bytes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def __call__(self, flags: int = 0, stream=None) -> None:
        if self._pro is not None:
            _check(lib().tern_gemm_batch_pro(self._arr, self._pro, len(self.entries), self.M, self.act,
                                             _ptr(self.workspace), int(self.workspace.numel()), flags,
                                             _stream(stream)), "tern_gemm_batch_pro")
            return
        _check(lib().tern_gemm_batch(self._arr, len(self.entries), self.M, self.act, _ptr(self.workspace),
                                     int(self.workspace.numel()), flags, _stream(stream)), "tern_gemm_batch")
