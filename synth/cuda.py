"""ctypes access to the device-side input generator (synth/libternsynth.so).

Fills caller-owned device buffers (torch tensors) with the same trits and int8 head weights that
synth.trits / synth.head_weights return on the host, bit for bit.
"""
from __future__ import annotations

import ctypes
import os

from . import KIND_HEAD, KIND_TRIT, P_DEFAULT, stream_key, thresholds

_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libternsynth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python synth/build.py`")
        L = ctypes.CDLL(path)
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        L.synth_trits.argtypes = [u64, u64, u64, i64, i64, i64, vp, vp]
        L.synth_trits.restype = ctypes.c_int
        L.synth_head.argtypes = [u64, i64, i64, i64, vp, vp]
        L.synth_head.restype = ctypes.c_int
        _LIB = L
    return _LIB


def _stream_ptr(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def trits_into(out, seed: int, tid: int, K: int, p=P_DEFAULT, row0: int = 0, stream=None) -> None:
    """out: int8 CUDA tensor with numel = N*K (rows row0..row0+N-1 of tensor tid)."""
    N = out.numel() // K
    t0, t1 = thresholds(p)
    rc = lib().synth_trits(stream_key(seed, KIND_TRIT, tid), t0, t1, N, K, row0, out.data_ptr(),
                           _stream_ptr(stream))
    if rc != 0:
        raise RuntimeError(f"synth_trits failed ({rc})")


def head_into(out, seed: int, tid: int, K: int, row0: int = 0, stream=None) -> None:
    V = out.numel() // K
    rc = lib().synth_head(stream_key(seed, KIND_HEAD, tid), V, K, row0, out.data_ptr(), _stream_ptr(stream))
    if rc != 0:
        raise RuntimeError(f"synth_head failed ({rc})")
