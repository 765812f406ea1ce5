"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function that
include/tern.h declares, sizes are computed right, and invalid arguments are rejected before
anything is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from bit_gemv_tern_b200 import build
    build.build()
    import bit_gemv_tern_b200 as tg
    return tg.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "tern.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = "\n".join(l for l in src.splitlines() if not l.lstrip().startswith("#"))
    return sorted(set(re.findall(r"\b(\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert "tern_gemv" in names and "i8_head_gemv_argmax" in names and len(names) >= 15
    for n in names:
        assert hasattr(L, n), n


def test_sizes(L):
    import bit_gemv_tern_b200 as tg
    assert tg.tern_packed_bytes(4096, 4096) == 4096 * 4096 // 4
    assert tg.tern_packed_bytes(4096, 100) == 0 and tg.tern_packed_bytes(0, 128) == 0
    assert tg.tern_base3_bytes(4096, 12288) == 4096 * 2458
    assert tg.i8_head_workspace_bytes(151936, 16) >= 16 + 8 * 16
    assert tg.i8_head_workspace_bytes(151936, 17) == 0


def test_argument_errors_before_launch(L):
    import bit_gemv_tern_b200 as tg
    fake = 1 << 40                      # never dereferenced: validation fails first
    m = tg._Matrix(64, 100, fake, fake)  # K % 128 != 0
    assert L.tern_gemv(ctypes.byref(m), 0, fake, None, fake, None) == tg.TERN_ESHAPE
    m = tg._Matrix(64, 128, None, fake)
    assert L.tern_gemv(ctypes.byref(m), 0, fake, None, fake, None) == tg.TERN_EINVAL
    m = tg._Matrix(64, 128, fake, fake)
    assert L.tern_gemv(ctypes.byref(m), 7, fake, None, fake, None) == tg.TERN_EINVAL        # bad act
    assert L.tern_gemv(ctypes.byref(m), 1, fake, None, fake, None) == tg.TERN_EINVAL        # int8 needs s_x
    assert L.tern_gemv(ctypes.byref(m), 0, fake + 4, None, fake, None) == tg.TERN_EINVAL    # misaligned x
    assert L.tern_gemm_small_m(ctypes.byref(m), 17, 0, fake, None, fake, None) == tg.TERN_ESHAPE
    assert L.tern_gemm_small_m(ctypes.byref(m), 0, 0, fake, None, fake, None) == tg.TERN_ESHAPE
    assert L.tern_gemv_ex(ctypes.byref(m), 0, fake, None, fake, 8, None) == tg.TERN_EINVAL   # unknown flag
    assert L.tern_pack(0, fake, 4, 96, fake, fake, None) == tg.TERN_ESHAPE
    assert L.tern_pack(5, fake, 4, 128, fake, fake, None) == tg.TERN_EINVAL
    assert L.tern_pack(0, fake, 4, 128, fake, None, None) == tg.TERN_EINVAL
    assert L.i8_head_gemv_argmax(fake, fake, 1000, 1024, 1, 0, fake, None, fake, fake, None, fake, 8, None) \
        == tg.TERN_EINVAL                                                                      # workspace too small
    assert L.i8_head_gemv_argmax(fake, fake, 1000, 1000, 1, 0, fake, None, fake, fake, None, fake, 256, None) \
        == tg.TERN_ESHAPE
    assert L.tern_quantize_act(fake, 0, 128, fake, fake, None) == tg.TERN_ESHAPE
    assert "TERN_ESHAPE" in tg.tern_status_string(tg.TERN_ESHAPE)
