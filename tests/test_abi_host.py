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
    assert L.tern_gemv(ctypes.byref(m), 0, fake, None, fake, None, None) == tg.TERN_ESHAPE
    m = tg._Matrix(64, 128, None, fake)
    assert L.tern_gemv(ctypes.byref(m), 0, fake, None, fake, None, None) == tg.TERN_EINVAL
    m = tg._Matrix(64, 128, fake, fake)
    assert L.tern_gemv(ctypes.byref(m), 7, fake, None, fake, None, None) == tg.TERN_EINVAL        # bad act
    assert L.tern_gemv(ctypes.byref(m), 1, fake, None, fake, None, None) == tg.TERN_EINVAL        # int8 needs s_x
    assert L.tern_gemv(ctypes.byref(m), 0, fake + 4, None, fake, None, None) == tg.TERN_EINVAL    # misaligned x
    assert L.tern_gemv(ctypes.byref(m), 0, fake, None, fake, fake, None) == tg.TERN_EINVAL        # acc in bf16 mode
    assert L.tern_gemv(ctypes.byref(m), 1, fake, fake, fake, fake + 2, None) == tg.TERN_EINVAL    # misaligned acc
    assert L.tern_gemm_small_m(ctypes.byref(m), 17, 0, fake, None, fake, None) == tg.TERN_ESHAPE
    assert L.tern_gemm_small_m(ctypes.byref(m), 0, 0, fake, None, fake, None) == tg.TERN_ESHAPE
    assert L.tern_gemv_ex(ctypes.byref(m), 0, fake, None, fake, None, 8, None) == tg.TERN_EINVAL   # unknown flag
    assert L.tern_pack(0, fake, 4, 96, fake, fake, None) == tg.TERN_ESHAPE
    assert L.tern_pack(5, fake, 4, 128, fake, fake, None) == tg.TERN_EINVAL
    assert L.tern_pack(0, fake, 4, 128, fake, None, None) == tg.TERN_EINVAL
    assert L.i8_head_gemv_argmax(fake, fake, 1000, 1024, 1, 0, fake, None, fake, fake, None, fake, 8, None) \
        == tg.TERN_EINVAL                                                                      # workspace too small
    assert L.i8_head_gemv_argmax(fake, fake, 1000, 1000, 1, 0, fake, None, fake, fake, None, fake, 256, None) \
        == tg.TERN_ESHAPE
    assert L.tern_quantize_act(fake, 0, 128, fake, fake, None) == tg.TERN_ESHAPE
    assert "TERN_ESHAPE" in tg.tern_status_string(tg.TERN_ESHAPE)


def test_list_and_prefill_argument_errors_before_launch(L):
    """tern_gemm_batch, tern_pack_batch and tern_gemm_prefill reject bad arguments before they
    encode a tensor map or launch anything."""
    import bit_gemv_tern_b200 as tg
    fake = 1 << 40
    ws = fake                                           # 16-byte aligned, never dereferenced
    m = tg._Matrix(256, 4096, fake, fake)
    items = (tg._Item * 2)()
    for it in items:
        it.W, it.x_dev, it.x_scale_dev, it.y_dev = m, fake, None, fake
    assert L.tern_gemm_batch(items, 2, 17, 0, ws, 1 << 20, 0, None) == tg.TERN_ESHAPE          # M > 16
    assert L.tern_gemm_batch(items, 2, 0, 0, ws, 1 << 20, 0, None) == tg.TERN_ESHAPE           # M < 1
    assert L.tern_gemm_batch(items, 0, 1, 0, ws, 1 << 20, 0, None) == tg.TERN_ESHAPE           # empty list
    assert L.tern_gemm_batch(items, 161, 1, 0, ws, 1 << 20, 0, None) == tg.TERN_ESHAPE         # > 160 items
    assert L.tern_gemm_batch(None, 2, 1, 0, ws, 1 << 20, 0, None) == tg.TERN_EINVAL
    assert L.tern_gemm_batch(items, 2, 1, 9, ws, 1 << 20, 0, None) == tg.TERN_EINVAL           # bad act
    assert L.tern_gemm_batch(items, 2, 1, 1, ws, 1 << 20, 0, None) == tg.TERN_EINVAL           # int8 needs s_x
    assert L.tern_gemm_batch(items, 2, 1, 0, ws + 8, 1 << 20, 0, None) == tg.TERN_EINVAL       # misaligned ws
    assert L.tern_gemm_batch(items, 2, 1, 0, ws, 1 << 20, 4, None) == tg.TERN_EINVAL           # unknown flag
    items[1].W = tg._Matrix(256, 16384, fake, fake)                                          # K > 12288
    assert L.tern_gemm_batch(items, 2, 1, 0, ws, 1 << 20, 0, None) == tg.TERN_ESHAPE
    items[1].W = m
    items[1].x_dev = fake + 4                                                                # misaligned x
    assert L.tern_gemm_batch(items, 2, 1, 0, ws, 1 << 20, 0, None) == tg.TERN_EINVAL

    packs = (tg._PackItem * 2)()
    for p in packs:
        p.src_dev, p.N, p.K, p.planes_dev = fake, 64, 128, fake
    flag = fake
    assert L.tern_pack_batch(0, packs, 0, flag, None) == tg.TERN_ESHAPE                         # empty list
    assert L.tern_pack_batch(0, packs, 257, flag, None) == tg.TERN_ESHAPE                       # > 256 items
    assert L.tern_pack_batch(4, packs, 2, flag, None) == tg.TERN_EINVAL                         # bad source kind
    assert L.tern_pack_batch(0, packs, 2, None, None) == tg.TERN_EINVAL                         # no flag
    assert L.tern_pack_batch(0, None, 2, flag, None) == tg.TERN_EINVAL
    packs[1].K = 96                                                                          # K % 128 != 0
    assert L.tern_pack_batch(0, packs, 2, flag, None) == tg.TERN_ESHAPE
    packs[1].K, packs[1].planes_dev = 128, fake + 4                                           # misaligned planes
    assert L.tern_pack_batch(0, packs, 2, flag, None) == tg.TERN_EINVAL
    packs[1].planes_dev, packs[1].src_dev = fake, fake + 4                                    # base-3 src: 4-aligned is fine,
    assert L.tern_pack_batch(0, packs, 2, flag, None) == tg.TERN_EINVAL                        # int8 src needs 16

    assert L.tern_gemm_prefill(ctypes.byref(m), 0, fake, fake, None) == tg.TERN_ESHAPE          # M < 1
    assert L.tern_gemm_prefill(ctypes.byref(m), 65537, fake, fake, None) == tg.TERN_ESHAPE      # M > 65536
    assert L.tern_gemm_prefill(ctypes.byref(m), 128, fake + 8, fake, None) == tg.TERN_EINVAL    # misaligned X
    assert L.tern_gemm_prefill(ctypes.byref(m), 128, fake, fake + 2, None) == tg.TERN_EINVAL    # misaligned Y
    assert L.tern_gemm_prefill(ctypes.byref(m), 128, None, fake, None) == tg.TERN_EINVAL


def test_fv5_batch_argument_errors_before_launch(L):
    """tern_fv5_gemv_batch rejects a bad list before it plans or launches anything."""
    import bit_gemv_tern_b200 as tg
    fake = 1 << 40                                      # never dereferenced: validation fails first
    items = (tg._Fv5BatchItem * 2)()
    for it in items:
        it.W = tg._Fv5Matrix(64, 4096, fake, fake)
        it.x, it.x_scale, it.y = fake, None, fake
    assert L.tern_fv5_gemv_batch(None, 2, 0, None) == tg.TERN_EINVAL
    assert L.tern_fv5_gemv_batch(items, 0, 0, None) == tg.TERN_ESHAPE                  # empty list
    assert L.tern_fv5_gemv_batch(items, 161, 0, None) == tg.TERN_ESHAPE                # > 160 items
    assert L.tern_fv5_gemv_batch(items, 2, 9, None) == tg.TERN_EINVAL                  # bad act
    assert L.tern_fv5_gemv_batch(items, 2, 1, None) == tg.TERN_EINVAL                  # int8 needs x_scale
    for bad in ((64, 4000), (64, 12800), (0, 4096)):                                   # K % 512, K > 12288, N < 1
        items[1].W = tg._Fv5Matrix(bad[0], bad[1], fake, fake)
        assert L.tern_fv5_gemv_batch(items, 2, 0, None) == tg.TERN_ESHAPE, bad
    items[1].W = tg._Fv5Matrix(64, 4096, fake + 4, fake)                               # planes not 16-aligned
    assert L.tern_fv5_gemv_batch(items, 2, 0, None) == tg.TERN_EINVAL
    items[1].W = tg._Fv5Matrix(64, 4096, fake, fake)
    items[1].x = fake + 4                                                              # x not 16-aligned
    assert L.tern_fv5_gemv_batch(items, 2, 0, None) == tg.TERN_EINVAL
    items[1].x, items[1].y = fake, None                                                # no output
    assert L.tern_fv5_gemv_batch(items, 2, 0, None) == tg.TERN_EINVAL
