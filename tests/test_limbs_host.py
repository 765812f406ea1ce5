"""Host checks of the exact three-limb encoding behind the bf16 activation mode (no GPU).

The bf16 paths split each activation x into X = rint(x * 2^(22 - E)), E the exponent of the
absmax (absmax < 2^E), and X into three int8 limbs L2, L1, L0 with X = L2 * 2^16 + L1 * 2^8 + L0.
These tests check, over every finite bf16 bit pattern, that the split reconstructs X, that
|L2| <= 64 (so every limb is a valid s8 tensor-core operand), and that X is exactly x * 2^(22 - E)
whenever |x| >= 2^(E - 15): the bf16 mantissa has 8 significant bits, so such an x is an integer
multiple of 2^(E - 22)."""
import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _all_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32)
    x = (bits << 16).view(np.float32).astype(np.float64)
    return x[np.isfinite(x)]


def _split(X):
    L0 = ((X & 0xFF) ^ 0x80) - 0x80                      # sign-extended low byte
    X1 = (X - L0) >> 8
    L1 = ((X1 & 0xFF) ^ 0x80) - 0x80
    L2 = (X1 - L1) >> 8
    return L2, L1, L0


@pytest.mark.parametrize("E", [-20, -3, 0, 1, 2, 3, 7, 40])
def test_limbs_reconstruct_and_fit(E):
    x = _all_bf16()
    x = x[np.abs(x) < 2.0 ** E]                         # the item's absmax is below 2^E
    X = np.rint(x * 2.0 ** (22 - E)).astype(np.int64)   # round half to even, like the kernels
    assert np.abs(X).max() <= 2 ** 22
    L2, L1, L0 = _split(X)
    assert (L2 * 65536 + L1 * 256 + L0 == X).all()
    for L in (L1, L0):
        assert L.min() >= -128 and L.max() <= 127
    assert np.abs(L2).max() <= 64


@pytest.mark.parametrize("E", [-3, 0, 2, 7])
def test_limbs_exact_above_the_cut(E):
    x = _all_bf16()
    x = x[(np.abs(x) < 2.0 ** E) & (np.abs(x) >= 2.0 ** (E - 15))]
    scaled = x * 2.0 ** (22 - E)                        # exact in fp64 (a power-of-two scaling)
    assert (scaled == np.rint(scaled)).all()            # already an integer: no rounding happens


def test_limbs_round_below_the_cut():
    """Values below 2^(E - 15) do round (the documented bound), by at most half a unit of 2^(E - 22)."""
    E = 2
    x = _all_bf16()
    x = x[(np.abs(x) < 2.0 ** (E - 15)) & (x != 0)]
    scaled = x * 2.0 ** (22 - E)
    err = np.abs(np.rint(scaled) - scaled)
    assert err.max() <= 0.5 and (err > 0).any()
