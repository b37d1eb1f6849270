"""The quantizer's reciprocal against the IEEE reciprocal, on the GPU, through the C ABI.

Quantize forms each row's r = RN(1/scale) from the hardware's approximate
reciprocal refined by one Newton-Raphson step in fused multiply-adds, and the
exactness of its codes rests on r being exactly the IEEE round-to-nearest
reciprocal (Markstein's correction of the quotient needs it).
semkv_check_reciprocal compares the two bit for bit over every float of the
given exponent fields.  Fields 1 .. 252 (b in [2^-126, 2^126), 2.1e9 values)
hold every scale a row can have (2^-28 .. 2^25).
"""
import pytest

from tests.gpu_common import kv_mod

pytestmark = pytest.mark.gpu


def test_reciprocal_is_ieee_for_every_normal_with_a_normal_reciprocal():
    kv = kv_mod()
    assert kv.semkv_check_reciprocal(1, 252) == 0


def test_reciprocal_check_is_not_vacuous():
    # above 2^126 the IEEE reciprocal is subnormal and the approximation flushes
    # it to zero, so the check must count those values
    kv = kv_mod()
    assert kv.semkv_check_reciprocal(253, 254) > 0


@pytest.mark.parametrize("lo,hi", [(0, 10), (10, 255), (20, 10)])
def test_reciprocal_check_rejects_bad_ranges(lo, hi):
    kv = kv_mod()
    with pytest.raises(kv.SemkvError):
        kv.semkv_check_reciprocal(lo, hi)
