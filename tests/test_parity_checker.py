"""The tolerance checker accepts the oracle's own outputs and rejects planted
mistakes (planted on the CPU, in copies of the oracle's outputs)."""
import numpy as np
import pytest

import workloads as w
from oracle import kq_oracle as o
from tests.parity import check_mx4, check_transform, check_transform_literal, relative_outside


@pytest.fixture(scope="module")
def case():
    c = w.make_case("stress", M=24)
    x64 = o.bf16_bits_to_float64(c.x_bits())
    y64 = o.transform(x64, c.params)
    cond = o.abs_transform(x64, c.params)
    q, s = o.quantize(c.x_bits(), c.params)
    return y64, cond, q, s


def test_oracle_outputs_pass_with_no_exemption(case):
    y64, cond, q, s = case
    st = check_mx4(q, s, y64, cond)
    assert st["scale_exempt"] == 0 and st["code_exempt"] == 0
    assert check_transform(y64.astype(np.float32), y64, cond) < 1e-6


def test_a_code_two_steps_off_fails(case):
    y64, cond, q, s = case
    codes = o.unpack_codes(q)
    i = np.argmax((codes & 7) == 3)
    r, c = divmod(int(i), codes.shape[1])
    codes[r, c] = (codes[r, c] & 8) | 5
    with pytest.raises(AssertionError):
        check_mx4(o.pack_codes(codes), s, y64, cond)


def test_a_wrong_scale_fails(case):
    y64, cond, q, s = case
    s2 = s.copy()
    s2[3, 7] += 1
    with pytest.raises(AssertionError):
        check_mx4(q, s2, y64, cond)


def test_swapped_nibbles_fail(case):
    y64, cond, q, s = case
    q2 = ((q >> 4) | (q << 4)).astype(np.uint8)
    with pytest.raises(AssertionError):
        check_mx4(q2, s, y64, cond)


def test_a_flipped_zero_sign_fails_for_products():
    y = np.zeros((1, 32))
    y[0, 0] = 4.0
    y[0, 1] = -0.01
    q, s = o.pack_codes(o.mxfp4_quantize(y)[0]), o.mxfp4_quantize(y)[1]
    codes = o.unpack_codes(q)
    codes[0, 1] = 0
    with pytest.raises(AssertionError):
        check_mx4(o.pack_codes(codes), s, y, np.zeros_like(y), strict_zero_sign=True)


def test_transform_error_beyond_tolerance_fails(case):
    y64, cond, q, s = case
    bad = y64.copy()
    bad[2, 5] += 2e-5 * cond[2, 5]
    with pytest.raises(AssertionError):
        check_transform(bad, y64, cond)


def test_literal_band_counts():
    """A code that differs where its scaled value sits on an E2M1 midpoint is
    inside the literal band; one that differs only because the componentwise
    band is wide (cancelling terms) is counted outside it; so is a scale byte
    that differs away from a power of two."""
    y = np.zeros((1, 64))
    y[0, 0] = 4.0            # block 0: scale 2^0, unit steps
    y[0, 1] = 1.25           # an exact midpoint between 1 and 1.5
    y[0, 2] = 2.2            # far from every midpoint
    y[0, 32] = 3.0           # block 1: amax 3, away from a power of two
    codes, s = o.mxfp4_quantize(y)
    cond = np.zeros_like(y)
    cond[0, 1] = 1.0
    cond[0, 2] = 1e5         # a cancelling sum: wide componentwise band
    cond[0, 32] = 1e5
    got = codes.copy()
    got[0, 1] = 3            # 1.5 instead of the even 1.0: on the midpoint
    got[0, 2] = 5            # 3.0 instead of 2.0: allowed by the wide band only
    st = check_mx4(o.pack_codes(got), s, y, cond)
    assert st["code_differs_under_gpu_scale"] == 2
    assert st["code_outside_literal"] == 1
    s2 = s.copy()
    s2[0, 1] += 1            # block 1 at twice the scale: 3.0 is coded as 3 (code 5), not 6
    got = codes.copy()
    got[0, 32] = 5
    st = check_mx4(o.pack_codes(got), s2, y, cond)
    assert st["scale_exempt"] == 1 and st["scale_outside_literal"] == 1


def test_relative_outside_counts_cancelling_entries():
    y64 = np.array([[1.0, 1e-9, -2.0]])
    y_gpu = y64 + np.array([[1e-7, 1e-7, 0.0]])
    assert relative_outside(y_gpu, y64) == 1


def test_literal_transform_check():
    """The literal reading passes values within 1e-5 of themselves and a
    double-precision residue where the oracle's sum is exactly zero, and
    fails a cancelling entry that only the componentwise band would pass."""
    y64 = np.array([[1.0, -2.0, 0.0, 1e-3]])
    cond = np.array([[3.0, 4.0, 5.0, 10.0]])
    ok = y64 * (1 + 5e-6)
    ok[0, 2] = 1e-16                        # residue of an exact cancellation
    assert check_transform_literal(ok, y64, cond) <= 5e-6 * 1.0001
    bad = y64.copy()
    bad[0, 3] = 1e-3 * (1 + 1e-3)           # 1e-6 of the terms, 1e-3 of the value
    assert check_transform(bad, y64, cond) < 1e-5
    with pytest.raises(AssertionError):
        check_transform_literal(bad, y64, cond)
    # A float32 subnormal output is within one subnormal step of the value.
    tiny = np.array([[5.1000693571781566e-43]])
    assert check_transform_literal(np.float32(tiny).astype(np.float64), tiny, tiny * 1e6) == 0.0
