"""The tolerance checker accepts the oracle's own outputs and rejects planted
mistakes (planted on the CPU, in copies of the oracle's outputs)."""
import numpy as np
import pytest

import workloads as w
from oracle import kq_oracle as o
from tests.parity import check_mx4, check_transform


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
