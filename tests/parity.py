"""Comparison of GPU outputs with the oracle under the stated tolerance rule.

Tolerance (the quantizer's stated bar, read componentwise):

* a transformed value may differ from the oracle's float64 value by at most
  ``TOL * (|x| |K|)_c`` -- ``TOL`` times the sum of the magnitudes of the
  terms it is made of, which is also an upper bound of ``|y_c|``;
* scale bytes and E2M1 codes must be bit-exact, except where the exact value
  lies within that band of a rounding boundary (an E2M1 midpoint after
  scaling, or a power of two for the block maximum).  There the GPU may take
  either side: a scale byte within the range the band allows, and a code
  between the codes of the band's two ends (one code step for any band this
  narrow);
* an element whose exact transformed value is zero may carry either sign
  when it comes from a sum (``strict_zero_sign=False``); a single product
  (the SmoothQuant comparator) keeps the sign of its input.

The helpers only compare; no value computed here is fed to the oracle.
"""
from __future__ import annotations

import numpy as np

from oracle import kq_oracle as o

TOL = 1e-5


def unpack(q: np.ndarray) -> np.ndarray:
    q = np.asarray(q, dtype=np.uint8)
    out = np.empty(q.shape[:-1] + (2 * q.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = q & 15
    out[..., 1::2] = q >> 4
    return out


def _signed_value(codes):
    mag = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])[codes & 7]
    return np.where(codes & 8, -mag, mag)


def check_transform(y_gpu: np.ndarray, y64: np.ndarray, cond: np.ndarray, tol: float = TOL):
    """Elementwise |y_gpu - y64| <= tol * cond.  Returns the worst ratio."""
    err = np.abs(np.asarray(y_gpu, dtype=np.float64) - y64)
    bound = tol * cond
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        detail = [(tuple(i), float(y_gpu[tuple(i)]), float(y64[tuple(i)]), float(cond[tuple(i)]))
                  for i in idx]
        raise AssertionError(f"{int(bad.sum())} transformed values outside tolerance: {detail}")
    with np.errstate(invalid="ignore", divide="ignore"):
        r = np.where(cond > 0, err / np.where(cond > 0, cond, 1), 0)
    return float(r.max()) if r.size else 0.0


def check_mx4(q_gpu, s_gpu, y64, cond, tol: float = TOL, strict_zero_sign: bool = False,
              block: int = 32):
    """Check packed codes and scale bytes against the oracle's quantization of
    ``y64`` (decided in float32), one scale per ``block`` elements.  Returns
    exemption counts."""
    y64 = np.asarray(y64, dtype=np.float64)
    M, d = y64.shape
    nb = d // block
    s_gpu = np.asarray(s_gpu, dtype=np.uint8).reshape(M, nb)
    c_gpu = unpack(q_gpu).reshape(M, d)
    codes_ref, s_ref = o.mxfp4_quantize(y64, block)

    yq = o.decision_values(y64)
    band = tol * np.asarray(cond, dtype=np.float64)
    blk = np.abs(yq).reshape(M, nb, block)
    bblk = band.reshape(M, nb, block)
    amax_lo = np.maximum(blk - bblk, 0).max(axis=2)
    amax_hi = (blk + bblk).max(axis=2)
    e_lo = o.e8m0_exponent(amax_lo) + 127
    e_hi = o.e8m0_exponent(amax_hi) + 127
    s_int = s_gpu.astype(np.int64)
    scale_ok = (s_int == s_ref) | ((s_int >= e_lo) & (s_int <= e_hi))
    if not scale_ok.all():
        idx = np.argwhere(~scale_ok)[:5]
        raise AssertionError(
            f"{int((~scale_ok).sum())} scale bytes differ: "
            f"{[(tuple(i), int(s_gpu[tuple(i)]), int(s_ref[tuple(i)])) for i in idx]}")

    # Codes under the scale the GPU chose (one of the allowed ones).
    X = np.repeat(np.ldexp(1.0, s_int - 127), block, axis=1)
    v = yq / X
    vb = band / X
    lo = _signed_value(o.e2m1_encode(v - vb))
    hi = _signed_value(o.e2m1_encode(v + vb))
    got = _signed_value(c_gpu)
    ok = (got >= lo) & (got <= hi)
    # Sign of zero codes: decided by the oracle's code where the band does not
    # reach zero, free where it does (or where the exact value is a zero sum).
    zero_gpu = (c_gpu & 7) == 0
    ref_same_scale = o.e2m1_encode(v)
    sign_must = ~((vb > 0) & (v - vb <= 0) & (v + vb >= 0))
    if not strict_zero_sign:
        sign_must &= y64 != 0
    sign_bad = zero_gpu & sign_must & ((c_gpu & 8) != (ref_same_scale & 8))
    ok &= ~sign_bad
    if not ok.all():
        idx = np.argwhere(~ok)[:8]
        raise AssertionError(
            f"{int((~ok).sum())} codes outside the allowed set: " + str(
                [(tuple(i), int(c_gpu[tuple(i)]), int(codes_ref[tuple(i)]), float(v[tuple(i)]),
                  float(vb[tuple(i)])) for i in idx]))
    differ = c_gpu != codes_ref
    zero_sign = differ & ((c_gpu & 7) == 0) & ((codes_ref & 7) == 0)
    return {
        "scale_exempt": int((s_int != s_ref).sum()),
        "code_exempt": int((differ & ~zero_sign).sum()),
        "zero_sign_exempt": int(zero_sign.sum()),
        "blocks": int(M * nb),
        "elements": int(M * d),
    }
