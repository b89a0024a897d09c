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
# E2M1 rounding boundaries: midpoints of neighbouring grid magnitudes.
MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


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
    # The literal reading of the rule, counted beside the componentwise one:
    # a differing scale byte whose block maximum is not within tol relative
    # of a power of two, and a differing code (against the oracle's code
    # under the scale the GPU chose) whose scaled value is not within tol
    # relative of an E2M1 midpoint.
    amax_ref = blk.max(axis=2)
    with np.errstate(divide="ignore"):
        p2 = np.ldexp(1.0, np.round(np.log2(np.where(amax_ref > 0, amax_ref, 1.0))).astype(np.int64))
    scale_lit = np.abs(amax_ref - p2) <= tol * p2
    s_diff = s_int != s_ref
    code_diff = (c_gpu != ref_same_scale) & ~(((c_gpu & 7) == 0) & ((ref_same_scale & 7) == 0))
    av = np.abs(v)
    near_mid = np.zeros(av.shape, dtype=bool)
    for mid in MIDPOINTS:
        near_mid |= np.abs(av - mid) <= tol * mid
    return {
        "scale_exempt": int(s_diff.sum()),
        "code_exempt": int((differ & ~zero_sign).sum()),
        "zero_sign_exempt": int(zero_sign.sum()),
        # a zero code of the other sign where the exact value is not zero
        "zero_sign_outside_literal": int((zero_sign & (y64 != 0)).sum()),
        "scale_outside_literal": int((s_diff & ~scale_lit).sum()),
        "code_differs_under_gpu_scale": int(code_diff.sum()),
        "code_outside_literal": int((code_diff & ~near_mid).sum()),
        "blocks": int(M * nb),
        "elements": int(M * d),
    }


# Absolute floors of the literal check: relative to the terms' magnitudes,
# because a sum the oracle cancels to exactly zero may come out as a residue
# of the double-precision rounding of its terms (about 1e-16 of them); and
# one float32 subnormal step, below which no float32 output can be relatively
# accurate.
LITERAL_FLOOR = 1e-12
F32_SUBNORMAL_STEP = 2.0 ** -149


def relative_outside(y_gpu: np.ndarray, y64: np.ndarray, tol: float = TOL,
                     cond: np.ndarray = None) -> int:
    """Entries with |y_gpu - y64| > tol |y64| (+ LITERAL_FLOOR cond when the
    terms' magnitudes are given): those that pass the componentwise bound
    only because their terms cancel."""
    err = np.abs(np.asarray(y_gpu, dtype=np.float64) - y64)
    bound = tol * np.abs(y64) + F32_SUBNORMAL_STEP
    if cond is not None:
        bound = bound + LITERAL_FLOOR * cond
    return int((err > bound).sum())


def check_transform_literal(y_gpu: np.ndarray, y64: np.ndarray, cond: np.ndarray,
                            tol: float = TOL) -> float:
    """The literal reading of the transform tolerance: every float32 value
    within tol of the oracle's value relative to that value itself (up to
    LITERAL_FLOOR of the terms' magnitudes and one float32 subnormal step),
    on top of the componentwise band.  Returns the worst
    |y_gpu - y64| / |y64| over entries that are normal float32 values."""
    check_transform(y_gpu, y64, cond, tol)
    n = relative_outside(y_gpu, y64, tol, cond)
    if n:
        err = np.abs(np.asarray(y_gpu, dtype=np.float64) - y64)
        bad = np.argwhere(err > tol * np.abs(y64) + LITERAL_FLOOR * cond + F32_SUBNORMAL_STEP)[:5]
        detail = [(tuple(i), float(y_gpu[tuple(i)]), float(y64[tuple(i)])) for i in bad]
        raise AssertionError(f"{n} transformed values outside {tol} relative: {detail}")
    err = np.abs(np.asarray(y_gpu, dtype=np.float64) - y64)
    nz = np.abs(y64) >= 2.0 ** -126
    return float((err[nz] / np.abs(y64[nz])).max()) if nz.any() else 0.0


def merge_stats(total: dict, part: dict) -> dict:
    """Adds one chunk's counts to a running total (worst ratios take the max)."""
    for k, v in part.items():
        if k.startswith("worst"):
            total[k] = max(total.get(k, 0.0), v)
        else:
            total[k] = total.get(k, 0) + v
    return total


def check_chunk(job):
    """Compares one row chunk of the GPU's outputs with the oracle; runs in a
    spawned worker (numpy only).  ``job`` = (kind, x_bits, aux, outputs):
    kind "kron" (aux = params; outputs q, s, y), "hadamard" (q, s) or
    "smooth" (aux = inv_s; q, s).  Returns the chunk's counts."""
    kind, bits, aux, out = job
    x64 = o.bf16_bits_to_float64(bits)
    if kind == "kron":
        y64 = o.transform(x64, aux)
        cond = o.abs_transform(x64, aux)
        st = {"worst_transform_ratio": check_transform(out["y"], y64, cond),
              "transform_outside_relative": relative_outside(out["y"], y64, cond=cond)}
        st.update(check_mx4(out["q"], out["s"], y64, cond))
    elif kind == "hadamard":
        y64 = o.transform_hadamard(x64)
        st = check_mx4(out["q"], out["s"], y64, o.abs_transform_hadamard(x64))
    else:
        y64 = o.transform_smooth(x64, aux)
        st = check_mx4(out["q"], out["s"], y64, np.zeros_like(y64), strict_zero_sign=True)
    return st
