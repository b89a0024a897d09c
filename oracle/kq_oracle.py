"""CPU oracle for the KroQuant online activation quantizer (float64, numpy).

TEST INFRASTRUCTURE ONLY.  This module is the checker the GPU path is compared
against.  Only the test-suite, the package's smoke check and the CPU-baseline
leg of the benchmark may import it; the product path never calls it and has
no CPU fallback.  It shares no code with the CUDA library.

It follows the method as the pages state it, one step at a time, with no
blocking, fusion or reordering beyond the definitions:

1. ``G_k = L_k U_k``, a 2x2 unit-determinant LU factor with three scalars,
   ``L = [[1, 0], [a, 1]]`` and ``U = [[b, c], [0, 1/b]]``
   (KroQuant review, "What carries the argument" and section 3.2 Eq. 6; the
   sign convention of ``U`` is the one whose determinant is +1, see
   ``lu_factor``).
2. ``K^(j) = G1 (x) G2 (x) G3 (x) G4 (x) G5``, an explicit dense Kronecker
   product, one 32x32 block per 32 channels (review, "What carries the
   argument"; section 3.2 Eq. 4: ``T`` is block diagonal).
3. The activation row is multiplied on the right, ``y = x T`` (review,
   "Circularity check", Eq. 1: ``A T (W T^-T)^T = A W^T``).
4. MXFP4 quantization of every 32-element block: one shared E8M0 power-of-two
   scale and E2M1 elements (the OCP Microscaling formats the paper cites for
   "MXFP4e2"; abstract and "Core claim").

Readings where the pages are silent:

* the scale exponent is ``floor(log2(amax)) - 2`` (2 = the largest E2M1
  exponent), clamped to ``[-127, 127]``; an all-zero block gets ``-127``;
* elements round to the nearest E2M1 value, ties to the even code, and
  saturate at +-6; the code keeps the sign bit of its input, so a negative
  value that rounds to zero gives code ``0x8``;
* the quantization decision is taken on the float32 value of the transformed
  element (the kernel's precision; the pages fix none);
* two codes per byte, the even element in the low nibble;
* E8M0 byte ``0xFF`` decodes to NaN.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.linalg

BLOCK = 32            # elements per MX block and per Kronecker block
N_FACTORS = 5         # 32 = 2**5, one 2x2 factor per index bit
E2M1_EMAX = 2         # exponent of the largest E2M1 value (6 = 1.5 * 2**2)
E8M0_BIAS = 127

# OCP E2M1 magnitudes, indexed by the 3-bit magnitude code.
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# --------------------------------------------------------------------------
# Step 1-2: the Kronecker-structured block transform
# --------------------------------------------------------------------------
def lu_factor(a: float, b: float, c: float) -> np.ndarray:
    """2x2 factor ``G = L U`` with ``L = [[1,0],[a,1]]``, ``U = [[b,c],[0,1/b]]``.

    Section 3.2 Eq. 6 of the KroQuant paper (as quoted by the review) writes
    ``U = [[a, b], [0, -1/a]]``, whose determinant is -1, while the review's
    summary and its axiom ledger call the factor "unit-determinant".  The form
    used here keeps three scalars and has determinant +1 for every ``b != 0``.
    """
    a, b, c = float(a), float(b), float(c)
    L = np.array([[1.0, 0.0], [a, 1.0]])
    U = np.array([[b, c], [0.0, 1.0 / b]])
    return L @ U


def block_factors(p_j: np.ndarray) -> list:
    """The 2x2 factors of one block from its ``[n, 3]`` parameters (n = 5 for
    32-element blocks, 4 for the 16-element variant)."""
    p_j = np.asarray(p_j, dtype=np.float64)
    return [lu_factor(*p_j[k]) for k in range(p_j.shape[0])]


def kron_factors(factors) -> np.ndarray:
    """``F1 (x) F2 (x) ... (x) F5`` as a dense matrix (numpy's Kronecker
    convention: the first factor acts on the most significant index bit)."""
    K = np.array([[1.0]])
    for G in factors:
        K = np.kron(K, G)
    return K


def kron_block(p_j: np.ndarray) -> np.ndarray:
    """Dense ``K^(j) = G1 (x) G2 (x) ...``: 32x32 from five factors, 16x16
    from four."""
    return kron_factors(block_factors(p_j))


def inverse_block(p_j: np.ndarray) -> np.ndarray:
    """``K^-1 = G1^-1 (x) ... (x) G5^-1`` (review, axiom ledger: the inverse of
    a Kronecker product factorizes); ``G^-1 = U^-1 L^-1`` in closed form."""
    inv = []
    for a, b, c in np.asarray(p_j, dtype=np.float64):
        U_inv = np.array([[1.0 / b, -c], [0.0, b]])
        L_inv = np.array([[1.0, 0.0], [-a, 1.0]])
        inv.append(U_inv @ L_inv)
    return kron_factors(inv)


def hadamard_block() -> np.ndarray:
    """Fixed orthonormal block Hadamard ``H_32 / sqrt(32)`` (Sylvester order),
    the comparator the paper initialises from (review, "Core claim")."""
    return scipy.linalg.hadamard(BLOCK).astype(np.float64) / math.sqrt(BLOCK)


def _apply_blocks(x64: np.ndarray, blocks, block: int = BLOCK) -> np.ndarray:
    x64 = np.asarray(x64, dtype=np.float64)
    M, d = x64.shape
    y = np.empty_like(x64)
    for j in range(d // block):
        sl = slice(block * j, block * (j + 1))
        y[:, sl] = x64[:, sl] @ blocks(j)
    return y


def transform(x64: np.ndarray, params: np.ndarray) -> np.ndarray:
    """``y = x T`` with ``T = diag(K^(1), ..., K^(d/32))``, float64."""
    params = np.asarray(params)
    return _apply_blocks(x64, lambda j: kron_block(params[j]))


def inverse_transform(y64: np.ndarray, params: np.ndarray) -> np.ndarray:
    """``x = y T^-1``, float64."""
    params = np.asarray(params)
    return _apply_blocks(y64, lambda j: inverse_block(params[j]))


def transform_hadamard(x64: np.ndarray) -> np.ndarray:
    """``y = x H_32 / sqrt(32)`` per block: the +-1 Sylvester sums first, then
    one division by ``sqrt(32)``.  For bf16 input the sums are exact in
    float64 (when a block's exponents span less than 40 binades), so a sum
    that cancels is exactly zero, and each output carries one rounding."""
    H = scipy.linalg.hadamard(BLOCK).astype(np.float64)
    return _apply_blocks(x64, lambda j: H) / math.sqrt(BLOCK)


def transform_smooth(x64: np.ndarray, inv_s: np.ndarray) -> np.ndarray:
    """Per-channel scaling ``x diag(s)^-1`` (SmoothQuant, as in the handbook
    page "Quantization: where diffusion differs from an LLM", section
    "SmoothQuant"), with the caller's float32 reciprocal scale."""
    inv = np.asarray(inv_s, dtype=np.float32).astype(np.float64)
    return np.asarray(x64, dtype=np.float64) * inv[None, :]


# --------------------------------------------------------------------------
# bfloat16 input
# --------------------------------------------------------------------------
def bf16_bits_to_float64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns (the top half of a float32)."""
    bits = np.asarray(bits, dtype=np.uint16)
    f32 = (bits.astype(np.uint32) << 16).view(np.float32)
    return f32.astype(np.float64)


# --------------------------------------------------------------------------
# Step 4: MXFP4 (E8M0 scale + E2M1 elements)
# --------------------------------------------------------------------------
def decision_values(y64: np.ndarray) -> np.ndarray:
    """The transformed values as the quantizer sees them: rounded once to
    float32 (round to nearest even), held exactly in float64."""
    return np.asarray(y64, dtype=np.float64).astype(np.float32).astype(np.float64)


def e8m0_exponent(amax):
    """Shared exponent of a block: ``floor(log2(amax)) - emax(E2M1)``, clamped
    to the E8M0 range; ``-127`` for an all-zero block.  Works elementwise."""
    amax = np.asarray(amax, dtype=np.float64)
    _, p = np.frexp(amax)            # amax = f * 2**p with 0.5 <= f < 1 (exact)
    e = (p.astype(np.int64) - 1) - E2M1_EMAX
    e = np.where(amax == 0.0, -E8M0_BIAS, e)
    return np.clip(e, -E8M0_BIAS, E8M0_BIAS)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code (4 bits: sign, 3-bit magnitude), ties to the even
    magnitude code, saturating at 6.  ``v`` is already divided by the scale."""
    v = np.asarray(v, dtype=np.float64)
    m = np.abs(v)
    code = np.zeros(v.shape, dtype=np.uint8)
    for k in range(len(E2M1_GRID) - 1):
        mid = 0.5 * (E2M1_GRID[k] + E2M1_GRID[k + 1])
        # past the midpoint -> at least k+1; on it -> the even one of k, k+1
        up = (m > mid) | ((m == mid) & (k % 2 == 1))
        code += up.astype(np.uint8)
    code |= (np.signbit(v).astype(np.uint8) << 3)
    return code


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    """Value of an E2M1 code from its bit fields: sign, 2-bit exponent (bias
    1), 1-bit mantissa; exponent field 0 is subnormal (0 or 0.5)."""
    code = np.asarray(code, dtype=np.uint8)
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = (code & 1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e.astype(np.int64) - 1))
    return np.where(s == 1, -mag, mag)


def mxfp4_quantize(y64: np.ndarray, block: int = BLOCK):
    """Quantize ``[M, d]`` values block by block (``block`` elements share
    one scale: 32 for MXFP4, 16 for the 16-element variant).

    Returns ``(codes [M, d] uint8 (unpacked), scale bytes [M, d/block] uint8)``.
    """
    yq = decision_values(y64)
    M, d = yq.shape
    nb = d // block
    blocks = yq.reshape(M, nb, block)
    amax = np.abs(blocks).max(axis=2)
    e = e8m0_exponent(amax)
    v = blocks * np.ldexp(1.0, -e)[:, :, None]        # exact: power-of-two scaling
    codes = e2m1_encode(v).reshape(M, d)
    return codes, (e + E8M0_BIAS).astype(np.uint8)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: element ``2i`` in the low nibble, ``2i+1`` high."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def e8m0_decode(scale: np.ndarray) -> np.ndarray:
    """``2**(s - 127)``; the byte 0xFF is NaN."""
    s = np.asarray(scale, dtype=np.int64)
    val = np.ldexp(1.0, s - E8M0_BIAS)
    return np.where(s == 255, np.nan, val)


def dequantize(q_packed: np.ndarray, scales: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Exact float64 value of packed codes times their block scales."""
    codes = unpack_codes(q_packed)
    M, d = codes.shape
    vals = e2m1_decode(codes).reshape(M, d // block, block)
    return (vals * e8m0_decode(scales)[:, :, None]).reshape(M, d)


# --------------------------------------------------------------------------
# The entry points the library exposes, end to end
# --------------------------------------------------------------------------
def quantize(x_bits: np.ndarray, params: np.ndarray):
    """KroQuant quantizer: bf16 bits ``[M, d]`` -> (packed codes, scales)."""
    codes, scales = mxfp4_quantize(transform(bf16_bits_to_float64(x_bits), params))
    return pack_codes(codes), scales


def quantize_hadamard(x_bits: np.ndarray):
    codes, scales = mxfp4_quantize(transform_hadamard(bf16_bits_to_float64(x_bits)))
    return pack_codes(codes), scales


def quantize_smooth(x_bits: np.ndarray, inv_s: np.ndarray):
    codes, scales = mxfp4_quantize(transform_smooth(bf16_bits_to_float64(x_bits), inv_s))
    return pack_codes(codes), scales


# --------------------------------------------------------------------------
# The 16-element variant: four factors per block, one scale per 16 elements
# (the review's "Where Pith is reading between the lines": other blockwise
# formats by changing the number of Kronecker factors).
# --------------------------------------------------------------------------
BLOCK16 = 16
N_FACTORS16 = 4


def transform16(x64: np.ndarray, params16: np.ndarray) -> np.ndarray:
    """``y = x T`` with 16x16 blocks ``G1 (x) G2 (x) G3 (x) G4``."""
    params16 = np.asarray(params16)
    return _apply_blocks(x64, lambda j: kron_block(params16[j]), BLOCK16)


def abs_transform16(x64: np.ndarray, params16: np.ndarray) -> np.ndarray:
    params16 = np.asarray(params16)
    return _apply_blocks(np.abs(x64), lambda j: np.abs(kron_block(params16[j])), BLOCK16)


def fold_weight16(w64: np.ndarray, params16: np.ndarray) -> np.ndarray:
    """``W' = W T16^-T``: each 16-column block of a weight row times
    ``(K16^(j))^-T`` (Eq. 1 with 16-element blocks)."""
    params16 = np.asarray(params16)
    return _apply_blocks(w64, lambda j: inverse_block(params16[j]).T, BLOCK16)


def abs_fold_weight16(w64: np.ndarray, params16: np.ndarray) -> np.ndarray:
    params16 = np.asarray(params16)
    return _apply_blocks(np.abs(w64), lambda j: np.abs(inverse_block(params16[j]).T), BLOCK16)


def quantize_weight16(w_bits: np.ndarray, params16: np.ndarray):
    """MXFP4 with 16-element blocks of ``W T16^-T``: (packed codes, scales
    ``[N, d/16]``)."""
    codes, scales = mxfp4_quantize(fold_weight16(bf16_bits_to_float64(w_bits), params16),
                                   BLOCK16)
    return pack_codes(codes), scales


def quantize16(x_bits: np.ndarray, params16: np.ndarray):
    """bf16 bits ``[M, d]`` -> (packed codes ``[M, d/2]``, scales ``[M, d/16]``)."""
    codes, scales = mxfp4_quantize(transform16(bf16_bits_to_float64(x_bits), params16), BLOCK16)
    return pack_codes(codes), scales


# --------------------------------------------------------------------------
# The normalization in front of the quantizer (review, "Core claim" and the
# axiom ledger: normalization layers and AdaLN between blocks are why the
# transform must run online; handbook page "Quantization: where diffusion
# differs from an LLM": AdaLN multiplies timestep-dependent scales and adds
# shifts onto the activations).  Reading: DiT's modulation
# ``h = LN(x) (1 + scale[b]) + shift[b]``, LayerNorm over the row without an
# affine part, row m belonging to sample ``b = m // tokens_per_sample``.
# --------------------------------------------------------------------------
def adaln_modulate(x64: np.ndarray, shift64: np.ndarray, scale64: np.ndarray,
                   tokens_per_sample: int, eps: float) -> np.ndarray:
    """``h = (x - mean) / sqrt(var + eps) * (1 + scale[b]) + shift[b]`` per
    row, mean and (biased) variance over the row's d channels, float64."""
    x64 = np.asarray(x64, dtype=np.float64)
    M = x64.shape[0]
    mu = x64.mean(axis=1, keepdims=True)
    var = ((x64 - mu) ** 2).mean(axis=1, keepdims=True)
    n = (x64 - mu) / np.sqrt(var + eps)
    b = np.arange(M) // int(tokens_per_sample)
    return n * (1.0 + np.asarray(scale64, dtype=np.float64)[b]) + \
        np.asarray(shift64, dtype=np.float64)[b]


def adaln_terms(x64: np.ndarray, shift64: np.ndarray, scale64: np.ndarray,
                tokens_per_sample: int, eps: float) -> np.ndarray:
    """``(|x| + mean(|x|)) / sqrt(var + eps) |1 + scale[b]| + |shift[b]|``:
    the magnitude of the terms each modulated value is made of (the mean is
    the sum of the terms ``x_i / d``, whose magnitudes add to ``mean(|x|)``)."""
    x64 = np.asarray(x64, dtype=np.float64)
    M = x64.shape[0]
    mu = x64.mean(axis=1, keepdims=True)
    var = ((x64 - mu) ** 2).mean(axis=1, keepdims=True)
    b = np.arange(M) // int(tokens_per_sample)
    return (np.abs(x64) + np.abs(x64).mean(axis=1, keepdims=True)) / np.sqrt(var + eps) * \
        np.abs(1.0 + np.asarray(scale64, dtype=np.float64)[b]) + \
        np.abs(np.asarray(shift64, dtype=np.float64)[b])


def quantize_adaln(x_bits: np.ndarray, shift_bits: np.ndarray, scale_bits: np.ndarray,
                   tokens_per_sample: int, eps: float, params: np.ndarray):
    """MXFP4(AdaLN(x) T): bf16 bits of x ``[M, d]`` and of shift / scale
    ``[B, d]`` -> (packed codes, scales)."""
    h = adaln_modulate(bf16_bits_to_float64(x_bits), bf16_bits_to_float64(shift_bits),
                       bf16_bits_to_float64(scale_bits), tokens_per_sample, eps)
    codes, scales = mxfp4_quantize(transform(h, params))
    return pack_codes(codes), scales


# --------------------------------------------------------------------------
# Weight side and the W4A4 product (review, "Circularity Check", Eq. 1:
# ``A T (W T^-T)^T = A W^T``, the inverse folded into the weights offline)
# --------------------------------------------------------------------------
def fold_weight(w64: np.ndarray, params: np.ndarray) -> np.ndarray:
    """``W' = W T^-T`` for weights ``W [N, d]`` (rows are output channels):
    each 32-column block of a row is multiplied on the right by
    ``(K^(j))^-T``, so that ``(x T) W'^T = x W^T``."""
    params = np.asarray(params)
    return _apply_blocks(w64, lambda j: inverse_block(params[j]).T)


def abs_fold_weight(w64: np.ndarray, params: np.ndarray) -> np.ndarray:
    """``|W| |K^-T|`` blockwise, the magnitude the fold's rounding is stated
    against."""
    params = np.asarray(params)
    return _apply_blocks(np.abs(w64), lambda j: np.abs(inverse_block(params[j]).T))


def quantize_weight(w_bits: np.ndarray, params: np.ndarray):
    """MXFP4 of the folded weights: bf16 bits ``[N, d]`` -> (packed codes
    ``[N, d/2]``, scales ``[N, d/32]``), the same quantizer as activations."""
    codes, scales = mxfp4_quantize(fold_weight(bf16_bits_to_float64(w_bits), params))
    return pack_codes(codes), scales


def mxfp4_gemm(qa: np.ndarray, sa: np.ndarray, qb: np.ndarray, sb: np.ndarray,
               block: int = BLOCK) -> np.ndarray:
    """``C = A B^T`` in float64 for MXFP4 operands ``A [M, K]`` and ``B [N, K]``
    (packed codes and per-``block`` scales along K): the product the W4A4
    layer computes, from the exact values the codes and scales stand for."""
    return dequantize(qa, sa, block) @ dequantize(qb, sb, block).T


def abs_mxfp4_gemm(qa: np.ndarray, sa: np.ndarray, qb: np.ndarray, sb: np.ndarray,
                   block: int = BLOCK) -> np.ndarray:
    """``|A| |B|^T``: the sum of the magnitudes of the products in each output."""
    return np.abs(dequantize(qa, sa, block)) @ np.abs(dequantize(qb, sb, block)).T


# --------------------------------------------------------------------------
# Magnitudes the tolerance rule is stated against
# --------------------------------------------------------------------------
def abs_transform(x64: np.ndarray, params: np.ndarray) -> np.ndarray:
    """``|x| |T|`` elementwise (``|K| = |G1| (x) ... (x) |G5|``): the size of
    the sum each transformed element is, used to state rounding tolerances."""
    params = np.asarray(params)
    return _apply_blocks(np.abs(x64), lambda j: np.abs(kron_block(params[j])))


def abs_transform_hadamard(x64: np.ndarray) -> np.ndarray:
    H = np.abs(hadamard_block())
    return _apply_blocks(np.abs(x64), lambda j: H)


def abs_inverse_transform(y64: np.ndarray, params: np.ndarray) -> np.ndarray:
    params = np.asarray(params)
    return _apply_blocks(np.abs(y64), lambda j: np.abs(inverse_block(params[j])))


PARAMS_PER_BLOCK = 3 * N_FACTORS          # three scalars per 2x2 factor


# --------------------------------------------------------------------------
# Scale layout the block-scaled tensor-core product reads (a data movement,
# no arithmetic): 128-row x 4-scale tiles of 512 bytes, row-tile major then
# K; inside a tile row r = r0 + 32 r1, scale i at byte 16 r0 + 4 r1 + i.
# Rows are padded to 128 and scale columns to 4 with zero bytes.
# --------------------------------------------------------------------------
def scales_to_mma(scales: np.ndarray) -> np.ndarray:
    """Row-major scale bytes ``[rows, K/32]`` -> the tiled layout (1-D)."""
    scales = np.asarray(scales, dtype=np.uint8)
    rows, ns = scales.shape
    rt, ct = -(-rows // 128), -(-ns // 4)
    out = np.zeros(rt * ct * 512, dtype=np.uint8)
    for r in range(rows):
        for k in range(ns):
            tile = (r // 128) * ct + k // 4
            rr = r % 128
            out[tile * 512 + 16 * (rr % 32) + 4 * (rr // 32) + k % 4] = scales[r, k]
    return out


def scales_from_mma(tiled: np.ndarray, rows: int, ns: int) -> np.ndarray:
    """Inverse of ``scales_to_mma`` for ``rows`` rows of ``ns`` scales."""
    tiled = np.asarray(tiled, dtype=np.uint8)
    ct = -(-ns // 4)
    out = np.empty((rows, ns), dtype=np.uint8)
    for r in range(rows):
        for k in range(ns):
            rr = r % 128
            out[r, k] = tiled[((r // 128) * ct + k // 4) * 512 + 16 * (rr % 32) + 4 * (rr // 32) +
                              k % 4]
    return out
