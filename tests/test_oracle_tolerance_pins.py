"""Pins for the oracle's tolerance magnitudes.

Every parity band of the GPU tests is ``1e-5`` times a magnitude that the
oracle computes: the sum of the absolute values of the terms that make up
each transformed, folded or multiplied value (``(|x| |K|)_c`` for the
transform; ``|W| |K^-T|`` for the weight fold; ``|A| |B|^T`` for the W4A4
product).  A slip in one of these functions (a dropped ``abs``, a missing
transpose, the wrong factor) would silently widen or narrow every band, so
each one is tied here to something other than its own code:

* the bound it exists for: ``|f(x)| <= abs_f(x)`` on signed random inputs;
* equality with ``f`` itself when every input and every matrix entry is
  non-negative (no term can cancel);
* single entries against the index formula written from the definition,
  ``sum_r |x_r| prod_k |F_k[bit_k(r), bit_k(c)]|``, with the 2x2 factors
  multiplied out by hand from ``(a, b, c)`` and inverted by the adjugate (not
  by the oracle's own ``lu_factor`` / ``inverse_block``);
* for the W4A4 product, a brute-force triple loop over values decoded by hand
  from the E2M1 table and ``2^(s - 127)``.

The last test plants plausible mistakes into copies of these functions (on
the CPU) and checks that each one fails at least one of the pins.

Sources: KroQuant review (pith.science), "What carries the argument"
(``K = G1 (x) ... (x) G5``, unit-determinant LU factors), "Circularity
Check" (Eq. 1, ``W T^-T``), and the OCP Microscaling definition of MXFP4 it
cites (E2M1 values, E8M0 scales).
"""
import math

import numpy as np
import pytest

import workloads as w
from oracle import kq_oracle as o

BOUND_SLACK = 1.0 + 1e-12


# ----------------------------------------------------------------- helpers
def _hand_factor(a, b, c):
    """``[[1,0],[a,1]] [[b,c],[0,1/b]]`` multiplied out on paper."""
    return np.array([[b, c], [a * b, a * c + 1.0 / b]], dtype=np.float64)


def _hand_inverse(a, b, c):
    """Inverse of a determinant-one 2x2 matrix: its adjugate."""
    g = _hand_factor(a, b, c)
    return np.array([[g[1, 1], -g[0, 1]], [-g[1, 0], g[0, 0]]])


def _bit(idx, k, n):
    """Index bit the k-th factor (0-based) of an n-factor product acts on:
    the first factor on the most significant bit."""
    return (idx >> (n - 1 - k)) & 1


def _index_abs_entry(vec, factors, c, transpose=False):
    """``sum_r |vec_r| prod_k |F_k[bit(r), bit(c)]|`` (``F_k[bit(c), bit(r)]``
    for the transposed product)."""
    n = len(factors)
    total = 0.0
    for r in range(1 << n):
        prod = 1.0
        for k, F in enumerate(factors):
            i, j = _bit(r, k, n), _bit(c, k, n)
            prod *= abs(F[j, i] if transpose else F[i, j])
        total += abs(vec[r]) * prod
    return total


def _signed_params(nb, n, seed):
    rng = np.random.default_rng(seed)
    p = np.empty((nb, n, 3))
    p[..., 0] = rng.uniform(-1.5, 1.5, (nb, n))
    p[..., 1] = rng.choice([-1.0, 1.0], (nb, n)) * 2.0 ** rng.uniform(-1.5, 1.5, (nb, n))
    p[..., 2] = rng.uniform(-1.5, 1.5, (nb, n))
    return p


def _forward_nonneg_params(nb, n, seed):
    """a >= 0, b > 0, c >= 0: every entry of G = [[b, c], [ab, ac + 1/b]] is
    non-negative."""
    rng = np.random.default_rng(seed)
    p = np.empty((nb, n, 3))
    p[..., 0] = rng.uniform(0.0, 1.0, (nb, n))
    p[..., 1] = 2.0 ** rng.uniform(-1, 1, (nb, n))
    p[..., 2] = rng.uniform(0.0, 1.0, (nb, n))
    return p


def _inverse_nonneg_params(nb, n, seed):
    """a <= 0, b > 0, c <= 0: every entry of G^-1 = [[ac + 1/b, -c], [-ab, b]]
    is non-negative."""
    p = _forward_nonneg_params(nb, n, seed)
    p[..., 0] *= -1.0
    p[..., 2] *= -1.0
    return p


def _signed_x(M, d, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, d)) * np.exp(rng.uniform(-3, 3, (1, d)))
    return x


# ------------------------------------------------------- the pin checks
# Each check takes the function under test so that the planted-mistake test
# below can run the same checks on a mutated copy.
def _check_abs_blockwise(abs_fn, fn, block, n, nonneg_params, factor_of, transpose, seed):
    """The three pins of a blockwise ``|x| |F|`` magnitude."""
    nb = 3
    d = block * nb
    x = _signed_x(5, d, seed)
    p = _signed_params(nb, n, seed + 1)
    mag = abs_fn(x, p)
    # 1. it bounds the value it is the magnitude of
    assert (np.abs(fn(x, p)) <= mag * BOUND_SLACK).all()
    # 2. no cancellation possible -> equal to the value itself
    xp = np.abs(x)
    pp = nonneg_params(nb, n, seed + 2)
    np.testing.assert_allclose(abs_fn(xp, pp), fn(xp, pp), rtol=1e-12, atol=0)
    # 3. entries against the index formula
    rng = np.random.default_rng(seed + 3)
    for _ in range(12):
        m, j, c = rng.integers(5), rng.integers(nb), rng.integers(block)
        factors = [factor_of(*p[j, k]) for k in range(n)]
        want = _index_abs_entry(x[m, block * j:block * (j + 1)], factors, c, transpose)
        assert mag[m, block * j + c] == pytest.approx(want, rel=1e-12)


def check_abs_transform(abs_fn=o.abs_transform):
    _check_abs_blockwise(abs_fn, o.transform, 32, 5, _forward_nonneg_params,
                         _hand_factor, False, 11)


def check_abs_inverse_transform(abs_fn=o.abs_inverse_transform):
    _check_abs_blockwise(abs_fn, o.inverse_transform, 32, 5, _inverse_nonneg_params,
                         _hand_inverse, False, 21)


def check_abs_fold_weight(abs_fn=o.abs_fold_weight):
    _check_abs_blockwise(abs_fn, o.fold_weight, 32, 5, _inverse_nonneg_params,
                         _hand_inverse, True, 31)


def check_abs_transform16(abs_fn=o.abs_transform16):
    _check_abs_blockwise(abs_fn, o.transform16, 16, 4, _forward_nonneg_params,
                         _hand_factor, False, 41)


def check_abs_fold_weight16(abs_fn=o.abs_fold_weight16):
    _check_abs_blockwise(abs_fn, o.fold_weight16, 16, 4, _inverse_nonneg_params,
                         _hand_inverse, True, 51)


def check_abs_transform_hadamard(abs_fn=o.abs_transform_hadamard):
    """|H_32 / sqrt(32)| has every entry 1/sqrt(32): each output of a block is
    the block's sum of |x| over sqrt(32), in every column."""
    x = _signed_x(4, 96, 61)
    mag = abs_fn(x)
    assert (np.abs(o.transform_hadamard(x)) <= mag * BOUND_SLACK).all()
    for j in range(3):
        s = np.abs(x[:, 32 * j:32 * (j + 1)]).sum(axis=1) / math.sqrt(32.0)
        np.testing.assert_allclose(mag[:, 32 * j:32 * (j + 1)],
                                   np.repeat(s[:, None], 32, axis=1), rtol=1e-13)
    # Column 0 of a Sylvester Hadamard matrix is all ones: there the value of
    # a non-negative input is its magnitude.
    xp = np.abs(x)
    np.testing.assert_allclose(abs_fn(xp)[:, 0::32], o.transform_hadamard(xp)[:, 0::32],
                               rtol=1e-13)


def _hand_value(code, s):
    """Value of one E2M1 code under scale byte s, decoded by hand."""
    table = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    v = table[code & 7] * 2.0 ** (int(s) - 127)
    return -v if code & 8 else v


def _random_operands(rows, K, block, seed, signed=True):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 16 if signed else 8, (rows, K)).astype(np.uint8)
    scales = rng.integers(120, 134, (rows, K // block)).astype(np.uint8)
    return codes, scales


def check_abs_mxfp4_gemm(abs_fn=o.abs_mxfp4_gemm):
    for block in (32, 16):
        M, N, K = 3, 4, 64
        ca, sa = _random_operands(M, K, block, 71 + block)
        cb, sb = _random_operands(N, K, block, 72 + block)
        qa, qb = o.pack_codes(ca), o.pack_codes(cb)
        mag = abs_fn(qa, sa, qb, sb, block)
        # 1. bound
        assert (np.abs(o.mxfp4_gemm(qa, sa, qb, sb, block)) <= mag * BOUND_SLACK).all()
        # 3. brute force: sum over k of |a_k b_k|, values decoded by hand
        for m in range(M):
            for n in range(N):
                want = sum(abs(_hand_value(ca[m, k], sa[m, k // block]) *
                               _hand_value(cb[n, k], sb[n, k // block])) for k in range(K))
                assert mag[m, n] == pytest.approx(want, rel=1e-15, abs=0)
        # 2. all sign bits clear -> the product itself
        ca, sa = _random_operands(M, K, block, 73 + block, signed=False)
        cb, sb = _random_operands(N, K, block, 74 + block, signed=False)
        qa, qb = o.pack_codes(ca), o.pack_codes(cb)
        np.testing.assert_array_equal(abs_fn(qa, sa, qb, sb, block),
                                      o.mxfp4_gemm(qa, sa, qb, sb, block))


# ----------------------------------------------------------------- tests
def test_abs_transform_pins():
    check_abs_transform()


def test_abs_inverse_transform_pins():
    check_abs_inverse_transform()


def test_abs_fold_weight_pins():
    check_abs_fold_weight()


def test_abs_transform16_pins():
    check_abs_transform16()


def test_abs_fold_weight16_pins():
    check_abs_fold_weight16()


def test_abs_transform_hadamard_pins():
    check_abs_transform_hadamard()


def test_abs_mxfp4_gemm_pins():
    check_abs_mxfp4_gemm()


def test_abs_transform_bounds_the_workload_transform():
    """The magnitude bounds the transform on a seeded DiT-shaped input too
    (outlier channels, the parameters' own distribution)."""
    c = w.make_case("flux_schnell", 0, 2, M=8)
    x64 = o.bf16_bits_to_float64(c.x_bits())
    assert (np.abs(o.transform(x64, c.params)) <= o.abs_transform(x64, c.params) *
            BOUND_SLACK).all()
    assert (np.abs(o.fold_weight(x64, c.params)) <= o.abs_fold_weight(x64, c.params) *
            BOUND_SLACK).all()


# --------------------------------------------------- planted mistakes
def _blocks(fn_block, block=32):
    """A blockwise magnitude built from a per-block matrix and an input map,
    so that a mutant differs from the oracle in exactly one place."""
    def f(x, p, xmap=np.abs):
        return o._apply_blocks(xmap(x), lambda j: fn_block(np.asarray(p)[j]), block)
    return f


MUTANTS = [
    # (name, check, mutated function)
    ("transform: abs of x dropped", check_abs_transform,
     lambda x, p: _blocks(lambda q: np.abs(o.kron_block(q)))(x, p, xmap=lambda v: v)),
    ("transform: abs of K dropped", check_abs_transform,
     _blocks(lambda q: o.kron_block(q))),
    ("transform: K transposed", check_abs_transform,
     _blocks(lambda q: np.abs(o.kron_block(q)).T)),
    ("transform: factors in reverse order", check_abs_transform,
     _blocks(lambda q: np.abs(o.kron_block(q[::-1])))),
    ("inverse: forward block instead of the inverse", check_abs_inverse_transform,
     _blocks(lambda q: np.abs(o.kron_block(q)))),
    ("inverse: transposed inverse", check_abs_inverse_transform,
     _blocks(lambda q: np.abs(o.inverse_block(q)).T)),
    ("fold: transpose missing", check_abs_fold_weight,
     _blocks(lambda q: np.abs(o.inverse_block(q)))),
    ("fold: abs of K^-T dropped", check_abs_fold_weight,
     _blocks(lambda q: o.inverse_block(q).T)),
    ("fold: K instead of K^-1", check_abs_fold_weight,
     _blocks(lambda q: np.abs(o.kron_block(q)).T)),
    ("fold: abs of w dropped", check_abs_fold_weight,
     lambda x, p: _blocks(lambda q: np.abs(o.inverse_block(q).T))(x, p, xmap=lambda v: v)),
    ("block-16 transform: K transposed", check_abs_transform16,
     _blocks(lambda q: np.abs(o.kron_block(q)).T, 16)),
    ("block-16 fold: transpose missing", check_abs_fold_weight16,
     _blocks(lambda q: np.abs(o.inverse_block(q)), 16)),
    ("hadamard: abs of x dropped", check_abs_transform_hadamard,
     lambda x: o._apply_blocks(x, lambda j: np.abs(o.hadamard_block()))),
    ("hadamard: abs of H dropped", check_abs_transform_hadamard,
     lambda x: o._apply_blocks(np.abs(x), lambda j: o.hadamard_block())),
    ("gemm: abs of B dropped", check_abs_mxfp4_gemm,
     lambda qa, sa, qb, sb, block=32: np.abs(o.dequantize(qa, sa, block)) @
     o.dequantize(qb, sb, block).T),
    ("gemm: B's scales ignored", check_abs_mxfp4_gemm,
     lambda qa, sa, qb, sb, block=32: np.abs(o.dequantize(qa, sa, block)) @
     np.abs(o.dequantize(qb, np.full_like(sb, 127), block)).T),
    ("gemm: scales taken per 32 whatever the block", check_abs_mxfp4_gemm,
     lambda qa, sa, qb, sb, block=32: np.abs(o.dequantize(qa, sa[:, ::32 // block], 32)) @
     np.abs(o.dequantize(qb, sb[:, ::32 // block], 32)).T),
]


@pytest.mark.parametrize("name,check,mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistakes_fail_a_pin(name, check, mutant):
    with pytest.raises(AssertionError):
        check(mutant)
