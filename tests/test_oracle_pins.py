"""Pins for the CPU oracle: each check ties a step of the oracle to something
other than its own code (a closed form, an index-level definition, a library
routine, brute force), so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails here.

Sources: the KroQuant review (pith.science, "What carries the argument",
section 3.2 Eq. 4 and Eq. 6, the axiom ledger, the abstract) and the OCP
Microscaling format it cites for MXFP4.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

import workloads as w
from oracle import kq_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_params(nb, seed):
    return w.draw_params(32 * nb, seed)


# ---------------------------------------------------------------- factors
def test_lu_factor_multiplied_out():
    """G = [[1,0],[a,1]] [[b,c],[0,1/b]] = [[b, c], [a b, a c + 1/b]], det 1."""
    rng = np.random.default_rng(1)
    for _ in range(200):
        a, c = rng.uniform(-3, 3, 2)
        b = rng.choice([-1, 1]) * 2.0 ** rng.uniform(-4, 4)
        G = o.lu_factor(a, b, c)
        assert G[0, 0] == b and G[0, 1] == c
        assert G[1, 0] == pytest.approx(a * b, rel=1e-15)
        assert G[1, 1] == pytest.approx(a * c + 1.0 / b, rel=1e-13, abs=1e-15)
        assert G[0, 0] * G[1, 1] - G[0, 1] * G[1, 0] == pytest.approx(1.0, abs=1e-12)


def test_kron_block_matches_index_formula():
    """K[r, c] = prod_k G_k[bit(r), bit(c)], G1 on index bit 4 (the MSB)."""
    p = rand_params(3, 11)
    for j in range(3):
        K = o.kron_block(p[j])
        G = o.block_factors(p[j])
        ref = np.ones((32, 32))
        for r in range(32):
            for c in range(32):
                for k in range(5):
                    sh = 4 - k
                    ref[r, c] *= G[k][(r >> sh) & 1, (c >> sh) & 1]
        np.testing.assert_allclose(K, ref, rtol=1e-13, atol=1e-15)


def test_transform_matches_factorwise_contraction():
    """y = x K equals applying each 2x2 factor to its own index bit of the
    row vector (x viewed as a 2x2x2x2x2 tensor), which fixes both the
    orientation (row vector times K) and the factor order."""
    rng = np.random.default_rng(2)
    nb = 4
    p = rand_params(nb, 12)
    x = rng.standard_normal((7, 32 * nb))
    y = o.transform(x, p)
    for j in range(nb):
        t = x[:, 32 * j:32 * (j + 1)].reshape(7, 2, 2, 2, 2, 2)
        for k, G in enumerate(o.block_factors(p[j])):
            t = np.moveaxis(np.tensordot(t, G, axes=([k + 1], [0])), -1, k + 1)
        np.testing.assert_allclose(y[:, 32 * j:32 * (j + 1)], t.reshape(7, 32),
                                   rtol=1e-12, atol=1e-12)


def test_unit_determinant_every_block_of_every_config():
    """det K = prod_k det(G_k)^16 = 1 for the factors G = [[1,0],[a,1]] [[b,c],[0,1/b]]."""
    for name, di, gi in w.all_case_keys():
        seed = w.case_seed(name, di, gi)
        d = w.CONFIGS[name]["d"][di]
        p = w.draw_params(d, seed)
        for j in range(d // 32):
            det = np.linalg.det(o.kron_block(p[j]))
            assert det == pytest.approx(1.0, rel=1e-9)


def test_inverse_round_trip():
    """(x K) K^-1 recovers x to 1e-12 relative, and K (G1^-1 (x) ...) = I."""
    rng = np.random.default_rng(3)
    p = rand_params(6, 13)
    x = rng.standard_normal((5, 192))
    back = o.inverse_transform(o.transform(x, p), p)
    for j in range(6):
        sl = slice(32 * j, 32 * (j + 1))
        err = np.linalg.norm(back[:, sl] - x[:, sl]) / np.linalg.norm(x[:, sl])
        assert err < 1e-12
        np.testing.assert_allclose(o.kron_block(p[j]) @ o.inverse_block(p[j]), np.eye(32),
                                   atol=1e-11)


def test_transform_invariance_eq1():
    """Eq. 1: (A T)(W T^-T)^T = A W^T with the inverse folded into W."""
    rng = np.random.default_rng(4)
    nb = 3
    p = rand_params(nb, 14)
    A = rng.standard_normal((6, 32 * nb))
    W = rng.standard_normal((5, 32 * nb))
    T_inv = scipy.linalg.block_diag(*[o.inverse_block(p[j]) for j in range(nb)])
    lhs = o.transform(A, p) @ (W @ T_inv.T).T
    np.testing.assert_allclose(lhs, A @ W.T, rtol=1e-10, atol=1e-10)


# -------------------------------------------------------------- Hadamard
def test_eq6_form_at_hadamard_init_gives_sylvester_hadamard():
    """With Eq. 6's factor L=[[1,0],[l,1]], U=[[a,b],[0,-1/a]] at l=1,
    a=b=1/sqrt2, every factor is H2/sqrt2 and K is scipy's H32/sqrt32."""
    s = 1 / math.sqrt(2)
    G = np.array([[1, 0], [1, 1]]) @ np.array([[s, s], [0, -1 / s]])
    K = o.kron_factors([G] * 5)
    np.testing.assert_allclose(K, scipy.linalg.hadamard(32) / math.sqrt(32), atol=1e-15)
    np.testing.assert_allclose(o.hadamard_block(), K, atol=1e-15)


def test_lu_form_signed_hadamard():
    """(a,b,c) = (-1, 1/sqrt2, 1/sqrt2) gives G = [[1,1],[-1,1]]/sqrt2, so
    K = diag((-1)^popcount(r)) H32 / sqrt32, orthonormal."""
    s = 1 / math.sqrt(2)
    p = np.array([[-1.0, s, s]] * 5)
    K = o.kron_block(p)
    D = np.diag([(-1) ** bin(r).count("1") for r in range(32)])
    np.testing.assert_allclose(K, D @ scipy.linalg.hadamard(32) / math.sqrt(32), atol=1e-14)
    np.testing.assert_allclose(K @ K.T, np.eye(32), atol=1e-14)


def test_hadamard_entries_closed_form():
    """Sylvester: H[r, c] = (-1)^popcount(r & c)."""
    H = o.hadamard_block() * math.sqrt(32)
    for r in range(32):
        for c in range(32):
            assert H[r, c] == (-1) ** bin(r & c).count("1")


# ------------------------------------------------------------------ E2M1
def test_e2m1_grid_from_bit_fields():
    """Magnitude codes 0..7 decode (sign, 2-bit exponent bias 1, 1 mantissa
    bit, subnormal at exponent 0) to 0, .5, 1, 1.5, 2, 3, 4, 6."""
    dec = o.e2m1_decode(np.arange(16, dtype=np.uint8))
    np.testing.assert_array_equal(dec[:8], [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(dec[8:], -np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6]))
    np.testing.assert_array_equal(o.E2M1_GRID, dec[:8])


def _brute_force_code(v):
    """Search all 16 codes for the nearest value; ties go to the even
    magnitude code; zero takes the sign of v."""
    vals = o.e2m1_decode(np.arange(16, dtype=np.uint8))
    best = None
    for code in range(16):
        if code == 8 and not np.signbit(v):
            continue
        if code == 0 and np.signbit(v):
            continue
        dist = abs(v - vals[code])
        key = (dist, (code & 7) % 2)          # nearer first, then even magnitude
        if best is None or key < best[0]:
            best = (key, code)
    return best[1]


def test_e2m1_encode_matches_brute_force():
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    mids = (grid[1:] + grid[:-1]) / 2
    pts = [0.0, -0.0, 7.999, 1e-30, -1e-30, 100.0, -100.0]
    for m in np.concatenate([grid, mids]):
        f = np.float32(m)
        for q in (np.nextafter(f, np.float32(-1)), f, np.nextafter(f, np.float32(10))):
            pts += [float(q), -float(q)]
    pts += list(np.linspace(-8, 8, 4001))
    pts = np.array(pts)
    got = o.e2m1_encode(pts)
    for v, g in zip(pts, got):
        assert g == _brute_force_code(v), (v, g)


def test_e2m1_ties_to_even_and_saturation():
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.5, -0.25, -5.0, -0.1])
    np.testing.assert_array_equal(
        o.e2m1_encode(v), [0, 2, 2, 4, 4, 6, 6, 7, 7, 8, 14, 8])


# ----------------------------------------------------------------- scale
def test_scale_rule_hand_cases():
    k = 3
    y = np.full((1, 32), 2.0 ** k)
    codes, s = o.mxfp4_quantize(y)
    assert s[0, 0] == k - 2 + 127 and (codes == 6).all()          # value 4 * 2^(k-2)
    y[0, 5] = 6 * 2.0 ** k                                          # amax = 1.5 * 2^(k+2)
    codes, s = o.mxfp4_quantize(y)
    assert s[0, 0] == k + 127 and codes[0, 5] == 7
    below = np.float32(2.0 ** k) - np.float32(2.0 ** (k - 24))      # largest fp32 < 2^k
    y = np.full((1, 32), float(below))
    codes, s = o.mxfp4_quantize(y)
    assert s[0, 0] == k - 3 + 127 and (codes == 7).all()           # ~8 saturates to 6
    codes, s = o.mxfp4_quantize(np.zeros((1, 32)))
    assert s[0, 0] == 0 and (codes == 0).all()
    codes, s = o.mxfp4_quantize(np.full((1, 32), 2.0 ** -130))      # subnormal amax
    assert s[0, 0] == 0


def test_decision_taken_in_float32():
    """0.25 + 1e-12 is 0.25 in float32, a tie that rounds down to code 0."""
    y = np.zeros((1, 32))
    y[0, 0] = 4.0
    y[0, 1] = 0.25 + 1e-12
    codes, s = o.mxfp4_quantize(y)
    assert s[0, 0] == 127 and codes[0, 1] == 0 and codes[0, 0] == 6


# -------------------------------------------------------------- packing
def test_pack_hadamard_unit_vectors():
    """x = e_i gives y_c = (-1)^popcount(i & c)/sqrt32: amax 2^-2.5, scale
    exponent -5 (byte 122), |v| = 2^2.5 = 5.66 -> 6 (code 7 / 0xF); the even
    element lands in the low nibble."""
    for i in (0, 5, 31):
        x = np.zeros((1, 32), dtype=np.uint16)
        x[0, i] = 0x3F80                                  # bf16 1.0
        q, s = o.quantize_hadamard(x)
        assert s[0, 0] == 122
        codes = [7 if bin(i & c).count("1") % 2 == 0 else 15 for c in range(32)]
        expect = [codes[2 * t] | (codes[2 * t + 1] << 4) for t in range(16)]
        assert list(q[0]) == expect


def test_identity_params_quantize_the_input():
    """a=0, b=1, c=0 gives G=I, K=I: the codes of x itself.  Smooth with unit
    scale is a single exact multiply and keeps the sign of -0.0 (code 0x8);
    the sign of an exact-zero sum x.K is not fixed by the arithmetic order
    the pages give, so there only the magnitude code is pinned."""
    vals = np.array([0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7.5,
                     -0.0, -.25, -.75, -5, -6, -1, -0.125, 0.125, 2.25, -3.5, 0.0625, -7.5,
                     1.0, 0.5, 3.0, -4.0], dtype=np.float32)
    bits = vals.view(np.uint32) >> 16
    x = bits.astype(np.uint16)[None, :]
    expect = np.array([0, 0, 1, 2, 2, 2, 3, 4, 4, 4, 5, 6, 6, 6, 7, 7,
                       8, 8, 10, 14, 15, 10, 8, 0, 4, 14, 0, 15, 2, 1, 5, 14])
    q2, s2 = o.quantize_smooth(x, np.ones(32, dtype=np.float32))
    assert s2[0, 0] == 127                                 # amax 7.5 -> exponent 0
    np.testing.assert_array_equal(o.unpack_codes(q2)[0], expect)
    p = np.zeros((1, 5, 3), dtype=np.float32)
    p[:, :, 1] = 1.0
    q, s = o.quantize(x, p)
    assert s[0, 0] == 127
    got = o.unpack_codes(q)[0]
    exact_zero = vals == 0
    np.testing.assert_array_equal(got[~exact_zero], expect[~exact_zero])
    assert ((got[exact_zero] & 7) == 0).all()


def test_smooth_divides_by_the_channel_scale():
    """x diag(s)^-1 with s = 2^k per channel equals quantizing the exactly
    pre-divided input with unit scale; s = 2 everywhere lowers every scale
    byte by one and keeps the codes."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    xv = o.bf16_bits_to_float64(bits)
    q1, s1 = o.quantize_smooth(bits, np.ones(64, dtype=np.float32))
    q2, s2 = o.quantize_smooth(bits, np.full(64, 0.5, dtype=np.float32))
    np.testing.assert_array_equal(q2, q1)
    np.testing.assert_array_equal(s2.astype(int), s1.astype(int) - 1)
    k = np.arange(64) % 3
    inv = (2.0 ** -k).astype(np.float32)
    pre = (xv * 2.0 ** -k).astype(np.float32)                 # exact in bf16
    pre_bits = (pre.view(np.uint32) >> 16).astype(np.uint16)
    q3, s3 = o.quantize_smooth(bits, inv)
    q4, s4 = o.quantize_smooth(pre_bits, np.ones(64, dtype=np.float32))
    np.testing.assert_array_equal(q3, q4)
    np.testing.assert_array_equal(s3, s4)


# ----------------------------------------------------------- invariants
def test_requantizing_dequantized_blocks_is_identity():
    rng = np.random.default_rng(5)
    y = rng.standard_t(3, (64, 256)) * np.exp(rng.uniform(-20, 20, (64, 1)))
    codes, s = o.mxfp4_quantize(y)
    q = o.pack_codes(codes)
    deq = o.dequantize(q, s)
    codes2, s2 = o.mxfp4_quantize(deq)
    np.testing.assert_array_equal(s2, s)
    np.testing.assert_array_equal(codes2, codes)


def test_dequantization_error_bound():
    """|deq - y| <= half the local grid step times X, or y saturated."""
    rng = np.random.default_rng(6)
    y = o.decision_values(rng.standard_normal((32, 512)) * 3)
    codes, s = o.mxfp4_quantize(y)
    deq = o.dequantize(o.pack_codes(codes), s)
    X = np.repeat(o.e8m0_decode(s), 32, axis=1)
    v = np.abs(y) / X
    step = np.where(v < 2, 0.5, np.where(v < 4, 1.0, 2.0))
    err = np.abs(deq - y) / X
    sat = v > 6
    assert (err[~sat] <= step[~sat] / 2 + 1e-15).all()
    assert (np.abs(deq[sat]) == 6 * X[sat]).all() and (v[sat] < 8).all()


def test_dequantize_exhaustive_small_table():
    codes = np.arange(16, dtype=np.uint8)
    for sb in (0, 1, 100, 127, 130, 254, 255):
        q = o.pack_codes(np.tile(codes, 2)[None, :])
        deq = o.dequantize(q, np.array([[sb]], dtype=np.uint8))[0]
        if sb == 255:
            assert np.isnan(deq).all()
        else:
            np.testing.assert_array_equal(deq[:16], o.e2m1_decode(codes) * 2.0 ** (sb - 127))


# ----------------------------------------------------- pages' own numbers
def test_parameter_counts_against_pages():
    with open(os.path.join(GOLDEN, "param_counts.json")) as f:
        g = json.load(f)
    assert o.BLOCK == g["block_size"]
    assert o.PARAMS_PER_BLOCK == g["params_per_block"]
    assert 3 * int(math.log2(o.BLOCK)) == g["params_per_block"]
    assert o.BLOCK ** 2 == g["dense_rotation_scalars_per_block"]
    assert o.PARAMS_PER_BLOCK < g["per_channel_scalars_per_block"] / 2
    p = w.draw_params(1152, 0)
    assert p.size == (1152 // 32) * g["params_per_block"]


def test_workload_generator_prefix_property():
    """Reduced cases are row prefixes of the full-size case."""
    a = w.make_case("sana", 1, M=1500)
    b = w.make_case("sana", 1, M=2100)
    assert np.array_equal(a.x_bits(), b.x_bits()[:1500])
    assert np.array_equal(a.params, b.params)


# ------------------------------------------------- 16-element variant
def test_block16_index_formula_det_and_inverse():
    p = w.draw_params16(48, 21)
    assert p.shape == (3, 4, 3)
    for j in range(3):
        K = o.kron_block(p[j])
        assert K.shape == (16, 16)
        G = o.block_factors(p[j])
        ref = np.ones((16, 16))
        for r in range(16):
            for c in range(16):
                for k in range(4):
                    sh = 3 - k
                    ref[r, c] *= G[k][(r >> sh) & 1, (c >> sh) & 1]
        np.testing.assert_allclose(K, ref, rtol=1e-13, atol=1e-15)
        assert np.linalg.det(K) == pytest.approx(1.0, rel=1e-10)
        np.testing.assert_allclose(K @ o.inverse_block(p[j]), np.eye(16), atol=1e-11)


def test_block16_hadamard_init_and_factorwise_transform():
    s = 1 / math.sqrt(2)
    G = np.array([[1, 0], [1, 1]]) @ np.array([[s, s], [0, -1 / s]])
    np.testing.assert_allclose(o.kron_factors([G] * 4), scipy.linalg.hadamard(16) / 4, atol=1e-15)
    rng = np.random.default_rng(22)
    p = w.draw_params16(64, 23)
    x = rng.standard_normal((5, 64))
    y = o.transform16(x, p)
    for j in range(4):
        t = x[:, 16 * j:16 * (j + 1)].reshape(5, 2, 2, 2, 2)
        for k, Gk in enumerate(o.block_factors(p[j])):
            t = np.moveaxis(np.tensordot(t, Gk, axes=([k + 1], [0])), -1, k + 1)
        np.testing.assert_allclose(y[:, 16 * j:16 * (j + 1)], t.reshape(5, 16), rtol=1e-12,
                                   atol=1e-12)


def test_block16_scale_per_16_elements():
    """Each 16 elements get their own exponent: 2^k fills give k - 2 + 127,
    and the two halves of a 32-element span are scaled independently."""
    y = np.concatenate([np.full(16, 8.0), np.full(16, 0.5)])[None, :]
    codes, s = o.mxfp4_quantize(y, 16)
    assert list(s[0]) == [3 - 2 + 127, -1 - 2 + 127] and (codes == 6).all()
    codes32, s32 = o.mxfp4_quantize(y)
    # one 32-wide scale (exponent 1): 0.5 / 2 = 0.25 is a tie that rounds to 0
    assert s32[0, 0] == 128 and codes[0, 16] == 6 and codes32[0, 16] == 0


def test_block16_parameter_count_is_3_log2_n():
    with open(os.path.join(GOLDEN, "param_counts.json")) as f:
        g = json.load(f)
    assert o.N_FACTORS16 * 3 == 3 * int(math.log2(16))
    assert g["params_per_block"] == 3 * int(math.log2(32))


def test_quantize16_identity_factors_use_16_element_scales():
    vals = np.concatenate([np.full(16, 8.0), np.full(16, 0.5)]).astype(np.float32)
    x = ((vals.view(np.uint32) >> 16).astype(np.uint16))[None, :]
    p = np.zeros((2, 4, 3), dtype=np.float32)
    p[:, :, 1] = 1.0                                     # a = c = 0, b = 1: G = I
    q, s = o.quantize16(x, p)
    assert list(s[0]) == [128, 124]                      # exponents 1 and -3
    assert (o.unpack_codes(q)[0] == 6).all()             # 8/2 = 4 and 0.5*8 = 4


# --------------------------------------------- weight fold and W4A4 product
def test_fold_weight_keeps_the_layer_output_eq1():
    """Eq. 1 through the oracle's own fold: (x T) fold(W)^T = x W^T.  A fold
    that used K instead of K^-1, or forgot the transpose, fails."""
    rng = np.random.default_rng(21)
    nb = 4
    p = rand_params(nb, 22)
    x = rng.standard_normal((7, 32 * nb))
    W = rng.standard_normal((9, 32 * nb))
    lhs = o.transform(x, p) @ o.fold_weight(W, p).T
    np.testing.assert_allclose(lhs, x @ W.T, rtol=1e-10, atol=1e-10)


def test_fold_weight_of_an_orthonormal_block_is_the_transform():
    """(a, b, c) = (-1, 1/sqrt2, 1/sqrt2) makes every factor orthonormal, so
    K^-T = K and folding a weight row equals transforming it."""
    s = 1 / math.sqrt(2)
    p = np.tile(np.array([-1.0, s, s]), (2, 5, 1))
    W = np.random.default_rng(23).standard_normal((3, 64))
    np.testing.assert_allclose(o.fold_weight(W, p), o.transform(W, p), atol=1e-12)


def test_fold_weight_single_factor_closed_form():
    """Only G5 non-trivial (bit 0 of the in-block index): the fold acts on
    adjacent pairs with G5^-T = [[g11, -g10], [-g01, g00]] (row-vector form,
    w' = w G5^-T)."""
    a, b, c = 0.5, 2.0, -0.75
    p = np.zeros((1, 5, 3))
    p[:, :, 1] = 1.0
    p[0, 4] = [a, b, c]
    g00, g01, g10, g11 = b, c, a * b, a * c + 1 / b
    W = np.random.default_rng(24).standard_normal((2, 32))
    got = o.fold_weight(W, p)
    w0, w1 = W[:, 0::2], W[:, 1::2]
    np.testing.assert_allclose(got[:, 0::2], w0 * g11 + w1 * (-g01), atol=1e-12)
    np.testing.assert_allclose(got[:, 1::2], w0 * (-g10) + w1 * g00, atol=1e-12)


def _pack_hand(codes):
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def test_mxfp4_gemm_brute_force():
    """Every output of the product equals a triple loop over values decoded
    by hand from the E2M1 table {0, .5, 1, 1.5, 2, 3, 4, 6} and 2^(s-127)."""
    rng = np.random.default_rng(25)
    M, N, K = 3, 4, 64
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    sa = rng.integers(120, 135, (M, K // 32), dtype=np.uint8)
    sb = rng.integers(120, 135, (N, K // 32), dtype=np.uint8)
    table = [0, 0.5, 1, 1.5, 2, 3, 4, 6]

    def val(code, s):
        v = table[int(code) & 7] * 2.0 ** (int(s) - 127)
        return -v if code & 8 else v

    C = o.mxfp4_gemm(_pack_hand(ca), sa, _pack_hand(cb), sb)
    for m in range(M):
        for n in range(N):
            ref = sum(val(ca[m, k], sa[m, k // 32]) * val(cb[n, k], sb[n, k // 32])
                      for k in range(K))
            assert C[m, n] == ref


def test_mxfp4_gemm_constant_operands_closed_form():
    """All codes 1.0 (code 2): C = K 2^(sa + sb - 254); code 6 (value 4)
    against code 0xB (value -1.5): C = -6 K."""
    M, N, K = 5, 6, 96
    qa = _pack_hand(np.full((M, K), 2))
    qb = _pack_hand(np.full((N, K), 2))
    sa = np.full((M, K // 32), 130, dtype=np.uint8)
    sb = np.full((N, K // 32), 121, dtype=np.uint8)
    assert (o.mxfp4_gemm(qa, sa, qb, sb) == K * 2.0 ** (130 + 121 - 254)).all()
    qa = _pack_hand(np.full((M, K), 6))
    qb = _pack_hand(np.full((N, K), 0xB))
    one_a = np.full((M, K // 32), 127, dtype=np.uint8)
    one_b = np.full((N, K // 32), 127, dtype=np.uint8)
    assert (o.mxfp4_gemm(qa, one_a, qb, one_b) == -6.0 * K).all()


def test_quantize_weight_with_identity_factors_is_the_activation_quantizer():
    """With G_k = I the fold is the identity, so the weight quantizer gives
    the activation quantizer's bytes on the same bf16 matrix."""
    rng = np.random.default_rng(26)
    W = rng.standard_normal((12, 96)).astype(np.float32)
    Wb = (W.view(np.uint32) >> 16).astype(np.uint16)
    p = np.zeros((3, 5, 3), dtype=np.float32)
    p[:, :, 1] = 1.0
    qw, sw = o.quantize_weight(Wb, p)
    qa, sa = o.quantize(Wb, p)
    assert np.array_equal(qw, qa) and np.array_equal(sw, sa)
    # and with an orthonormal block (K^-T = K) it is the transformed quantizer
    s2 = 1 / math.sqrt(2)
    p = np.tile(np.array([-1.0, s2, s2], dtype=np.float32), (3, 5, 1))
    qw, sw = o.quantize_weight(Wb, p)
    qa, sa = o.quantize(Wb, p)
    assert np.array_equal(sw, sa)
    assert (o.unpack_codes(qw) != o.unpack_codes(qa)).mean() < 0.01


# ----------------------------------------------------- LayerNorm + AdaLN
def test_adaln_without_modulation_is_torch_layer_norm():
    """scale = shift = 0: the oracle's modulation is LayerNorm without an
    affine part, as torch's layer_norm computes it (float64)."""
    import torch
    rng = np.random.default_rng(31)
    x = rng.standard_normal((9, 96)) * 3 + 1.5
    z = np.zeros((1, 96))
    h = o.adaln_modulate(x, z, z, tokens_per_sample=9, eps=1e-6)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (96,), eps=1e-6).numpy()
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-12)


def test_adaln_normalized_rows_have_zero_mean_and_known_variance():
    rng = np.random.default_rng(32)
    x = rng.standard_normal((5, 64)) * 7 - 3
    z = np.zeros((1, 64))
    eps = 0.25
    h = o.adaln_modulate(x, z, z, 5, eps)
    var = x.var(axis=1)
    np.testing.assert_allclose(h.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(h.var(axis=1), var / (var + eps), rtol=1e-12)


def test_adaln_constant_row_gives_the_shift_and_samples_take_their_own_rows():
    """A constant row normalizes to 0, so h = shift[b]; rows [b T, (b+1) T)
    use sample b's shift and scale."""
    d, T = 32, 3
    x = np.full((7, d), 2.5)
    shift = np.arange(3 * d, dtype=np.float64).reshape(3, d)
    scale = np.full((3, d), 9.0)
    h = o.adaln_modulate(x, shift, scale, T, 1e-6)
    for m in range(7):
        np.testing.assert_array_equal(h[m], shift[m // T])
    # with a non-constant row the scale of its own sample applies
    x = np.tile(np.array([1.0, -1.0] * (d // 2)), (4, 1))          # mean 0, var 1
    scale = np.array([[0.0] * d, [1.0] * d])
    h = o.adaln_modulate(x, np.zeros((2, d)), scale, 2, 0.0)
    np.testing.assert_allclose(h[:2], x[:2], rtol=1e-15)
    np.testing.assert_allclose(h[2:], 2 * x[2:], rtol=1e-15)


def test_quantize_adaln_with_identity_factors_quantizes_the_modulated_rows():
    """G_k = I: the fused path is MXFP4 of AdaLN(x) itself.  A row of +-1
    (mean 0, variance 1) with scale 1, shift 0 and eps 0 gives h = +-2
    exactly: amax 2, e = floor(log2 2) - 2 = -1 (byte 126), 2 / 2^-1 = 4 is
    code 6, with the sign of x."""
    d = 64
    vals = np.array([1.0, -1.0] * (d // 2), dtype=np.float32)
    xb = ((vals.view(np.uint32) >> 16).astype(np.uint16))[None, :]
    one = ((np.full((1, d), 1.0, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16))
    zero = np.zeros((1, d), dtype=np.uint16)
    p = np.zeros((2, 5, 3), dtype=np.float32)
    p[:, :, 1] = 1.0
    q, s = o.quantize_adaln(xb, zero, one, 1, 0.0, p)
    assert list(s[0]) == [126, 126]
    codes = o.unpack_codes(q)[0]
    assert (codes[0::2] == 6).all() and (codes[1::2] == 0xE).all()


def test_adaln_terms_bound_the_modulated_values():
    """|h| <= terms everywhere (the terms are the magnitudes h is summed
    from), with equality-level tightness on a row of one sign."""
    rng = np.random.default_rng(33)
    x = rng.standard_normal((6, 64)) * 4
    shift = rng.standard_normal((2, 64))
    scale = rng.standard_normal((2, 64))
    h = o.adaln_modulate(x, shift, scale, 3, 1e-6)
    t = o.adaln_terms(x, shift, scale, 3, 1e-6)
    assert (np.abs(h) <= t * (1 + 1e-12)).all()


# ------------------------------------------------ tensor-core scale layout
def test_scales_to_mma_places_every_byte_once_and_pads_with_zero():
    rows, ns = 130, 6                          # two row tiles, two scale tiles
    s = (np.arange(rows * ns) % 251 + 1).astype(np.uint8).reshape(rows, ns)
    t = o.scales_to_mma(s)
    assert t.size == 2 * 2 * 512
    assert np.count_nonzero(t) == rows * ns    # every (nonzero) byte once, padding zero
    np.testing.assert_array_equal(o.scales_from_mma(t, rows, ns), s)


def test_scales_to_mma_hand_positions():
    """Row 33 (r0 = 1, r1 = 1), scale 5 (tile column 1, i = 1) of a 1-tile-
    high array with 8 scale columns: tile 1, byte 16 + 4 + 1 = 21."""
    s = np.zeros((40, 8), dtype=np.uint8)
    s[33, 5] = 7
    t = o.scales_to_mma(s)
    assert np.flatnonzero(t).tolist() == [512 + 21]
    s = np.zeros((400, 4), dtype=np.uint8)
    s[256 + 100, 2] = 9                        # tile row 2: r0 = 4, r1 = 3
    assert np.flatnonzero(o.scales_to_mma(s)).tolist() == [2 * 512 + 16 * 4 + 4 * 3 + 2]


def test_fold_weight16_keeps_the_layer_output_eq1():
    rng = np.random.default_rng(41)
    p16 = w.draw_params16(64, seed=42)
    x = rng.standard_normal((5, 64))
    W = rng.standard_normal((7, 64))
    lhs = o.transform16(x, p16) @ o.fold_weight16(W, p16).T
    np.testing.assert_allclose(lhs, x @ W.T, rtol=1e-10, atol=1e-10)


def test_quantize_weight16_with_identity_or_orthonormal_factors():
    """With G_k = I the 16-element fold is the identity, so the block-16
    weight quantizer gives quantize16's bytes on the same bf16 matrix; with
    an orthonormal block (K^-T = K) it quantizes the transformed rows."""
    rng = np.random.default_rng(43)
    W = rng.standard_normal((10, 64)).astype(np.float32)
    W[:, 5] *= 40.0
    Wb = (W.view(np.uint32) >> 16).astype(np.uint16)
    p = np.zeros((4, 4, 3), dtype=np.float32)
    p[:, :, 1] = 1.0
    qw, sw = o.quantize_weight16(Wb, p)
    qa, sa = o.quantize16(Wb, p)
    assert sw.shape == (10, 4) and qw.shape == (10, 32)
    assert np.array_equal(qw, qa) and np.array_equal(sw, sa)
    s2 = 1 / math.sqrt(2)
    p = np.tile(np.array([-1.0, s2, s2], dtype=np.float32), (4, 4, 1))
    qw, sw = o.quantize_weight16(Wb, p)
    qa, sa = o.quantize16(Wb, p)
    assert np.array_equal(sw, sa)
    assert (o.unpack_codes(qw) != o.unpack_codes(qa)).mean() < 0.01


def test_block16_product_brute_force():
    """mxfp4_gemm with 16-element scale blocks against a triple loop over
    hand-decoded values."""
    rng = np.random.default_rng(43)
    M, N, K = 2, 3, 64
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    sa = rng.integers(120, 135, (M, K // 16), dtype=np.uint8)
    sb = rng.integers(120, 135, (N, K // 16), dtype=np.uint8)
    table = [0, 0.5, 1, 1.5, 2, 3, 4, 6]

    def val(code, s):
        v = table[int(code) & 7] * 2.0 ** (int(s) - 127)
        return -v if code & 8 else v

    C = o.mxfp4_gemm(_pack_hand(ca), sa, _pack_hand(cb), sb, block=16)
    for m in range(M):
        for n in range(N):
            assert C[m, n] == sum(val(ca[m, k], sa[m, k // 16]) * val(cb[n, k], sb[n, k // 16])
                                  for k in range(K))


def test_hadamard_cancelling_sum_is_exactly_zero():
    """x H_32 / sqrt(32) with x = e_0 + e_1: H[0][c] + H[1][c] is 2 for even c
    and 0 for odd c (Sylvester order: row 1 alternates signs), so the odd
    outputs are exact zeros and the even ones 2 / sqrt(32)."""
    x = np.zeros((1, 32))
    x[0, 0] = x[0, 1] = 1.0
    y = o.transform_hadamard(x)[0]
    assert (y[1::2] == 0.0).all()
    np.testing.assert_allclose(y[0::2], 2.0 / math.sqrt(32.0), rtol=1e-15)
