"""GPU parity of the fused LayerNorm + AdaLN modulation + transform + MXFP4
path (kq_quantize_adaln / kq_transform_adaln) against the CPU oracle.

The modulated value h is a sum of terms whose magnitudes add to
``(|x| + mean|x|) rstd |1 + scale| + |shift|`` (``oracle.adaln_terms``); the
transformed value's tolerance band is 1e-5 times those magnitudes carried
through ``|K|``, the same componentwise rule as the quantizer alone.
"""
import numpy as np
import pytest
import torch

import workloads as w
from oracle import kq_oracle as o
from tests.parity import TOL, check_mx4, check_transform

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")
DEV = "cuda:0"
EPS = 1e-6


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _run(x, shift, scale, T, params, eps=EPS):
    xd, sd, cd = x.to(DEV), shift.to(DEV), scale.to(DEV)
    pd = torch.from_numpy(np.ascontiguousarray(params)).to(DEV)
    q, s = kq.quantize_adaln(xd, sd, cd, T, pd, eps)
    y = kq.transform_adaln(xd, sd, cd, T, pd, eps)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), y.cpu().numpy()


def _check(x, shift, scale, T, params, q, s, y, rows=None, eps=EPS, bound=True):
    x64 = o.bf16_bits_to_float64(_bits(x))
    sh64 = o.bf16_bits_to_float64(_bits(shift))
    sc64 = o.bf16_bits_to_float64(_bits(scale))
    h = o.adaln_modulate(x64, sh64, sc64, T, eps)
    terms = o.adaln_terms(x64, sh64, sc64, T, eps)
    if rows is not None:
        h, terms, q, s, y = h[rows], terms[rows], q[rows], s[rows], y[rows]
    y64 = o.transform(h, params)
    cond = o.abs_transform(terms, params)
    worst = check_transform(y, y64, cond)
    st = check_mx4(q, s, y64, cond)
    if bound:
        assert st["scale_exempt"] <= max(2, st["blocks"] // 1000)
        assert st["code_exempt"] <= max(4, st["elements"] // 10000)
    return worst


@pytest.mark.parametrize("key", w.all_case_keys(), ids=lambda k: f"{k[0]}-d{k[1]}-g{k[2]}")
def test_adaln_reduced_configs_elementwise(key):
    """First 67 rows (256 for tiny) with 16 tokens per sample, so that the
    sample changes inside a CTA's row groups."""
    name, di, gi = key
    M = 256 if name == "tiny" else 67
    c = w.make_case(name, di, gi, M=M)
    T = 16
    shift, scale = w.draw_adaln(-(-M // T), c.d, c.seed)
    q, s, y = _run(c.x, shift, scale, T, c.params)
    assert _check(c.x, shift, scale, T, c.params, q, s, y) < TOL


@pytest.mark.parametrize("name,di", [("stress", 0), ("flux_schnell", 1), ("pixart_sigma", 0)])
def test_adaln_full_size_sampled_rows(name, di):
    c = w.make_case(name, di, 0)
    T = w.TOKENS_PER_SAMPLE[name]
    shift, scale = w.draw_adaln(-(-c.M // T), c.d, c.seed)
    q, s, y = _run(c.x, shift, scale, T, c.params)
    rng = np.random.default_rng(c.seed)
    rows = np.array(sorted({0, 1, T - 1, min(T, c.M - 1), c.M - 1} |
                           set(rng.choice(c.M, 10, replace=False).tolist())))
    _check(c.x, shift, scale, T, c.params, q, s, y, rows=rows)


@pytest.mark.parametrize("d", [32, 64, 32 * 37, 32 * 383, 12288])
def test_adaln_widths(d):
    """One block per row (256 rows per group) up to 384 blocks (one row per
    group), and block counts that leave threads idle."""
    M, T = 70, 9
    x = w.random_bf16((M, d), seed=d, scale=3.0)
    shift, scale = w.draw_adaln(-(-M // T), d, seed=d)
    p = w.draw_params(d, seed=d)
    q, s, y = _run(x, shift, scale, T, p)
    _check(x, shift, scale, T, p, q, s, y)


def test_adaln_constant_rows_and_large_mean():
    """A constant row normalizes to 0 (h = shift); a row with a large common
    offset normalizes like the offset-free row."""
    d, M, T = 256, 8, 4
    x = w.random_bf16((M, d), seed=3).float()
    x[0] = 5.0
    x[1] = -2.0
    x[2] += 1000.0
    xb = x.to(torch.bfloat16)
    shift, scale = w.draw_adaln(2, d, seed=4)
    p = w.draw_params(d, seed=5)
    q, s, y = _run(xb, shift, scale, T, p, eps=1e-5)
    _check(xb, shift, scale, T, p, q, s, y, eps=1e-5, bound=False)


def test_adaln_plain_form_fallback():
    c = w.make_case("pixart_sigma", 0, 0, M=40)
    p = c.params.copy()
    p[7, 2] = [-1.0, 1.0, 1.0]
    shift, scale = w.draw_adaln(3, c.d, c.seed)
    q, s, y = _run(c.x, shift, scale, 16, p)
    _check(c.x, shift, scale, 16, p, q, s, y)


def test_adaln_identity_modulation_matches_quantize_of_layer_norm():
    """scale = shift = 0 and identity factors: the codes are the MXFP4 of
    LayerNorm(x) as the oracle computes it."""
    c = w.make_case("sana", 0, 0, M=64)
    z = torch.zeros((1, c.d), dtype=torch.bfloat16)
    p = np.zeros((c.d // 32, 5, 3), dtype=np.float32)
    p[:, :, 1] = 1.0
    q, s, y = _run(c.x, z, z, 64, p)
    _check(c.x, z, z, 64, p, q, s, y)


def test_adaln_rejects_bad_arguments_and_no_wait_gave_up():
    lib = kq.lib()
    st = torch.cuda.current_stream().cuda_stream
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    sh = torch.zeros((1, 64), dtype=torch.bfloat16, device=DEV)
    p = torch.zeros((2, 5, 3), dtype=torch.float32, device=DEV)
    q = torch.empty((4, 32), dtype=torch.uint8, device=DEV)
    s = torch.empty((4, 2), dtype=torch.uint8, device=DEV)
    assert lib.kq_quantize_adaln(x.data_ptr(), 4, 64, sh.data_ptr(), sh.data_ptr(), 0, 1e-6,
                                 p.data_ptr(), q.data_ptr(), s.data_ptr(), st) == 1
    assert lib.kq_quantize_adaln(x.data_ptr(), 4, 64, sh.data_ptr() + 2, sh.data_ptr(), 4, 1e-6,
                                 p.data_ptr(), q.data_ptr(), s.data_ptr(), st) == 1
    assert kq.device_status() == 0


@pytest.mark.parametrize("name,di,T", [("pixart_sigma", 0, 128), ("flux_schnell", 1, 75)])
def test_adaln_tiled_scales_feed_the_tiled_gemm(name, di, T):
    """kq_quantize_adaln_tiled writes the same codes and the tiled image of
    the row-major scales; the normalized layer's product through the tiled
    GEMM equals the row-major one bit for bit.  The wide case pairs a
    thread's two rows and straddles samples (75 tokens a sample)."""
    c = w.make_case(name, di, 0, M=300)
    shift, scale = w.draw_adaln(-(-c.M // T), c.d, c.seed)
    xd, sd, cd = c.x.to(DEV), shift.to(DEV), scale.to(DEV)
    pd = torch.from_numpy(c.params).to(DEV)
    q, s = kq.quantize_adaln(xd, sd, cd, T, pd)
    qt, st = kq.quantize_adaln_tiled(xd, sd, cd, T, pd)
    torch.cuda.synchronize()
    assert torch.equal(q, qt)
    assert np.array_equal(st.cpu().numpy(), o.scales_to_mma(s.cpu().numpy()))
    W = w.draw_weight(512, c.d, c.seed).to(DEV)
    qb, sb = kq.quantize_weight(W, pd)
    qbt, sbt = kq.quantize_weight_tiled(W, pd)
    assert torch.equal(kq.gemm_mxfp4(q, s, qb, sb), kq.gemm_mxfp4_tiled(qt, st, qbt, sbt))
