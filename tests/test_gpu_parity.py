"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Every case is seeded and synthetic (``workloads``); expected values come only
from ``oracle.kq_oracle``.  Reduced sizes are checked element by element;
the full DiT-shaped sizes run in the benchmark's launch configuration and are
checked on sampled rows plus a property that holds at any size (quantizing
the dequantized output reproduces it exactly).
"""
import numpy as np
import pytest
import torch

import workloads as w
from oracle import kq_oracle as o
from tests.parity import TOL, check_mx4, check_transform, check_transform_literal

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")
DEV = "cuda:0"


def _gpu(t):
    return t.to(DEV)


def _params_dev(p):
    return torch.from_numpy(np.ascontiguousarray(p)).to(DEV)


def _run_all_variants(x_bits, x_t, params, inv_s):
    """GPU outputs of the three quantizers and the transform for one input."""
    xd = _gpu(x_t)
    pd = _params_dev(params)
    sd = _params_dev(inv_s)
    q, s = kq.quantize(xd, pd)
    qh, sh = kq.quantize_hadamard(xd)
    qs, ss = kq.quantize_smooth(xd, sd)
    y = kq.transform(xd, pd)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in
            dict(q=q, s=s, qh=qh, sh=sh, qs=qs, ss=ss, y=y).items()}


def _check_rows(out, x_bits, params, inv_s, rows=None, bound_exemptions=True):
    """Oracle comparison on all rows, or on the given row indices."""
    if rows is not None:
        x_bits = x_bits[rows]
        out = {k: v[rows] for k, v in out.items()}
    x64 = o.bf16_bits_to_float64(x_bits)
    y64 = o.transform(x64, params)
    cond = o.abs_transform(x64, params)
    # kq_transform runs in double: the literal 1e-5 relative bound holds.
    check_transform_literal(out["y"], y64, cond)
    worst = check_transform(out["y"], y64, cond)
    st = check_mx4(out["q"], out["s"], y64, cond)
    yh = o.transform_hadamard(x64)
    sth = check_mx4(out["qh"], out["sh"], yh, o.abs_transform_hadamard(x64))
    ys = o.transform_smooth(x64, inv_s)
    # A single float32 product is exact on both sides: no tolerance band.
    sts = check_mx4(out["qs"], out["ss"], ys, np.zeros_like(ys), strict_zero_sign=True)
    assert sts["scale_exempt"] == 0 and sts["code_exempt"] == 0
    if bound_exemptions:
        # Boundary cases are rare on these inputs (about one element in ten
        # million at full size), and every difference lies inside the literal
        # band: within 1e-5 relative of an E2M1 midpoint or a power of two.
        for stats in (st, sth):
            assert stats["scale_exempt"] <= max(2, stats["blocks"] // 100000)
            assert stats["code_exempt"] <= max(4, stats["elements"] // 1000000)
            assert stats["scale_outside_literal"] == 0
            assert stats["code_outside_literal"] == 0
    return worst, st, sth


REDUCED_M = 67          # G = 67 * nb spans several 256-block tiles with a ragged tail


@pytest.mark.parametrize("key", w.all_case_keys(), ids=lambda k: f"{k[0]}-d{k[1]}-g{k[2]}")
def test_reduced_configs_elementwise(key):
    name, di, gi = key
    M = w.CONFIGS[name]["M"] if name == "tiny" else REDUCED_M
    c = w.make_case(name, di, gi, M=M)
    out = _run_all_variants(c.x_bits(), c.x, c.params, c.inv_s)
    worst, st, sth = _check_rows(out, c.x_bits(), c.params, c.inv_s)
    assert worst < TOL


def _sample_rows(M, seed):
    rng = np.random.default_rng(seed)
    rows = set(range(4)) | set(range(M - 4, M)) | set(rng.choice(M, 16, replace=False).tolist())
    return np.array(sorted(rows))


def _requantize_is_identity(q, s, M, d):
    """quantize(dequantize(q, s)) == (q, s) on the GPU, at any size: every
    dequantized value is exact in bf16 and re-quantizes to itself."""
    qd, sd = _gpu(torch.from_numpy(q)), _gpu(torch.from_numpy(s))
    deq = kq.dequantize(qd, sd)
    xb = deq.to(torch.bfloat16)
    assert torch.equal(xb.float(), deq)
    ones = torch.ones(d, dtype=torch.float32, device=DEV)
    q2, s2 = kq.quantize_smooth(xb, ones)
    assert torch.equal(s2, sd)
    assert torch.equal(q2, qd)


@pytest.mark.parametrize("key", w.all_case_keys(), ids=lambda k: f"{k[0]}-d{k[1]}-g{k[2]}")
def test_full_size_sampled_rows(key):
    name, di, gi = key
    c = w.make_case(name, di, gi)
    out = _run_all_variants(c.x_bits(), c.x, c.params, c.inv_s)
    rows = _sample_rows(c.M, c.seed)
    _check_rows(out, c.x_bits(), c.params, c.inv_s, rows=rows)
    _requantize_is_identity(out["q"], out["s"], c.M, c.d)


IMPLS = {"panel": kq.KQ_IMPL_PANEL, "tma": kq.KQ_IMPL_TMA, "direct": kq.KQ_IMPL_DIRECT,
         "mma": kq.KQ_IMPL_MMA, "warp": kq.KQ_IMPL_WARP}


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("key", [("sana", 1, 0), ("flux_schnell", 1, 2), ("tiny", 0, 0)],
                         ids=lambda k: f"{k[0]}-d{k[1]}-g{k[2]}")
def test_each_implementation_against_oracle(impl, key):
    name, di, gi = key
    c = w.make_case(name, di, gi, M=301 if name != "tiny" else 256)
    q, s = kq.quantize(_gpu(c.x), _params_dev(c.params), impl=IMPLS[impl])
    x64 = o.bf16_bits_to_float64(c.x_bits())
    st = check_mx4(q.cpu().numpy(), s.cpu().numpy(), o.transform(x64, c.params),
                   o.abs_transform(x64, c.params))
    assert st["scale_outside_literal"] == 0 and st["code_outside_literal"] == 0


@pytest.mark.parametrize("key", w.all_case_keys(), ids=lambda k: f"{k[0]}-d{k[1]}-g{k[2]}")
def test_tensor_core_transform_all_configs(key):
    """The tcgen05 path (dense K as three bf16 terms) on every config, with a
    ragged last 128-row tile."""
    name, di, gi = key
    c = w.make_case(name, di, gi, M=200 if name != "tiny" else 256)
    q, s = kq.quantize(_gpu(c.x), _params_dev(c.params), impl=kq.KQ_IMPL_MMA)
    x64 = o.bf16_bits_to_float64(c.x_bits())
    st = check_mx4(q.cpu().numpy(), s.cpu().numpy(), o.transform(x64, c.params),
                   o.abs_transform(x64, c.params))
    assert st["scale_exempt"] <= max(2, st["blocks"] // 100000)
    assert st["code_exempt"] <= max(4, st["elements"] // 1000000)
    assert st["scale_outside_literal"] == 0 and st["code_outside_literal"] == 0


def test_table_implementations_agree_bitwise():
    """The flat TMA and the direct kernel run the same four-term stages."""
    c = w.make_case("sana", 1, M=301)
    xd, pd = _gpu(c.x), _params_dev(c.params)
    q1, s1 = kq.quantize(xd, pd, impl=kq.KQ_IMPL_TMA)
    q2, s2 = kq.quantize(xd, pd, impl=kq.KQ_IMPL_DIRECT)
    assert torch.equal(q1, q2) and torch.equal(s1, s2)


def test_singular_shear_factor_takes_the_plain_form():
    """(a, b, c) = (-1, 1, 1) gives G = [[1, 1], [-1, 0]] (det 1, g11 = 0):
    the scaled-shear form cannot hold it, so its panel runs the plain
    four-term stages; the other panels keep the shear form."""
    c = w.make_case("flux_schnell", 0, 0, M=150)
    p = c.params.copy()
    p[5, 2] = [-1.0, 1.0, 1.0]                 # block 5, factor G3
    p[90, 0] = [-1.0, 1.0, 1.0]                # a block in another panel
    pd = _params_dev(p)
    xd = _gpu(c.x)
    q, s = kq.quantize(xd, pd)
    y = kq.transform(xd, pd)
    x64 = o.bf16_bits_to_float64(c.x_bits())
    y64 = o.transform(x64, p)
    cond = o.abs_transform(x64, p)
    check_transform_literal(y.cpu().numpy(), y64, cond)
    check_mx4(q.cpu().numpy(), s.cpu().numpy(), y64, cond)


def test_panel_kernel_one_and_many_thread_rows_per_block():
    """The panel kernel at widths where many thread-rows of a CTA share each
    column block (36 blocks: 32 rows; 144 blocks: 8) and where one does (229
    blocks, a prime width: the whole row is one panel), and with the plain
    form forced on one panel by a singular factor in block 7: each matches
    the oracle."""
    for nb, M, singular in ((36, 131, False), (144, 37, False), (229, 9, False), (36, 70, True)):
        d = nb * 32
        x = w.random_bf16((M, d), seed=nb + M)
        p = w.draw_params(d, 4)
        if singular:
            p = p.copy()
            p[7, 1] = [-1.0, 1.0, 1.0]
        q, s = kq.quantize(_gpu(x), _params_dev(p), impl=kq.KQ_IMPL_PANEL)
        torch.cuda.synchronize()
        x64 = o.bf16_bits_to_float64(x.view(torch.int16).numpy().view(np.uint16))
        y64 = o.transform(x64, p)
        st = check_mx4(q.cpu().numpy(), s.cpu().numpy(), y64, o.abs_transform(x64, p))
        assert st["scale_exempt"] <= 2 and st["code_exempt"] <= max(4, st["elements"] // 10000)


# ------------------------------------------------------------- edge cases
def _edge(x_t, params, inv_s=None, bound=True):
    if inv_s is None:
        inv_s = np.ones(x_t.shape[1], dtype=np.float32)
    out = _run_all_variants(None, x_t, params, inv_s)
    bits = x_t.view(torch.int16).numpy().view(np.uint16)
    _check_rows(out, bits, params, inv_s, bound_exemptions=bound)
    return out


def test_single_block():
    x = w.random_bf16((1, 32), seed=1)
    _edge(x, w.draw_params(32, 1))


def test_wide_and_prime_width_rows():
    """512 blocks (one 256-wide panel pair), 513 = 27 * 19 (57-wide panels)
    and 521 blocks (prime: no useful panel, the flat TMA/direct path)."""
    for nb in (512, 513, 521):
        d = nb * 32
        x = w.random_bf16((5, d), seed=d)
        _edge(x, w.draw_params(d, 2))


def test_zero_subnormal_and_huge_blocks():
    d = 128
    x = np.zeros((4, d), dtype=np.float32)
    x[1, 32:64] = 2.0 ** -133                  # bf16 subnormals
    x[1, 64:96] = -(2.0 ** -130)
    x[2, :] = np.linspace(-1e30, 1e30, d)
    x[3, 0:32] = -0.0
    x[3, 32] = 1e-38
    t = torch.from_numpy(x).to(torch.bfloat16)
    out = _edge(t, w.draw_params(d, 3), bound=False)
    assert (out["s"][0] == 0).all() and (out["q"][0] & 0x77 == 0).all()


def test_exact_ties_and_signed_zero_through_smooth():
    """Grid points and midpoints (exact in bf16) with unit scale: every E2M1
    tie is decided on identical float32 values on both sides."""
    vals = [0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7.5,
            -0.0, -.25, -.75, -5, -6, -1, -0.125, 0.125, 2.25, -3.5, 0.0625, -7.5,
            1.0, 0.5, 3.0, -4.0]
    base = np.array(vals, dtype=np.float32)
    rows = [base * np.float32(2.0 ** k) for k in (-20, -1, 0, 3, 60)]
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    assert torch.equal(x.float(), torch.from_numpy(np.stack(rows)))
    _edge(x, w.draw_params(32, 4))


def test_empty_input_is_a_no_op():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    p = _params_dev(w.draw_params(64, 5))
    q, s = kq.quantize(x, p)
    assert q.shape == (0, 32) and s.shape == (0, 2)


def test_more_than_2_31_elements():
    """Offsets past 2^31 elements (4.3 GB of bf16) in the TMA path."""
    M, d = (1 << 17) + 3, 16384
    x = w.device_randn_bf16((M, d), seed=77, device=DEV)
    p = w.draw_params(d, 6)
    pd = _params_dev(p)
    q, s = kq.quantize(x, pd)
    torch.cuda.synchronize()
    rows = np.array([0, 1, (1 << 17) - 1, M - 2, M - 1])
    xb = x[torch.from_numpy(rows).to(DEV)].cpu()
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    x64 = o.bf16_bits_to_float64(bits)
    y64 = o.transform(x64, p)
    check_mx4(q[torch.from_numpy(rows).to(DEV)].cpu().numpy(),
              s[torch.from_numpy(rows).to(DEV)].cpu().numpy(), y64, o.abs_transform(x64, p))
    del x, q, s
    torch.cuda.empty_cache()


# ------------------------------------------------------- auxiliary entries
def test_dequantize_exhaustive():
    """Every code byte under every scale byte, bit-exact (NaN for 0xFF)."""
    q = np.tile(np.arange(256, dtype=np.uint8), (256, 1))          # [256, 256] -> d = 512
    s = np.repeat(np.arange(256, dtype=np.uint8)[:, None], 16, axis=1)
    y = kq.dequantize(_gpu(torch.from_numpy(q)), _gpu(torch.from_numpy(s))).cpu().numpy()
    with np.errstate(over="ignore"):
        ref = o.dequantize(q, s).astype(np.float32)
    nan = np.isnan(ref)
    assert (np.isnan(y) == nan).all()
    assert np.array_equal(y[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_inverse_transform_and_round_trip():
    c = w.make_case("flux_schnell", 0, 1, M=97)
    pd = _params_dev(c.params)
    rng = np.random.default_rng(9)
    yr = (rng.standard_normal((97, c.d)) * 3).astype(np.float32)
    xg = kq.inverse_transform(_gpu(torch.from_numpy(yr)), pd).cpu().numpy()
    y64 = yr.astype(np.float64)
    check_transform_literal(xg, o.inverse_transform(y64, c.params),
                            o.abs_inverse_transform(y64, c.params))
    yt = kq.transform(_gpu(c.x), pd)
    back = kq.inverse_transform(yt, pd).cpu().numpy()
    x64 = o.bf16_bits_to_float64(c.x_bits())
    # two float32 passes: bound by the magnitudes each pass sums
    cond2 = o.abs_inverse_transform(o.abs_transform(x64, c.params), c.params)
    check_transform(back, x64, cond2, tol=2 * TOL)


def test_invalid_arguments_are_rejected_on_device():
    lib = kq.lib()
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    q = torch.zeros((4, 32), dtype=torch.uint8, device=DEV)
    s = torch.zeros((4, 2), dtype=torch.uint8, device=DEV)
    p = _params_dev(w.draw_params(64, 7))
    assert lib.kq_quantize(x.data_ptr(), 4, 48, p.data_ptr(), q.data_ptr(), s.data_ptr(), None) == 1
    assert lib.kq_quantize(x.data_ptr() + 2, 4, 64, p.data_ptr(), q.data_ptr(), s.data_ptr(),
                           None) == 1
    assert lib.kq_quantize_ex(x.data_ptr(), 4, 64, p.data_ptr(), q.data_ptr(), s.data_ptr(), 9,
                              None) == 1


def test_no_device_wait_gave_up():
    assert kq.device_status() == 0
