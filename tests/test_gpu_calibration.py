"""GPU parity of the calibration kernels and of the calibration loop against
the CPU oracle (``oracle.kq_calibration``).

Tolerances, from the arithmetic:

* parameter gradient: every entry is a sum of products u_p G_q over the
  rows, accumulated in float32 (at most a few hundred terms per thread, then
  two fixed-order sums), with the stage inputs u recovered from the float32
  transformed operand through one 2x2 inverse: the error is within
  (rows per thread + 64) 2^-24 kappa of the sum of the terms' magnitudes,
  kappa bounding |F||F^-1|; the test allows 1e-4 of that magnitude;
* residual: one float32 subtraction and one multiply per element, the sum of
  squares of the exact differences in double: 2 ulp elementwise and 1e-11
  relative for the sum;
* Adam: a handful of float32 operations per parameter, measured against the
  magnitudes of the terms each moment is made of (the updates can cancel),
  and 1e-5 of the step those magnitudes give plus 4 ulp for the parameter.
"""
import numpy as np
import pytest
import torch

import workloads as w
from oracle import kq_calibration as c
from oracle import kq_oracle as o

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")
from w4a4_post_quantization_b200 import calibrate as kc  # noqa: E402

DEV = "cuda:0"


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("inv", [False, True], ids=["activation", "weight"])
@pytest.mark.parametrize("M,d", [(67, 64), (300, 1152), (1000, 96)])
def test_params_grad_kernel(inv, M, d):
    x = w.random_bf16((M, d), seed=M + d, scale=2.0)
    p = w.draw_params(d, seed=d + 1)
    x64 = o.bf16_bits_to_float64(_bits(x))
    z64 = o.fold_weight(x64, p) if inv else o.transform(x64, p)
    z = z64.astype(np.float32)
    zq = c.fake_quant(z.astype(np.float64)).astype(np.float32)
    g = np.random.default_rng([M, d, 7]).standard_normal((M, d)).astype(np.float32)
    lam = 0.37
    ws = torch.zeros((kq.params_grad_workspace_bytes(M, d),), dtype=torch.uint8, device=DEV)
    for _ in range(2):                       # the workspace is reusable
        dp, reg = kq.transform_params_grad(_dev(z), _dev(zq), _dev(g), _dev(p), inv, lam, ws)
    torch.cuda.synchronize()
    G = g.astype(np.float64) + 2 * lam * (z.astype(np.float64) - zq.astype(np.float64))
    ref = c.transform_params_grad(x64, G, p, inverse_transpose=inv)
    mag = c.abs_transform_params_grad(x64, np.abs(G), p, inverse_transpose=inv)
    err = np.abs(dp.cpu().numpy().astype(np.float64) - ref)
    assert (err <= 1e-4 * mag + 1e-30).all(), float((err / np.maximum(mag, 1e-30)).max())
    reg_ref = np.sum((zq.astype(np.float64) - z.astype(np.float64)) ** 2)
    assert abs(float(reg.item()) - reg_ref) <= 1e-5 * reg_ref


def test_params_grad_is_deterministic():
    M, d = 2048, 384
    rng = np.random.default_rng(3)
    z = _dev(rng.standard_normal((M, d)).astype(np.float32))
    zq = _dev(rng.standard_normal((M, d)).astype(np.float32))
    g = _dev(rng.standard_normal((M, d)).astype(np.float32))
    p = _dev(w.draw_params(d, seed=4))
    ws = torch.zeros((kq.params_grad_workspace_bytes(M, d),), dtype=torch.uint8, device=DEV)
    a, ra = kq.transform_params_grad(z, zq, g, p, False, 0.5, ws)
    a, ra = a.clone(), ra.clone()
    b, rb = kq.transform_params_grad(z, zq, g, p, False, 0.5, ws)
    assert torch.equal(a, b) and torch.equal(ra, rb)


def test_residual_kernel():
    rng = np.random.default_rng(5)
    y = rng.standard_normal(100003).astype(np.float32)
    r = rng.standard_normal(100003).astype(np.float32)
    ws = torch.zeros((kq.residual_workspace_bytes(),), dtype=torch.uint8, device=DEV)
    out, ss = kq.residual(_dev(y), _dev(r), 0.25, ws)
    diff = y.astype(np.float64) - r.astype(np.float64)
    np.testing.assert_allclose(out.cpu().numpy(), (0.25 * diff).astype(np.float32), rtol=2.5e-7,
                               atol=0)
    assert abs(float(ss.item()) - np.sum(diff ** 2)) <= 1e-12 * np.sum(diff ** 2) * 10


def test_adam_kernel_matches_oracle():
    rng = np.random.default_rng(6)
    n = 3000
    p = rng.standard_normal(n).astype(np.float32)
    g0 = rng.standard_normal(n).astype(np.float32)
    g1 = (rng.standard_normal(n) * 0.1).astype(np.float32)
    m = (rng.standard_normal(n) * 0.01).astype(np.float32)
    v = (rng.random(n) * 0.01).astype(np.float32)
    pd, md, vd = _dev(p), _dev(m), _dev(v)
    kq.adam_step(pd, _dev(g0), _dev(g1), md, vd, 7, 1e-2)
    ref_p, ref_m, ref_v = c.adam_step(p.astype(np.float64), g0.astype(np.float64) +
                                      g1.astype(np.float64), m.astype(np.float64),
                                      v.astype(np.float64), 7, 1e-2)
    # Bounds against the magnitudes of the terms each value is made of (the
    # moment updates can cancel).
    u = 2.0 ** -24
    ga = np.abs(g0.astype(np.float64)) + np.abs(g1.astype(np.float64))
    m_terms = c.ADAM_BETA1 * np.abs(m) + (1 - c.ADAM_BETA1) * ga
    v_terms = c.ADAM_BETA2 * np.abs(v) + (1 - c.ADAM_BETA2) * ga * ga
    assert (np.abs(md.cpu().numpy() - ref_m) <= 6 * u * m_terms).all()
    assert (np.abs(vd.cpu().numpy() - ref_v) <= 8 * u * v_terms).all()
    corr1, corr2 = 1 - c.ADAM_BETA1 ** 7, 1 - c.ADAM_BETA2 ** 7
    step_terms = 1e-2 * (m_terms / corr1) / (np.sqrt(ref_v / corr2) + c.ADAM_EPS)
    assert (np.abs(pd.cpu().numpy() - ref_p) <= 1e-5 * step_terms +
            4 * np.spacing(np.abs(p))).all()


def _layer(M, d, N, seed, outliers=()):
    x = w.random_bf16((M, d), seed=seed).float()
    for ch, gain in outliers:
        x[:, ch] *= gain
    x = x.to(torch.bfloat16)
    wt = w.draw_weight(N, d, seed)
    return x, wt


def test_calibration_loop_matches_the_oracle():
    """Loss at the initialization (and the regularization weights from it)
    agree with the oracle; the first step's gradient moves the parameters
    the same way; ten steps lower the loss on both sides alike."""
    x, wt = _layer(256, 128, 96, seed=11, outliers=((5, 40.0), (70, 25.0)))
    x64, w64 = o.bf16_bits_to_float64(_bits(x)), o.bf16_bits_to_float64(_bits(wt))
    cal = kc.LayerCalibrator(x.to(DEV), wt.to(DEV))
    l_gpu = cal.losses()
    l_ref = c.losses(x64, w64, c.hadamard_params(4))
    for a, b in zip(l_gpu, l_ref):
        assert abs(a - b) <= 1e-3 * b, (l_gpu, l_ref)
    hist = cal.run(10)
    p_ref, hist_ref, _ = c.calibrate(x64, w64, steps=10)
    assert abs(hist[0] - hist_ref[0]) <= 2e-3 * hist_ref[0]
    assert hist[-1] < hist[0] and hist_ref[-1] < hist_ref[0]
    assert abs(hist[-1] - hist_ref[-1]) <= 0.05 * hist_ref[-1], (hist, hist_ref)
    # First-step direction: Adam's first update is lr sign(g) per parameter.
    cal1 = kc.LayerCalibrator(x.to(DEV), wt.to(DEV))
    cal1.run(1)
    d_gpu = cal1.params.cpu().numpy() - c.hadamard_params(4)
    p1, _, _ = c.calibrate(x64, w64, steps=1)
    d_ref = p1 - c.hadamard_params(4)
    agree = np.sign(d_gpu) == np.sign(d_ref)
    assert agree.mean() >= 0.95, agree.mean()


def test_calibration_improves_on_the_hadamard_initialization():
    """Outliers inside one 32-block: the calibrated transform's output error
    falls below the Hadamard initialization's."""
    x, wt = _layer(1024, 256, 256, seed=12, outliers=((3, 60.0), (9, 30.0), (100, 45.0)))
    cal = kc.LayerCalibrator(x.to(DEV), wt.to(DEV))
    l0 = cal.losses()[0]
    cal.run(100)
    l1 = cal.losses()[0]
    assert l1 < l0
    assert kq.device_status() == 0
