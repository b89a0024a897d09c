"""GPU parity of the weight-side fold ``W T^-T`` and its MXFP4 quantization
against the CPU oracle (review, "Circularity Check", Eq. 1: the inverse
transform is folded into the weights offline, so that
``(x T)(W T^-T)^T = x W^T``).

Weights are seeded synthetic ``N(0, 1/d)`` matrices (``workloads.draw_weight``)
with the activations' parameters for the same hidden size; expected values
come only from ``oracle.kq_oracle``.
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


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _run(W, params):
    wd = W.to(DEV)
    pd = torch.from_numpy(np.ascontiguousarray(params)).to(DEV)
    q, s = kq.quantize_weight(wd, pd)
    f = kq.fold_weight(wd, pd)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), f.cpu().numpy()


def _check(W, params, q, s, f, bound=True):
    w64 = o.bf16_bits_to_float64(_bits(W))
    f64 = o.fold_weight(w64, params)
    cond = o.abs_fold_weight(w64, params)
    check_transform_literal(f, f64, cond)
    worst = check_transform(f, f64, cond)
    st = check_mx4(q, s, f64, cond)
    if bound:
        assert st["scale_exempt"] <= max(2, st["blocks"] // 1000)
        assert st["code_exempt"] <= max(4, st["elements"] // 10000)
    return worst


# (layer, N) pairs shaped like DiT linear layers of each hidden size.
LAYERS = [("tiny", 0, 96), ("pixart_sigma", 0, 211), ("pixart_sigma", 1, 67),
          ("sana", 0, 150), ("sana", 1, 67), ("flux_schnell", 0, 133),
          ("flux_schnell", 1, 67), ("stress", 0, 67)]


@pytest.mark.parametrize("name,di,N", LAYERS, ids=lambda v: str(v))
def test_fold_and_quantize_weight_elementwise(name, di, N):
    c = w.make_case(name, di, 0, M=16)
    W = w.draw_weight(N, c.d, c.seed)
    q, s, f = _run(W, c.params)
    assert _check(W, c.params, q, s, f) < TOL


def test_fold_weight_plain_form_fallback():
    """(a, b, c) = (-1, 1, 1): G^-T has a zero diagonal entry, so the fold's
    shear form cannot hold it and that CTA takes the plain stages."""
    c = w.make_case("flux_schnell", 0, 0, M=16)
    p = c.params.copy()
    p[3, 1] = [-1.0, 1.0, 1.0]
    p[77, 4] = [-1.0, 1.0, 1.0]
    W = w.draw_weight(150, c.d, c.seed)
    q, s, f = _run(W, p)
    _check(W, p, q, s, f)


def test_eq1_through_the_gpu_fold():
    """(x T)(W T^-T)^T from the GPU's float32 transform and fold equals
    x W^T: the invariance holds within float32 rounding of both factors."""
    c = w.make_case("pixart_sigma", 0, 0, M=64)
    W = w.draw_weight(96, c.d, c.seed)
    pd = torch.from_numpy(c.params).to(DEV)
    y = kq.transform(c.x.to(DEV), pd).double().cpu().numpy()
    f = kq.fold_weight(W.to(DEV), pd).double().cpu().numpy()
    x64 = o.bf16_bits_to_float64(c.x_bits())
    w64 = o.bf16_bits_to_float64(_bits(W))
    lhs = y @ f.T
    ref = x64 @ w64.T
    # float32 errors of y and f, each within 1e-5 of their magnitude sums
    bound = 1e-5 * (o.abs_transform(x64, c.params) @ np.abs(f).T +
                    np.abs(y) @ o.abs_fold_weight(w64, c.params).T) + 1e-12
    assert (np.abs(lhs - ref) <= 2 * bound).all()


def test_weight_entries_reject_bad_arguments():
    lib = kq.lib()
    wd = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    p = torch.zeros((2, 5, 3), dtype=torch.float32, device=DEV)
    q = torch.empty((4, 32), dtype=torch.uint8, device=DEV)
    s = torch.empty((4, 2), dtype=torch.uint8, device=DEV)
    st = torch.cuda.current_stream().cuda_stream
    assert lib.kq_quantize_weight(wd.data_ptr() + 2, 4, 64, p.data_ptr(), q.data_ptr(),
                                  s.data_ptr(), st) == 1
    assert lib.kq_quantize_weight(wd.data_ptr(), 4, 60, p.data_ptr(), q.data_ptr(),
                                  s.data_ptr(), st) == 1
    assert lib.kq_quantize_weight(wd.data_ptr(), 0, 64, p.data_ptr(), q.data_ptr(),
                                  s.data_ptr(), st) == 0
