"""Randomised shapes: every implementation against the oracle on seeded
random (M, d) pairs, including one-row inputs, widths with few or prime
numbers of blocks, and ragged tiles."""
import numpy as np
import pytest
import torch

import workloads as w
from oracle import kq_oracle as o
from tests.parity import check_mx4

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")

IMPLS = [kq.KQ_IMPL_AUTO, kq.KQ_IMPL_PANEL, kq.KQ_IMPL_TMA, kq.KQ_IMPL_DIRECT, kq.KQ_IMPL_MMA,
         kq.KQ_IMPL_WARP]


def _shapes():
    rng = np.random.default_rng(2024)
    shapes = [(1, 32), (1, 64), (3, 96), (129, 32 * 7), (300, 32 * 13), (257, 32 * 160)]
    for _ in range(10):
        shapes.append((int(rng.integers(1, 400)), 32 * int(rng.integers(1, 420))))
    return shapes


@pytest.mark.parametrize("shape", _shapes(), ids=lambda s: f"{s[0]}x{s[1]}")
def test_random_shape_all_implementations(shape):
    M, d = shape
    x = w.random_bf16((M, d), seed=M * 7919 + d, scale=3.0)
    p = w.draw_params(d, seed=d)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    x64 = o.bf16_bits_to_float64(bits)
    y64, cond = o.transform(x64, p), o.abs_transform(x64, p)
    xd, pd = x.cuda(), torch.from_numpy(p).cuda()
    ran = 0
    for impl in IMPLS:
        try:
            q, s = kq.quantize(xd, pd, impl=impl)
        except kq.KQError as err:
            # an explicit implementation may decline a shape it cannot tile
            assert impl != kq.KQ_IMPL_AUTO and err.status == 1, err
            continue
        ran += 1
        check_mx4(q.cpu().numpy(), s.cpu().numpy(), y64, cond)
    assert ran >= 2
