"""Failure detection without a GPU fault: a bounded in-kernel wait on a
barrier that nothing completes gives up, reports through the device error
word, and the context stays usable for real work afterwards."""
import numpy as np
import pytest
import torch

import workloads as w
from oracle import kq_oracle as o
from tests.parity import check_mx4

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")


def test_wait_that_runs_out_is_reported_and_cleared():
    assert kq.device_status() == 0
    lib = kq.lib()
    assert lib.kq_selftest_wait_timeout(torch.cuda.current_stream().cuda_stream) == 0
    flags = kq.device_status()
    assert flags == 4                     # KQ_DEVERR_SELFTEST only
    assert kq.device_status() == 0        # read-and-clear


def test_device_usable_after_the_timeout():
    lib = kq.lib()
    lib.kq_selftest_wait_timeout(None)
    kq.device_status()
    c = w.make_case("tiny")
    q, s = kq.quantize(c.x.cuda(), torch.from_numpy(c.params).cuda())
    x64 = o.bf16_bits_to_float64(c.x_bits())
    check_mx4(q.cpu().numpy(), s.cpu().numpy(), o.transform(x64, c.params),
              o.abs_transform(x64, c.params))
    assert kq.device_status() == 0
