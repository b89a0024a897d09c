"""kq_quantize_host: host-resident activations streamed through a device
workspace give exactly what kq_quantize gives on device-resident ones."""
import numpy as np
import pytest
import torch

import workloads as w

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")


def _host_run(c, ws_bytes, stream=None):
    x = c.x.pin_memory()
    p = torch.from_numpy(c.params).cuda()
    q = torch.empty((c.M, c.d // 2), dtype=torch.uint8).pin_memory()
    s = torch.empty((c.M, c.d // 32), dtype=torch.uint8).pin_memory()
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    kq.quantize_host(x, p, q, s, ws, stream=stream)
    torch.cuda.synchronize()
    return q, s


@pytest.mark.parametrize("rows_per_chunk", [1, 7, 100, 100000])
def test_host_pipeline_matches_device_path(rows_per_chunk):
    c = w.make_case("sana", 1, M=301)
    ws_bytes = kq.host_workspace_bytes(c.d, rows_per_chunk)
    q, s = _host_run(c, ws_bytes)
    qd, sd = kq.quantize(c.x.cuda(), torch.from_numpy(c.params).cuda())
    assert torch.equal(q, qd.cpu()) and torch.equal(s, sd.cpu())


def test_host_pipeline_twice_in_a_row_on_a_side_stream():
    c = w.make_case("flux_schnell", 1, 2, M=333)
    st = torch.cuda.Stream()
    ws_bytes = kq.host_workspace_bytes(c.d, 50)
    with torch.cuda.stream(st):
        q1, s1 = _host_run(c, ws_bytes, stream=st.cuda_stream)
        q2, s2 = _host_run(c, ws_bytes, stream=st.cuda_stream)
    qd, sd = kq.quantize(c.x.cuda(), torch.from_numpy(c.params).cuda())
    for q, s in ((q1, s1), (q2, s2)):
        assert torch.equal(q, qd.cpu()) and torch.equal(s, sd.cpu())


def test_full_stress_shape_through_host_memory():
    c = w.make_case("stress")
    q, s = _host_run(c, 64 << 20)
    qd, sd = kq.quantize(c.x.cuda(), torch.from_numpy(c.params).cuda())
    assert torch.equal(q, qd.cpu()) and torch.equal(s, sd.cpu())
