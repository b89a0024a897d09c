"""kq_quantize_host_static, the entry point for callers that cannot allocate
device memory (for example a serving process whose memory pool already holds
nearly all of the GPU, where cudaMalloc could fail or stall the device): it
must give exactly what the workspace-based kq_quantize_host gives, on two
calls in a row through the same built-in staging area.  Called through the
C ABI.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as w

pytestmark = pytest.mark.gpu


def _lib():
    from w4a4_post_quantization_b200 import _lib as L
    return L.lib()


def _run(fn_name, c, lib, stream, workspace=None):
    x = c.x.pin_memory()
    p = torch.from_numpy(c.params).cuda()
    q = torch.full((c.M, c.d // 2), 0xAB, dtype=torch.uint8).pin_memory()
    s = torch.full((c.M, c.d // 32), 0xCD, dtype=torch.uint8).pin_memory()
    if workspace is None:
        rc = getattr(lib, fn_name)(x.data_ptr(), c.M, c.d, p.data_ptr(), q.data_ptr(),
                                   s.data_ptr(), stream)
    else:
        rc = getattr(lib, fn_name)(x.data_ptr(), c.M, c.d, p.data_ptr(), q.data_ptr(),
                                   s.data_ptr(), workspace.data_ptr(), workspace.numel(), stream)
    assert rc == 0, lib.kq_status_string(rc)
    torch.cuda.synchronize()
    return q, s


def test_static_staging_matches_workspace_entry_twice():
    lib = _lib()
    stream = torch.cuda.current_stream().cuda_stream
    # 2000 rows of width 12288 need several passes through the 16 MiB area.
    cases = [w.make_case("stress", M=2000), w.make_case("sana", 1, M=777)]
    for c in cases:
        ws = torch.empty(lib.kq_quantize_host_workspace_bytes(c.d, 256), dtype=torch.uint8,
                         device="cuda")
        q_ref, s_ref = _run("kq_quantize_host", c, lib, stream, workspace=ws)
        for _ in range(2):
            q, s = _run("kq_quantize_host_static", c, lib, stream)
            assert torch.equal(q, q_ref) and torch.equal(s, s_ref)


def test_static_staging_rejects_rows_too_wide():
    lib = _lib()
    d = 32 * ((16 << 20) // 64)            # one row of x alone fills the area
    rc = lib.kq_quantize_host_static(ctypes.c_void_p(0x10000), 1, d, ctypes.c_void_p(0x10000),
                                     ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), None)
    assert rc == 1
