"""The launches survive CUDA-graph stream capture (they use programmatic
dependent launch, which capture must accept) and the replayed graph gives
the eager results bit for bit."""
import numpy as np
import pytest
import torch

import workloads as w

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")
DEV = "cuda:0"


def test_quantizer_gemm_and_adaln_replay_from_a_graph():
    c = w.make_case("flux_schnell", 0, 0, M=512)
    x = c.x.to(DEV)
    p = torch.from_numpy(c.params).to(DEV)
    wt = w.draw_weight(768, c.d, c.seed).to(DEV)
    shift, scale = (t.to(DEV) for t in w.draw_adaln(1, c.d, c.seed))
    # Eager results.
    q0, s0 = kq.quantize(x, p)
    qa0, sa0 = kq.quantize_tiled(x, p)
    qb0, sb0 = kq.quantize_weight_tiled(wt, p)
    y0 = kq.gemm_mxfp4_tiled(qa0, sa0, qb0, sb0, out_dtype=torch.bfloat16)
    qh0, sh0 = kq.quantize_adaln(x, shift, scale, 512, p, 1e-6)
    torch.cuda.synchronize()
    # The same calls captured into one graph, on preallocated outputs.
    q, s = torch.empty_like(q0), torch.empty_like(s0)
    qa, sa = torch.empty_like(qa0), torch.empty_like(sa0)
    qb, sb = torch.empty_like(qb0), torch.empty_like(sb0)
    y = torch.empty_like(y0)
    qh, sh = torch.empty_like(qh0), torch.empty_like(sh0)
    stream = torch.cuda.Stream(DEV)
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        kq.quantize(x, p, q, s)                   # warm the stream once outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            kq.quantize(x, p, q, s)
            kq.quantize_tiled(x, p, qa, sa)
            kq.quantize_weight_tiled(wt, p, qb, sb)
            kq.gemm_mxfp4_tiled(qa, sa, qb, sb, out=y, out_dtype=torch.bfloat16)
            kq.quantize_adaln(x, shift, scale, 512, p, 1e-6, qh, sh)
    for t in (q, s, qa, sa, qb, sb, y, qh, sh):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for a, b in ((q, q0), (s, s0), (qa, qa0), (sa, sa0), (qb, qb0), (sb, sb0), (y, y0), (qh, qh0),
                 (sh, sh0)):
        assert torch.equal(a, b)
    assert kq.device_status() == 0
    del g
