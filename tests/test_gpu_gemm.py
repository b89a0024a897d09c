"""GPU parity of the W4A4 MXFP4 product (block-scaled tcgen05 GEMM) against
the CPU oracle's exact product of the decoded operands.

Tolerance, from the arithmetic: every product A[m][k] B[n][k] of two E2M1
values and two E8M0 scales is exact, and the tensor core adds 64-term
partial sums into a float32 accumulator, one rounding per partial sum, so
``|C_gpu - C| <= (K/64 + 1) 2^-24 (|A| |B|^T)``; the test allows four times
that (``(K/64 + 1) 2^-22``), which also covers a partial sum formed with a
rounding of its own.  bf16 output is the float32 result rounded once.
"""
import numpy as np
import pytest
import torch

import workloads as w
from oracle import kq_oracle as o

pytestmark = pytest.mark.gpu

kq = pytest.importorskip("w4a4_post_quantization_b200")
DEV = "cuda:0"


def gemm_tol(K):
    return (K / 64 + 1) * 2.0 ** -22


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def random_operands(M, N, K, seed, s_lo=120, s_hi=135):
    rng = np.random.default_rng([seed, 31])
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qb = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(s_lo, s_hi, (M, K // 32), dtype=np.uint8)
    sb = rng.integers(s_lo, s_hi, (N, K // 32), dtype=np.uint8)
    return qa, sa, qb, sb


def check_gemm(c_gpu, qa, sa, qb, sb, rows=None):
    K = qa.shape[1] * 2
    if rows is not None:
        qa, sa, c_gpu = qa[rows], sa[rows], c_gpu[rows]
    ref = o.mxfp4_gemm(qa, sa, qb, sb)
    mag = o.abs_mxfp4_gemm(qa, sa, qb, sb)
    err = np.abs(np.asarray(c_gpu, dtype=np.float64) - ref)
    bound = gemm_tol(K) * mag
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{int(bad.sum())} outputs outside tolerance: " + str(
            [(tuple(i), float(c_gpu[tuple(i)]), float(ref[tuple(i)]), float(mag[tuple(i)]))
             for i in idx]))
    with np.errstate(invalid="ignore", divide="ignore"):
        r = np.where(mag > 0, err / np.where(mag > 0, mag, 1), 0)
    return float(r.max())


def run(qa, sa, qb, sb, out_dtype=torch.float32):
    c = kq.gemm_mxfp4(_dev(qa), _dev(sa), _dev(qb), _dev(sb), out_dtype=out_dtype)
    torch.cuda.synchronize()
    return c


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (130, 300, 544), (1, 8, 32), (257, 520, 1152),
                                   (64, 40, 2240), (300, 256, 96)])
def test_random_operands(M, N, K):
    """Random codes (all 16, both signs) and scales: tile edges in M and N,
    K not a multiple of the 256-element stage, scale rows not 4-byte
    multiples (K = 2240, 96)."""
    qa, sa, qb, sb = random_operands(M, N, K, seed=M * 7 + N + K)
    c = run(qa, sa, qb, sb).cpu().numpy()
    assert check_gemm(c, qa, sa, qb, sb) <= gemm_tol(K)


def test_exact_small_integer_products():
    """Codes of +-{0.5 .. 6} with unit scales and K = 64: every partial sum is
    a multiple of 0.25 below 2^11, exact in float32, so C is bit-exact."""
    qa, sa, qb, sb = random_operands(128, 256, 64, seed=5, s_lo=127, s_hi=128)
    c = run(qa, sa, qb, sb).cpu().numpy()
    assert np.array_equal(c.astype(np.float64), o.mxfp4_gemm(qa, sa, qb, sb))


def test_scales_select_the_right_block():
    """One nonzero scale block at a time: moving a single large scale along K
    (and across rows of A and B) must move the result with it, which pins
    the scale layout in tensor memory (row groups of 32, 4 scales per word,
    two words per stage)."""
    M, N, K = 160, 272, 512
    qa = np.full((M, K // 2), 0x22, dtype=np.uint8)       # every element 1.0
    qb = np.full((N, K // 2), 0x22, dtype=np.uint8)
    rng = np.random.default_rng(7)
    for trial in range(6):
        # every partial sum is a multiple of 2 below 2^15: exact in float32
        sa = np.full((M, K // 32), 127 - 4, dtype=np.uint8)
        sb = np.full((N, K // 32), 127, dtype=np.uint8)
        m, kb = int(rng.integers(M)), int(rng.integers(K // 32))
        n, kb2 = int(rng.integers(N)), int(rng.integers(K // 32))
        sa[m, kb] = 127 + 6
        sb[n, kb2] = 127 + 3
        c = run(qa, sa, qb, sb).cpu().numpy()
        assert np.array_equal(c.astype(np.float64), o.mxfp4_gemm(qa, sa, qb, sb)), (trial, m, kb,
                                                                                    n, kb2)


def test_bf16_output_is_the_rounded_float32_result():
    qa, sa, qb, sb = random_operands(200, 264, 640, seed=9)
    c32 = run(qa, sa, qb, sb)
    c16 = run(qa, sa, qb, sb, out_dtype=torch.bfloat16)
    assert torch.equal(c16, c32.to(torch.bfloat16))


@pytest.mark.parametrize("name,di,N", [("pixart_sigma", 0, 1152), ("sana", 0, 2240),
                                       ("flux_schnell", 0, 3072)], ids=lambda v: str(v))
def test_transformed_layer_end_to_end(name, di, N):
    """x -> kq_quantize, W -> kq_quantize_weight, then the GEMM: C matches
    the oracle's product of those operands, and the operands match the
    oracle's quantizers (checked elsewhere) -- here the product is checked on
    every output of a reduced token count."""
    c = w.make_case(name, di, 0, M=192)
    W = w.draw_weight(N, c.d, c.seed)
    pd = _dev(c.params)
    qa, sa = kq.quantize(c.x.to(DEV), pd)
    qb, sb = kq.quantize_weight(W.to(DEV), pd)
    C = kq.gemm_mxfp4(qa, sa, qb, sb)
    torch.cuda.synchronize()
    check_gemm(C.cpu().numpy(), qa.cpu().numpy(), sa.cpu().numpy(), qb.cpu().numpy(),
               sb.cpu().numpy())


def test_full_size_layer_sampled_rows():
    """FLUX-shaped MLP projection at full token count (4608 x 3072 -> 12288):
    sampled rows of C against the oracle."""
    c = w.make_case("flux_schnell", 0, 0)
    W = w.draw_weight(12288, c.d, c.seed)
    pd = _dev(c.params)
    qa, sa = kq.quantize(c.x.to(DEV), pd)
    qb, sb = kq.quantize_weight(W.to(DEV), pd)
    C = kq.gemm_mxfp4(qa, sa, qb, sb).cpu().numpy()
    rows = np.array([0, 1, 127, 128, 2047, c.M - 2, c.M - 1])
    check_gemm(C, qa.cpu().numpy(), sa.cpu().numpy(), qb.cpu().numpy(), sb.cpu().numpy(), rows=rows)


def test_gemm_empty_and_device_status():
    qa = torch.zeros((0, 32), dtype=torch.uint8, device=DEV)
    sa = torch.zeros((0, 2), dtype=torch.uint8, device=DEV)
    qb = torch.zeros((16, 32), dtype=torch.uint8, device=DEV)
    sb = torch.zeros((16, 2), dtype=torch.uint8, device=DEV)
    assert kq.gemm_mxfp4(qa, sa, qb, sb).shape == (0, 16)
    assert kq.device_status() == 0


@pytest.mark.parametrize("rows,K", [(1, 32), (130, 544), (300, 2240), (256, 12288)])
def test_scales_to_tiled_matches_the_oracle(rows, K):
    s = np.random.default_rng(rows + K).integers(0, 255, (rows, K // 32), dtype=np.uint8)
    t = kq.scales_to_tiled(_dev(s), K)
    torch.cuda.synchronize()
    assert np.array_equal(t.cpu().numpy(), o.scales_to_mma(s))


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (130, 300, 544), (1, 8, 32),
                                   (257, 520, 1152), (64, 40, 2240), (300, 256, 96)])
def test_tiled_scales_give_the_same_product(M, N, K):
    """The tiled-scale kernel reads the same codes and scales and runs the
    same MMAs: its output equals the row-major kernel's bit for bit, and the
    oracle's product within the tolerance."""
    qa, sa, qb, sb = random_operands(M, N, K, seed=M * 5 + N + K)
    c_row = run(qa, sa, qb, sb)
    c_tiled = kq.gemm_mxfp4_tiled(_dev(qa), kq.scales_to_tiled(_dev(sa), K), _dev(qb),
                                  kq.scales_to_tiled(_dev(sb), K))
    torch.cuda.synchronize()
    assert torch.equal(c_row, c_tiled)
    check_gemm(c_tiled.cpu().numpy(), qa, sa, qb, sb)
    c16 = kq.gemm_mxfp4_tiled(_dev(qa), kq.scales_to_tiled(_dev(sa), K), _dev(qb),
                              kq.scales_to_tiled(_dev(sb), K), out_dtype=torch.bfloat16)
    assert torch.equal(c16, c_tiled.to(torch.bfloat16))


@pytest.mark.parametrize("name,di,N", [("pixart_sigma", 0, 1152), ("sana", 0, 2240),
                                       ("flux_schnell", 0, 3072)], ids=lambda v: str(v))
def test_quantizers_write_the_tiled_layout(name, di, N):
    """kq_quantize_tiled / kq_quantize_weight_tiled give the same codes as
    the row-major quantizers and the tiled image of their scales (padding
    of each row's last 4-scale column zero); the layer's product through
    them equals the row-major product bit for bit."""
    c = w.make_case(name, di, 0, M=192)
    W = w.draw_weight(N, c.d, c.seed)
    pd = _dev(c.params)
    x, wd = c.x.to(DEV), W.to(DEV)
    qa, sa = kq.quantize(x, pd)
    qb, sb = kq.quantize_weight(wd, pd)
    qa_t, ta = kq.quantize_tiled(x, pd)
    qb_t, tb = kq.quantize_weight_tiled(wd, pd)
    torch.cuda.synchronize()
    assert torch.equal(qa, qa_t) and torch.equal(qb, qb_t)
    assert np.array_equal(ta.cpu().numpy(), o.scales_to_mma(sa.cpu().numpy()))
    assert np.array_equal(tb.cpu().numpy(), o.scales_to_mma(sb.cpu().numpy()))
    c_row = kq.gemm_mxfp4(qa, sa, qb, sb)
    c_tiled = kq.gemm_mxfp4_tiled(qa_t, ta, qb_t, tb)
    assert torch.equal(c_row, c_tiled)


@pytest.mark.parametrize("M,N,K,dt", [(4096, 4096, 1152, torch.bfloat16),
                                      (2048, 4104, 544, torch.float32),
                                      (2100, 2048, 4096, torch.bfloat16),
                                      (300, 520, 96, torch.float32),
                                      (384, 768, 12320, torch.bfloat16)])
def test_persistent_and_per_tile_kernels_agree(M, N, K, dt, monkeypatch):
    """The persistent tiled-scale kernel (several tiles per CTA, TMA stores
    overlapping the next tile) and the one-tile-per-CTA kernel run the same
    MMAs on the same stages: identical outputs."""
    qa, sa, qb, sb = random_operands(M, N, K, seed=M + N + K + 3)
    ta, tb = kq.scales_to_tiled(_dev(sa), K), kq.scales_to_tiled(_dev(sb), K)
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("KQ_GEMM_PERSISTENT", flag)
        outs.append(kq.gemm_mxfp4_tiled(_dev(qa), ta, _dev(qb), tb, out_dtype=dt))
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    rows = np.array([0, 1, 127, 128, M // 2, M - 1])
    check_gemm(outs[0].float().cpu().numpy() if dt == torch.float32 else
               outs[0].float().cpu().numpy(), qa, sa, qb, sb, rows=rows) \
        if dt == torch.float32 else None
    assert kq.device_status() == 0


@pytest.mark.parametrize("M,N,K,dt", [(256, 256, 256, torch.float32),
                                      (300, 520, 544, torch.float32),
                                      (1, 8, 32, torch.float32),
                                      (2048, 4096, 1152, torch.bfloat16),
                                      (384, 768, 12320, torch.bfloat16)])
def test_cta_pair_kernel_agrees(M, N, K, dt, monkeypatch):
    """The CTA-pair kernel (clusters of two, tcgen05.mma.cta_group::2 on
    256 x 256 tiles, each CTA loading half of B) gives the persistent
    one-CTA kernel's output bit for bit, within the tolerance of the exact
    product on sampled rows; tile edges in M and N, partial last k-tiles."""
    qa, sa, qb, sb = random_operands(M, N, K, seed=M * 3 + N + K)
    ta, tb = kq.scales_to_tiled(_dev(sa), K), kq.scales_to_tiled(_dev(sb), K)
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("KQ_GEMM_PAIR", flag)
        outs.append(kq.gemm_mxfp4_tiled(_dev(qa), ta, _dev(qb), tb, out_dtype=dt))
    torch.cuda.synchronize()
    assert kq.device_status() == 0
    assert torch.equal(outs[0], outs[1])
    if dt == torch.float32:
        rows = np.unique(np.array([0, min(1, M - 1), min(127, M - 1), min(128, M - 1), M // 2, M - 1]))
        check_gemm(outs[0].cpu().numpy(), qa, sa, qb, sb, rows=rows)
