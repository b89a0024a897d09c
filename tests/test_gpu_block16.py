"""GPU parity of the 16-element variant (16x16 Kronecker blocks of four
factors, one E8M0 scale per 16 elements) against the CPU oracle.

KroQuant review, "Where Pith is reading between the lines": the transform
extends to other block formats by changing the number of Kronecker factors.
Inputs are the seeded DiT-shaped activations of ``workloads`` with their
16-block parameters from ``workloads.draw_params16``; expected values come
only from ``oracle.kq_oracle``.
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
REDUCED_M = 67


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _run(x_t, params16):
    xd = x_t.to(DEV)
    pd = _dev(params16)
    q, s = kq.quantize16(xd, pd)
    y = kq.transform16(xd, pd)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), y.cpu().numpy()


def _check(x_bits, params16, q, s, y, bound=True):
    x64 = o.bf16_bits_to_float64(x_bits)
    y64 = o.transform16(x64, params16)
    cond = o.abs_transform16(x64, params16)
    check_transform_literal(y, y64, cond)
    worst = check_transform(y, y64, cond)
    st = check_mx4(q, s, y64, cond, block=16)
    if bound:
        assert st["scale_exempt"] <= max(2, st["blocks"] // 1000)
        assert st["code_exempt"] <= max(4, st["elements"] // 10000)
    return worst, st


def _bits(x_t):
    return x_t.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("key", w.all_case_keys(), ids=lambda k: f"{k[0]}-d{k[1]}-g{k[2]}")
def test_block16_reduced_configs_elementwise(key):
    name, di, gi = key
    M = w.CONFIGS[name]["M"] if name == "tiny" else REDUCED_M
    c = w.make_case(name, di, gi, M=M)
    p16 = w.draw_params16(c.d, c.seed)
    q, s, y = _run(c.x, p16)
    worst, _ = _check(c.x_bits(), p16, q, s, y)
    assert worst < TOL


@pytest.mark.parametrize("key", [("stress", 0, 0), ("flux_schnell", 1, 2), ("sana", 0, 0)],
                         ids=lambda k: f"{k[0]}-d{k[1]}-g{k[2]}")
def test_block16_full_size_sampled_rows(key):
    name, di, gi = key
    c = w.make_case(name, di, gi)
    p16 = w.draw_params16(c.d, c.seed)
    q, s, y = _run(c.x, p16)
    rng = np.random.default_rng(c.seed)
    rows = np.array(sorted(set(range(3)) | set(range(c.M - 3, c.M)) |
                           set(rng.choice(c.M, 12, replace=False).tolist())))
    _check(c.x_bits()[rows], p16, q[rows], s[rows], y[rows])


def test_block16_matches_oracle_bytes_on_tiny():
    """Packed codes and scales equal the oracle's bytes except inside the
    tolerance band (counted, and rare)."""
    c = w.make_case("tiny", 0, 0)
    p16 = w.draw_params16(c.d, c.seed)
    q, s, y = _run(c.x, p16)
    q_ref, s_ref = o.quantize16(c.x_bits(), p16)
    assert q.shape == q_ref.shape and s.shape == s_ref.shape
    assert (q != q_ref).mean() < 1e-3 and (s != s_ref).mean() < 1e-3


def test_block16_singular_factor_takes_the_plain_form():
    """(a, b, c) = (-1, 1, 1) gives g11 = 0: that CTA's units run the plain
    four-term stages, in either 16-block of a unit."""
    c = w.make_case("flux_schnell", 0, 0, M=150)
    p16 = w.draw_params16(c.d, c.seed)
    p16[10, 1] = [-1.0, 1.0, 1.0]               # block 0 of unit 5
    p16[181, 3] = [-1.0, 1.0, 1.0]              # block 1 of unit 90
    q, s, y = _run(c.x, p16)
    _check(c.x_bits(), p16, q, s, y)


def test_block16_large_shear_growth_takes_the_plain_form():
    c = w.make_case("tiny", 0, 0, M=40)
    p16 = w.draw_params16(c.d, c.seed)
    p16[7] = [[300.0, 1.0, 0.0]] * 4             # growth 301^4 > 2^24
    q, s, y = _run(c.x, p16)
    _check(c.x_bits(), p16, q, s, y)


@pytest.mark.parametrize("d", [32, 64, 32 * 389, 32 * 1031])
def test_block16_odd_widths(d):
    """One unit per row, and prime unit counts (panels of one column unit)."""
    x = w.random_bf16((37, d), seed=d)
    p16 = w.draw_params16(d, seed=d)
    q, s, y = _run(x, p16)
    _check(_bits(x), p16, q, s, y)


def test_block16_zero_and_huge_blocks():
    d = 128
    x = w.random_bf16((9, d), seed=5).float().numpy()
    x[0] = 0.0                                   # all-zero row: scale byte 0
    x[1, :16] = 0.0                              # one zero 16-block next to a live one
    x[2] *= 2.0 ** 60
    x[3] *= 2.0 ** -100
    xt = torch.from_numpy(x).to(torch.bfloat16)
    p16 = w.draw_params16(d, seed=11)
    q, s, y = _run(xt, p16)
    _check(_bits(xt), p16, q, s, y, bound=False)
    assert (s[0] == 0).all() and s[1, 0] == 0 and s[1, 1] != 0
    assert ((q[0] & 0x77) == 0).all()


def test_block16_empty_and_invalid():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    p16 = torch.zeros((4, 4, 3), dtype=torch.float32, device=DEV)
    q, s = kq.quantize16(x, p16)
    assert q.shape == (0, 32) and s.shape == (0, 4)
    lib = kq.lib()
    xd = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    qd = torch.empty((4, 32), dtype=torch.uint8, device=DEV)
    sd = torch.empty((4 * 4 + 1,), dtype=torch.uint8, device=DEV)
    # A scale array that is not 2-byte aligned is rejected before any launch.
    st = lib.kq_quantize16(xd.data_ptr(), 4, 64, p16.data_ptr(), qd.data_ptr(),
                           sd.data_ptr() + 1, torch.cuda.current_stream().cuda_stream)
    assert st == 1
    st = lib.kq_transform16(xd.data_ptr(), 4, 48, p16.data_ptr(), qd.data_ptr(),
                            torch.cuda.current_stream().cuda_stream)
    assert st == 1
    assert kq.device_status() == 0


# ----------------------------------------------- block-16 W4A4 layer path
def test_block16_weight_fold_and_quantizer():
    c = w.make_case("flux_schnell", 0, 0, M=16)
    p16 = w.draw_params16(c.d, c.seed)
    W = w.draw_weight(150, c.d, c.seed)
    pd = _dev(p16)
    q, s = kq.quantize_weight16(W.to(DEV), pd)
    f = kq.fold_weight16(W.to(DEV), pd)
    torch.cuda.synchronize()
    w64 = o.bf16_bits_to_float64(_bits(W))
    f64 = o.fold_weight16(w64, p16)
    cond = o.abs_fold_weight16(w64, p16)
    check_transform_literal(f.cpu().numpy(), f64, cond)
    st = check_mx4(q.cpu().numpy(), s.cpu().numpy(), f64, cond, block=16)
    assert st["scale_exempt"] <= 2 and st["code_exempt"] <= 8


@pytest.mark.parametrize("name,di,N", [("pixart_sigma", 0, 1152), ("sana", 0, 2240),
                                       ("stress", 0, 520)], ids=lambda v: str(v))
def test_block16_layer_product(name, di, N):
    """Block-16 quantizers with tiled scales feed the block16 tensor-core
    product; the codes match the row-major quantizers, the tiled scales the
    oracle's tiled image, and the product the oracle's exact product of the
    GPU's operands within the float32-accumulation bound."""
    c = w.make_case(name, di, 0, M=200)
    p16 = w.draw_params16(c.d, c.seed)
    W = w.draw_weight(N, c.d, c.seed)
    pd, xd, wd = _dev(p16), c.x.to(DEV), W.to(DEV)
    qa, sa = kq.quantize16(xd, pd)
    qb, sb = kq.quantize_weight16(wd, pd)
    qat, sat = kq.quantize16_tiled(xd, pd)
    qbt, sbt = kq.quantize_weight16_tiled(wd, pd)
    C = kq.gemm_mxfp4_16_tiled(qat, sat, qbt, sbt)
    C16 = kq.gemm_mxfp4_16_tiled(qat, sat, qbt, sbt, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(qa, qat) and torch.equal(qb, qbt)
    assert np.array_equal(sat.cpu().numpy(), o.scales_to_mma(sa.cpu().numpy()))
    assert np.array_equal(sbt.cpu().numpy(), o.scales_to_mma(sb.cpu().numpy()))
    assert torch.equal(C16, C.to(torch.bfloat16))
    qa_, sa_, qb_, sb_ = (t.cpu().numpy() for t in (qa, sa, qb, sb))
    ref = o.mxfp4_gemm(qa_, sa_, qb_, sb_, block=16)
    mag = o.abs_mxfp4_gemm(qa_, sa_, qb_, sb_, block=16)
    K = c.d
    assert (np.abs(C.cpu().numpy() - ref) <= (K / 64 + 1) * 2.0 ** -22 * mag).all()


def test_block16_product_random_operands_and_exact_sums():
    rng = np.random.default_rng(77)
    for (M, N, K) in [(130, 300, 544), (128, 256, 64), (257, 520, 2240)]:
        ca = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
        cb = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
        lo, hi = (127, 128) if K == 64 else (120, 135)
        sa = rng.integers(lo, hi, (M, K // 16), dtype=np.uint8)
        sb = rng.integers(lo, hi, (N, K // 16), dtype=np.uint8)
        C = kq.gemm_mxfp4_16_tiled(_dev(ca), _dev(o.scales_to_mma(sa)), _dev(cb),
                                   _dev(o.scales_to_mma(sb))).cpu().numpy()
        ref = o.mxfp4_gemm(ca, sa, cb, sb, block=16)
        if K == 64:
            assert np.array_equal(C.astype(np.float64), ref)   # small exact sums
        mag = o.abs_mxfp4_gemm(ca, sa, cb, sb, block=16)
        assert (np.abs(C - ref) <= (K / 64 + 1) * 2.0 ** -22 * mag).all(), (M, N, K)


@pytest.mark.parametrize("M,N,K,dt", [(2048, 4096, 1152, torch.bfloat16),
                                      (300, 520, 96, torch.float32),
                                      (384, 768, 4128, torch.bfloat16)])
def test_block16_persistent_and_per_tile_kernels_agree(M, N, K, dt, monkeypatch):
    """The persistent kernel with scales per 16 (several tiles per CTA, three
    stages) and the one-tile-per-CTA kernel run the same MMAs: identical
    outputs, within the tolerance of the exact product on sampled rows."""
    rng = np.random.default_rng(M + N + K)
    ca = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    cb = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(120, 135, (M, K // 16), dtype=np.uint8)
    sb = rng.integers(120, 135, (N, K // 16), dtype=np.uint8)
    args = (_dev(ca), _dev(o.scales_to_mma(sa)), _dev(cb), _dev(o.scales_to_mma(sb)))
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("KQ_GEMM16_PERSISTENT", flag)
        outs.append(kq.gemm_mxfp4_16_tiled(*args, out_dtype=dt))
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    rows = np.array([0, 1, 127, 128, M // 2, M - 1])
    ref = o.mxfp4_gemm(ca[rows], sa[rows], cb, sb, block=16)
    mag = o.abs_mxfp4_gemm(ca[rows], sa[rows], cb, sb, block=16)
    got = outs[0].float().cpu().numpy()[rows].astype(np.float64)
    tol = (K / 64 + 1) * 2.0 ** -22 * mag + (np.abs(ref) * 2.0 ** -8 if dt == torch.bfloat16 else 0)
    assert (np.abs(got - ref) <= tol).all()
    assert kq.device_status() == 0
