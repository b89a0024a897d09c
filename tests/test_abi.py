"""The C-ABI library loads without a GPU, exports every entry point the
header declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from w4a4_post_quantization_b200 import build
    build.build()
    from w4a4_post_quantization_b200 import _lib
    return _lib.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n


def test_binding_covers_the_header():
    from w4a4_post_quantization_b200 import _lib
    assert sorted(_lib.SIGNATURES) == _declared()


def test_status_strings_and_version(lib):
    assert lib.kq_status_string(0) == b"ok"
    assert lib.kq_status_string(1) == b"invalid argument"
    assert lib.kq_status_string(123) == b"unknown status"
    assert lib.kq_version() >> 16 == 1


FAKE = 0x10000          # 16-byte aligned, never dereferenced: checks fail first


@pytest.mark.parametrize("M,d", [(-1, 64), (4, 0), (4, 48), (4, 16), (1 << 30, 1 << 20)])
def test_bad_shapes(lib, M, d):
    assert lib.kq_quantize(FAKE, M, d, FAKE, FAKE, FAKE, None) == 1
    assert lib.kq_quantize_hadamard(FAKE, M, d, FAKE, FAKE, None) == 1
    assert lib.kq_quantize_smooth(FAKE, M, d, FAKE, FAKE, FAKE, None) == 1
    assert lib.kq_transform(FAKE, M, d, FAKE, FAKE, None) == 1
    assert lib.kq_inverse_transform(FAKE, M, d, FAKE, FAKE, None) == 1
    assert lib.kq_dequantize(FAKE, FAKE, M, d, FAKE, None) == 1
    assert lib.kq_quantize16(FAKE, M, d, FAKE, FAKE, FAKE, None) == 1
    assert lib.kq_transform16(FAKE, M, d, FAKE, FAKE, None) == 1
    assert lib.kq_quantize_weight(FAKE, M, d, FAKE, FAKE, FAKE, None) == 1
    assert lib.kq_fold_weight(FAKE, M, d, FAKE, FAKE, None) == 1
    if d < 32 or d % 32:
        assert lib.kq_gemm_mxfp4(FAKE, FAKE, FAKE, FAKE, 4, 4, d, FAKE, 0, None) == 1
    assert lib.kq_gemm_mxfp4(FAKE, FAKE, FAKE, FAKE, -1, 4, 64, FAKE, 0, None) == 1


def test_null_and_misaligned_pointers(lib):
    assert lib.kq_quantize(None, 4, 64, FAKE, FAKE, FAKE, None) == 1
    assert lib.kq_quantize(FAKE, 4, 64, None, FAKE, FAKE, None) == 1
    assert lib.kq_quantize(FAKE, 4, 64, FAKE, None, FAKE, None) == 1
    assert lib.kq_quantize(FAKE, 4, 64, FAKE, FAKE, None, None) == 1
    assert lib.kq_quantize(FAKE + 8, 4, 64, FAKE, FAKE, FAKE, None) == 1      # x not 16-B aligned
    assert lib.kq_quantize(FAKE, 4, 64, FAKE + 2, FAKE, FAKE, None) == 1      # params not 4-B
    assert lib.kq_quantize(FAKE, 4, 64, FAKE, FAKE + 4, FAKE, None) == 1      # q not 16-B
    assert lib.kq_quantize_smooth(FAKE, 4, 64, FAKE + 4, FAKE, FAKE, None) == 1
    assert lib.kq_quantize_ex(FAKE, 4, 64, FAKE, FAKE, FAKE, 7, None) == 1
    assert lib.kq_dequantize(FAKE, FAKE, 4, 64, FAKE + 4, None) == 1
    assert lib.kq_device_status(None) == 1
    assert lib.kq_quantize16(FAKE, 4, 64, FAKE, FAKE, FAKE + 1, None) == 1    # scales16 not 2-B
    assert lib.kq_quantize16(FAKE, 4, 64, None, FAKE, FAKE, None) == 1
    assert lib.kq_quantize16(FAKE, 1, 32 * 65536, FAKE, FAKE, FAKE, None) == 1   # too wide
    assert lib.kq_transform16(FAKE, 4, 64, FAKE, FAKE + 8, None) == 1         # y not 16-B
    assert lib.kq_gemm_mxfp4(FAKE, FAKE, FAKE, FAKE, 4, 4, 64, FAKE, 2, None) == 1   # dtype
    assert lib.kq_gemm_mxfp4(FAKE + 8, FAKE, FAKE, FAKE, 4, 4, 64, FAKE, 0, None) == 1
    assert lib.kq_gemm_mxfp4(FAKE, FAKE, FAKE, FAKE, 4, 4, 64, FAKE + 4, 1, None) == 1
    assert lib.kq_gemm_mxfp4(FAKE, None, FAKE, FAKE, 4, 4, 64, FAKE, 0, None) == 1
    assert lib.kq_gemm_mxfp4_tiled(FAKE, FAKE + 4, FAKE, FAKE, 4, 4, 64, FAKE, 0, None) == 1
    assert lib.kq_gemm_mxfp4_tiled(FAKE, FAKE, FAKE, FAKE, 4, 4, 48, FAKE, 0, None) == 1
    assert lib.kq_scales_to_tiled(FAKE, 4, 48, FAKE, None) == 1
    assert lib.kq_scales_to_tiled(FAKE, 4, 64, FAKE + 4, None) == 1
    assert lib.kq_scales_tiled_bytes(0, 64) == 0 and lib.kq_scales_tiled_bytes(130, 544) == 2 * 5 * 512
    ada = lambda *a: lib.kq_quantize_adaln(*a)
    assert ada(FAKE, 4, 64, FAKE, FAKE, 0, 1e-6, FAKE, FAKE, FAKE, None) == 1      # tokens
    assert ada(FAKE, 4, 64, FAKE, FAKE, 4, -1.0, FAKE, FAKE, FAKE, None) == 1      # eps
    assert ada(FAKE, 4, 64, FAKE + 2, FAKE, 4, 1e-6, FAKE, FAKE, FAKE, None) == 1  # shift
    assert ada(FAKE, 4, 64, FAKE, FAKE, 4, float("nan"), FAKE, FAKE, FAKE, None) == 1
    assert ada(FAKE, 4, 32 * 385, FAKE, FAKE, 4, 1e-6, FAKE, FAKE, FAKE, None) == 1
    assert lib.kq_transform_adaln(FAKE, 4, 64, FAKE, FAKE, 4, 1e-6, FAKE, FAKE + 8, None) == 1
    assert lib.kq_gemm_mxfp4(FAKE, FAKE, FAKE, FAKE, 1 << 31, 4, 64, FAKE, 0, None) == 1


def test_block16_tiled_and_weight_entries_check_on_the_host(lib):
    """The block-16, tiled-scale and weight-side entry points reject bad
    shapes, null and misaligned pointers before any CUDA call."""
    for f in (lib.kq_quantize16_tiled, lib.kq_quantize_weight16, lib.kq_quantize_weight16_tiled,
              lib.kq_quantize_tiled, lib.kq_quantize_weight_tiled):
        assert f(FAKE, 4, 48, FAKE, FAKE, FAKE, None) == 1           # d not a multiple of 32
        assert f(FAKE, -1, 64, FAKE, FAKE, FAKE, None) == 1
        assert f(None, 4, 64, FAKE, FAKE, FAKE, None) == 1
        assert f(FAKE, 4, 64, None, FAKE, FAKE, None) == 1
        assert f(FAKE + 8, 4, 64, FAKE, FAKE, FAKE, None) == 1       # x not 16-B aligned
        assert f(FAKE, 4, 64, FAKE, FAKE + 4, FAKE, None) == 1       # q not 16-B aligned
        assert f(None, 0, 64, None, None, None, None) == 0            # empty: nothing to do
    assert lib.kq_quantize16_tiled(FAKE, 4, 64, FAKE, FAKE, FAKE + 4, None) == 1       # tiled: 16-B
    assert lib.kq_quantize_weight16_tiled(FAKE, 4, 64, FAKE, FAKE, FAKE + 4, None) == 1
    assert lib.kq_quantize_weight16(FAKE, 4, 64, FAKE, FAKE, FAKE + 1, None) == 1      # 2-B scales
    assert lib.kq_fold_weight16(FAKE, 4, 64, FAKE, FAKE + 4, None) == 1
    assert lib.kq_fold_weight16(FAKE, 4, 64, None, FAKE, None) == 1
    assert lib.kq_scales16_tiled_bytes(0, 64) == 0 and lib.kq_scales16_tiled_bytes(4, 48) == 0
    assert lib.kq_scales16_tiled_bytes(130, 544) == 2 * 9 * 512     # 34 scales: nine 4-columns
    g16 = lib.kq_gemm_mxfp4_16_tiled
    assert g16(FAKE, FAKE, FAKE, FAKE, 4, 4, 48, FAKE, 0, None) == 1             # K % 32
    assert g16(FAKE, FAKE, FAKE, FAKE, 4, 4, 64, FAKE, 2, None) == 1             # dtype
    assert g16(FAKE, FAKE + 4, FAKE, FAKE, 4, 4, 64, FAKE, 0, None) == 1         # tiled: 16-B
    assert g16(FAKE, FAKE, None, FAKE, 4, 4, 64, FAKE, 0, None) == 1
    assert g16(None, None, None, None, 0, 4, 64, None, 0, None) == 0


def test_calibration_entries_check_on_the_host(lib):
    grad = lib.kq_transform_params_grad
    ws = lib.kq_transform_params_grad_workspace_bytes(16, 64)
    assert ws > 256 and lib.kq_transform_params_grad_workspace_bytes(16, 48) == 0
    assert grad(FAKE, FAKE, FAKE, 0, 64, FAKE, 0, 0.1, FAKE, FAKE, FAKE, ws, None) == 1   # M < 1
    assert grad(FAKE, FAKE, FAKE, 16, 48, FAKE, 0, 0.1, FAKE, FAKE, FAKE, ws, None) == 1
    assert grad(FAKE, FAKE, None, 16, 64, FAKE, 0, 0.1, FAKE, FAKE, FAKE, ws, None) == 1
    assert grad(FAKE + 4, FAKE, FAKE, 16, 64, FAKE, 0, 0.1, FAKE, FAKE, FAKE, ws, None) == 1
    assert grad(FAKE, FAKE, FAKE, 16, 64, FAKE, 0, float("nan"), FAKE, FAKE, FAKE, ws, None) == 1
    assert grad(FAKE, FAKE, FAKE, 16, 64, FAKE, 0, 0.1, FAKE, FAKE, FAKE + 16, ws, None) == 1
    res = lib.kq_residual
    rws = lib.kq_residual_workspace_bytes()
    assert res(FAKE, FAKE, 0, 1.0, FAKE, FAKE, FAKE, rws, None) == 1               # n < 1
    assert res(FAKE, FAKE, 8, 1.0, FAKE, FAKE, FAKE, rws - 1, None) == 1           # workspace
    assert res(FAKE, FAKE, 8, float("inf"), FAKE, FAKE, FAKE, rws, None) == 1
    assert res(FAKE, FAKE, 8, 1.0, FAKE, FAKE + 4, FAKE, rws, None) == 1           # sumsq 8-B
    adam = lib.kq_adam_step
    assert adam(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 1e-2, 0.9, 0.999, 1e-8, None) == 1
    assert adam(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 0, 1e-2, 0.9, 0.999, 1e-8, None) == 1   # step 0
    assert adam(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 1, 1e-2, 1.0, 0.999, 1e-8, None) == 1   # beta1
    assert adam(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 1, 1e-2, 0.9, 0.999, 0.0, None) == 1    # eps
    assert adam(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 1, float("nan"), 0.9, 0.999, 1e-8, None) == 1
    assert adam(None, FAKE, FAKE, FAKE, FAKE, 8, 1, 1e-2, 0.9, 0.999, 1e-8, None) == 1


def test_empty_input_needs_no_device(lib):
    assert lib.kq_quantize(None, 0, 64, None, None, None, None) == 0
    assert lib.kq_dequantize(None, None, 0, 64, None, None) == 0
    assert lib.kq_quantize16(None, 0, 64, None, None, None, None) == 0
    assert lib.kq_gemm_mxfp4(None, None, None, None, 0, 16, 64, None, 0, None) == 0
    assert lib.kq_quantize_adaln(None, 0, 64, None, None, 4, 1e-6, None, None, None, None) == 0


def test_binding_refuses_host_tensors():
    import torch
    import w4a4_post_quantization_b200 as kq
    x = torch.zeros((2, 64), dtype=torch.bfloat16)
    p = torch.zeros((2, 5, 3), dtype=torch.float32)
    with pytest.raises(ValueError):
        kq.quantize(x, p)


def test_missing_library_fails_loudly(tmp_path):
    from w4a4_post_quantization_b200 import _lib
    with pytest.raises(ImportError):
        _lib.load_library(str(tmp_path / "libkq.so"))


def test_host_pipeline_argument_checks(lib):
    need = lib.kq_quantize_host_workspace_bytes(64, 1)
    assert need >= 2 * (64 * 2 + 32 + 2)
    assert lib.kq_quantize_host_workspace_bytes(48, 1) == 0
    assert lib.kq_quantize_host_workspace_bytes(64, 0) == 0
    # too small a workspace, misaligned workspace, bad shape, null pointers
    assert lib.kq_quantize_host(FAKE, 4, 64, FAKE, FAKE, FAKE, FAKE, need - 1, None) == 1
    assert lib.kq_quantize_host(FAKE, 4, 64, FAKE, FAKE, FAKE, FAKE + 16, need, None) == 1
    assert lib.kq_quantize_host(FAKE, 4, 48, FAKE, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.kq_quantize_host(None, 4, 64, FAKE, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.kq_quantize_host(FAKE, 0, 64, FAKE, FAKE, FAKE, FAKE, need, None) == 0
