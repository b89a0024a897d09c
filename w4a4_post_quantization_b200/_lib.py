"""ctypes binding of ``libkq.so`` (the C ABI declared in ``include/kq.h``).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, their device pointers and the current CUDA stream are passed to
the library, and a non-zero status raises.  Every step of the computation runs
in the library's kernels; there is no CPU fallback, and a missing library
raises ImportError.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkq.so")

KQ_OK, KQ_ERR_INVALID, KQ_ERR_CUDA, KQ_ERR_DEVICE, KQ_ERR_TIMEOUT = 0, 1, 2, 3, 4
KQ_IMPL_AUTO, KQ_IMPL_TMA, KQ_IMPL_DIRECT, KQ_IMPL_WARP, KQ_IMPL_PANEL, KQ_IMPL_MMA = 0, 1, 2, 3, 4, 5
KQ_OUT_F32, KQ_OUT_BF16 = 0, 1

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int

# name -> (argtypes); every entry point returns int unless listed in _RESTYPE.
SIGNATURES = {
    "kq_quantize": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_quantize_ex": [_p, _i64, _i64, _p, _p, _p, _int, _p],
    "kq_quantize_hadamard": [_p, _i64, _i64, _p, _p, _p],
    "kq_quantize_smooth": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_transform": [_p, _i64, _i64, _p, _p, _p],
    "kq_quantize16": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_quantize_weight16": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_fold_weight16": [_p, _i64, _i64, _p, _p, _p],
    "kq_quantize16_tiled": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_quantize_weight16_tiled": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_scales16_tiled_bytes": [_i64, _i64],
    "kq_gemm_mxfp4_16_tiled": [_p, _p, _p, _p, _i64, _i64, _i64, _p, _int, _p],
    "kq_transform16": [_p, _i64, _i64, _p, _p, _p],
    "kq_quantize_weight": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_fold_weight": [_p, _i64, _i64, _p, _p, _p],
    "kq_gemm_mxfp4": [_p, _p, _p, _p, _i64, _i64, _i64, _p, _int, _p],
    "kq_gemm_mxfp4_tiled": [_p, _p, _p, _p, _i64, _i64, _i64, _p, _int, _p],
    "kq_scales_tiled_bytes": [_i64, _i64],
    "kq_quantize_tiled": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_quantize_weight_tiled": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_scales_to_tiled": [_p, _i64, _i64, _p, _p],
    "kq_transform_params_grad_workspace_bytes": [_i64, _i64],
    "kq_transform_params_grad": [_p, _p, _p, _i64, _i64, _p, _int, ctypes.c_float, _p, _p, _p,
                                 ctypes.c_size_t, _p],
    "kq_residual_workspace_bytes": [],
    "kq_residual": [_p, _p, _i64, ctypes.c_float, _p, _p, _p, ctypes.c_size_t, _p],
    "kq_adam_step": [_p, _p, _p, _p, _p, _i64, _int, ctypes.c_double, ctypes.c_double,
                     ctypes.c_double, ctypes.c_double, _p],
    "kq_quantize_adaln": [_p, _i64, _i64, _p, _p, _i64, ctypes.c_float, _p, _p, _p, _p],
    "kq_quantize_adaln_tiled": [_p, _i64, _i64, _p, _p, _i64, ctypes.c_float, _p, _p, _p, _p],
    "kq_transform_adaln": [_p, _i64, _i64, _p, _p, _i64, ctypes.c_float, _p, _p, _p],
    "kq_inverse_transform": [_p, _i64, _i64, _p, _p, _p],
    "kq_dequantize": [_p, _p, _i64, _i64, _p, _p],
    "kq_quantize_host": [_p, _i64, _i64, _p, _p, _p, _p, ctypes.c_size_t, _p],
    "kq_quantize_host_workspace_bytes": [_i64, _i64],
    "kq_quantize_host_static": [_p, _i64, _i64, _p, _p, _p, _p],
    "kq_status_string": [_int],
    "kq_last_cuda_error": [],
    "kq_device_status": [ctypes.POINTER(_int)],
    "kq_version": [],
    "kq_selftest_wait_timeout": [_p],
}
_RESTYPE = {"kq_status_string": ctypes.c_char_p,
            "kq_quantize_host_workspace_bytes": ctypes.c_size_t,
            "kq_transform_params_grad_workspace_bytes": ctypes.c_size_t,
            "kq_residual_workspace_bytes": ctypes.c_size_t,
            "kq_scales_tiled_bytes": ctypes.c_size_t,
            "kq_scales16_tiled_bytes": ctypes.c_size_t}


class KQError(RuntimeError):
    def __init__(self, fn: str, status: int, lib):
        msg = lib.kq_status_string(status).decode()
        if status == KQ_ERR_CUDA:
            msg += f" (cudaError {lib.kq_last_cuda_error()})"
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


def load_library(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it first (python -c 'import __graft_entry__ as g; g.build()')")
    lib = ctypes.CDLL(path)
    for name, args in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = _RESTYPE.get(name, ctypes.c_int)
    return lib


_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        _LIB = load_library()
    return _LIB


def _check(name: str, status: int) -> None:
    if status != KQ_OK:
        raise KQError(name, status, lib())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device) -> int:
    """The handle of the current stream of `device` (without building a
    torch.cuda.Stream object per call where torch offers the raw query)."""
    if _raw_stream is not None:
        return _raw_stream(device.index if device.index is not None
                           else torch.cuda.current_device())
    return torch.cuda.current_stream(device).cuda_stream


def _dev_tensor(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _shape(x: torch.Tensor):
    if x.dim() != 2:
        raise ValueError("x must be 2-D [M, d]")
    M, d = x.shape
    if d % 32 != 0 or d == 0:
        raise ValueError("d must be a positive multiple of 32")
    return M, d


def _out_codes(x, q, scales):
    M, d = _shape(x)
    if q is None:
        q = torch.empty((M, d // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((M, d // 32), dtype=torch.uint8, device=x.device)
    _dev_tensor(q, torch.uint8, "q")
    _dev_tensor(scales, torch.uint8, "scales")
    if tuple(q.shape) != (M, d // 2) or tuple(scales.shape) != (M, d // 32):
        raise ValueError("output shapes must be [M, d/2] and [M, d/32]")
    return M, d, q, scales


def _params(params: torch.Tensor, d: int) -> torch.Tensor:
    _dev_tensor(params, torch.float32, "params")
    if params.numel() != (d // 32) * 15:
        raise ValueError("params must hold [d/32, 5, 3] float32 values")
    return params


def quantize(x: torch.Tensor, params: torch.Tensor, q=None, scales=None, impl: int = KQ_IMPL_AUTO):
    """MXFP4(x T): returns (packed codes uint8 [M, d/2], scale bytes uint8 [M, d/32])."""
    _dev_tensor(x, torch.bfloat16, "x")
    M, d, q, scales = _out_codes(x, q, scales)
    _params(params, d)
    if impl == KQ_IMPL_AUTO:
        st = lib().kq_quantize(x.data_ptr(), M, d, params.data_ptr(), q.data_ptr(),
                               scales.data_ptr(), _stream(x.device))
    else:
        st = lib().kq_quantize_ex(x.data_ptr(), M, d, params.data_ptr(), q.data_ptr(),
                                  scales.data_ptr(), impl, _stream(x.device))
    _check("kq_quantize", st)
    return q, scales


def quantize_hadamard(x: torch.Tensor, q=None, scales=None):
    _dev_tensor(x, torch.bfloat16, "x")
    M, d, q, scales = _out_codes(x, q, scales)
    st = lib().kq_quantize_hadamard(x.data_ptr(), M, d, q.data_ptr(), scales.data_ptr(),
                                    _stream(x.device))
    _check("kq_quantize_hadamard", st)
    return q, scales


def quantize_smooth(x: torch.Tensor, inv_s: torch.Tensor, q=None, scales=None):
    _dev_tensor(x, torch.bfloat16, "x")
    M, d, q, scales = _out_codes(x, q, scales)
    _dev_tensor(inv_s, torch.float32, "inv_s")
    if inv_s.numel() != d:
        raise ValueError("inv_s must hold d float32 values")
    st = lib().kq_quantize_smooth(x.data_ptr(), M, d, inv_s.data_ptr(), q.data_ptr(),
                                  scales.data_ptr(), _stream(x.device))
    _check("kq_quantize_smooth", st)
    return q, scales


def transform(x: torch.Tensor, params: torch.Tensor, y=None):
    """y = x T in float32."""
    _dev_tensor(x, torch.bfloat16, "x")
    M, d = _shape(x)
    _params(params, d)
    if y is None:
        y = torch.empty((M, d), dtype=torch.float32, device=x.device)
    _dev_tensor(y, torch.float32, "y")
    st = lib().kq_transform(x.data_ptr(), M, d, params.data_ptr(), y.data_ptr(), _stream(x.device))
    _check("kq_transform", st)
    return y


def _params16(params16: torch.Tensor, d: int) -> torch.Tensor:
    _dev_tensor(params16, torch.float32, "params16")
    if params16.numel() != (d // 16) * 12:
        raise ValueError("params16 must hold [d/16, 4, 3] float32 values")
    return params16


def quantize16(x: torch.Tensor, params16: torch.Tensor, q=None, scales16=None):
    """16-element variant: returns (packed codes uint8 [M, d/2], scale bytes
    uint8 [M, d/16])."""
    _dev_tensor(x, torch.bfloat16, "x")
    M, d = _shape(x)
    _params16(params16, d)
    if q is None:
        q = torch.empty((M, d // 2), dtype=torch.uint8, device=x.device)
    if scales16 is None:
        scales16 = torch.empty((M, d // 16), dtype=torch.uint8, device=x.device)
    _dev_tensor(q, torch.uint8, "q")
    _dev_tensor(scales16, torch.uint8, "scales16")
    if tuple(q.shape) != (M, d // 2) or tuple(scales16.shape) != (M, d // 16):
        raise ValueError("output shapes must be [M, d/2] and [M, d/16]")
    st = lib().kq_quantize16(x.data_ptr(), M, d, params16.data_ptr(), q.data_ptr(),
                             scales16.data_ptr(), _stream(x.device))
    _check("kq_quantize16", st)
    return q, scales16


def quantize_weight16(w: torch.Tensor, params16: torch.Tensor, q=None, scales16=None):
    """MXFP4 with 16-element blocks of W T16^-T: (codes [N, d/2], scales [N, d/16])."""
    _dev_tensor(w, torch.bfloat16, "w")
    N, d = _shape(w)
    _params16(params16, d)
    if q is None:
        q = torch.empty((N, d // 2), dtype=torch.uint8, device=w.device)
    if scales16 is None:
        scales16 = torch.empty((N, d // 16), dtype=torch.uint8, device=w.device)
    st = lib().kq_quantize_weight16(w.data_ptr(), N, d, params16.data_ptr(), q.data_ptr(),
                                    scales16.data_ptr(), _stream(w.device))
    _check("kq_quantize_weight16", st)
    return q, scales16


def fold_weight16(w: torch.Tensor, params16: torch.Tensor, out=None):
    """W T16^-T in float32."""
    _dev_tensor(w, torch.bfloat16, "w")
    N, d = _shape(w)
    _params16(params16, d)
    if out is None:
        out = torch.empty((N, d), dtype=torch.float32, device=w.device)
    st = lib().kq_fold_weight16(w.data_ptr(), N, d, params16.data_ptr(), out.data_ptr(),
                                _stream(w.device))
    _check("kq_fold_weight16", st)
    return out


def _quantize16_tiled(fn, x, params16, q=None, scales=None):
    _dev_tensor(x, torch.bfloat16, "x")
    M, d = _shape(x)
    _params16(params16, d)
    if q is None:
        q = torch.empty((M, d // 2), dtype=torch.uint8, device=x.device)
    n = int(lib().kq_scales16_tiled_bytes(M, d))
    if scales is None:
        scales = torch.zeros((n,), dtype=torch.uint8, device=x.device)
    if scales.numel() < n:
        raise ValueError("scales must hold kq_scales16_tiled_bytes(M, d) bytes")
    st = getattr(lib(), fn)(x.data_ptr(), M, d, params16.data_ptr(), q.data_ptr(),
                            scales.data_ptr(), _stream(x.device))
    _check(fn, st)
    return q, scales


def quantize16_tiled(x, params16, q=None, scales=None):
    return _quantize16_tiled("kq_quantize16_tiled", x, params16, q, scales)


def quantize_weight16_tiled(w, params16, q=None, scales=None):
    return _quantize16_tiled("kq_quantize_weight16_tiled", w, params16, q, scales)


def gemm_mxfp4_16_tiled(qa, sa16_tiled, qb, sb16_tiled, out=None, out_dtype=torch.float32):
    """C = A B^T for block-16 operands with tiled scales."""
    for t, n in ((qa, "qa"), (sa16_tiled, "sa16_tiled"), (qb, "qb"), (sb16_tiled, "sb16_tiled")):
        _dev_tensor(t, torch.uint8, n)
    M, K = qa.shape[0], 2 * qa.shape[1]
    N = qb.shape[0]
    if tuple(qb.shape) != (N, K // 2):
        raise ValueError("qb must be [N, K/2]")
    if sa16_tiled.numel() < lib().kq_scales16_tiled_bytes(M, K) or \
            sb16_tiled.numel() < lib().kq_scales16_tiled_bytes(N, K):
        raise ValueError("tiled scale arrays are too small")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=qa.device)
    code = KQ_OUT_F32 if out_dtype == torch.float32 else KQ_OUT_BF16
    st = lib().kq_gemm_mxfp4_16_tiled(qa.data_ptr(), sa16_tiled.data_ptr(), qb.data_ptr(),
                                      sb16_tiled.data_ptr(), M, N, K, out.data_ptr(), code,
                                      _stream(qa.device))
    _check("kq_gemm_mxfp4_16_tiled", st)
    return out


def transform16(x: torch.Tensor, params16: torch.Tensor, y=None):
    """y = x T16 in float32 (16-element blocks)."""
    _dev_tensor(x, torch.bfloat16, "x")
    M, d = _shape(x)
    _params16(params16, d)
    if y is None:
        y = torch.empty((M, d), dtype=torch.float32, device=x.device)
    _dev_tensor(y, torch.float32, "y")
    st = lib().kq_transform16(x.data_ptr(), M, d, params16.data_ptr(), y.data_ptr(),
                              _stream(x.device))
    _check("kq_transform16", st)
    return y


def quantize_weight(w: torch.Tensor, params: torch.Tensor, q=None, scales=None):
    """MXFP4(W T^-T) of bf16 weights [N, d]: (codes uint8 [N, d/2], scales
    uint8 [N, d/32]), the operand that meets quantize(x, params)."""
    _dev_tensor(w, torch.bfloat16, "w")
    N, d, q, scales = _out_codes(w, q, scales)
    _params(params, d)
    st = lib().kq_quantize_weight(w.data_ptr(), N, d, params.data_ptr(), q.data_ptr(),
                                  scales.data_ptr(), _stream(w.device))
    _check("kq_quantize_weight", st)
    return q, scales


def fold_weight(w: torch.Tensor, params: torch.Tensor, out=None):
    """W T^-T in float32 [N, d]."""
    _dev_tensor(w, torch.bfloat16, "w")
    N, d = _shape(w)
    _params(params, d)
    if out is None:
        out = torch.empty((N, d), dtype=torch.float32, device=w.device)
    _dev_tensor(out, torch.float32, "out")
    st = lib().kq_fold_weight(w.data_ptr(), N, d, params.data_ptr(), out.data_ptr(),
                              _stream(w.device))
    _check("kq_fold_weight", st)
    return out


def gemm_mxfp4(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
               out=None, out_dtype=torch.float32):
    """C = A B^T for MXFP4 operands A (codes [M, K/2], scales [M, K/32]) and
    B (codes [N, K/2], scales [N, K/32]); C is [M, N] float32 or bf16."""
    for t, n in ((qa, "qa"), (sa, "sa"), (qb, "qb"), (sb, "sb")):
        _dev_tensor(t, torch.uint8, n)
        if t.dim() != 2:
            raise ValueError(f"{n} must be 2-D")
    M, K = qa.shape[0], 2 * qa.shape[1]
    N = qb.shape[0]
    if tuple(qb.shape) != (N, K // 2) or tuple(sa.shape) != (M, K // 32) or \
            tuple(sb.shape) != (N, K // 32):
        raise ValueError("operand shapes must be [M, K/2], [M, K/32], [N, K/2], [N, K/32]")
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=qa.device)
    _dev_tensor(out, out_dtype, "out")
    if tuple(out.shape) != (M, N):
        raise ValueError("out must be [M, N]")
    code = KQ_OUT_F32 if out_dtype == torch.float32 else KQ_OUT_BF16
    st = lib().kq_gemm_mxfp4(qa.data_ptr(), sa.data_ptr(), qb.data_ptr(), sb.data_ptr(), M, N, K,
                             out.data_ptr(), code, _stream(qa.device))
    _check("kq_gemm_mxfp4", st)
    return out


def _adaln_args(x, shift, scale, tokens_per_sample):
    _dev_tensor(x, torch.bfloat16, "x")
    M, d = _shape(x)
    B = max(1, -(-M // int(tokens_per_sample)))
    for t, n in ((shift, "shift"), (scale, "scale")):
        _dev_tensor(t, torch.bfloat16, n)
        if t.dim() != 2 or t.shape[1] != d or t.shape[0] < B:
            raise ValueError(f"{n} must be bf16 [B, d] with B >= ceil(M / tokens_per_sample)")
    return M, d


def quantize_adaln(x: torch.Tensor, shift: torch.Tensor, scale: torch.Tensor,
                   tokens_per_sample: int, params: torch.Tensor, eps: float = 1e-6,
                   q=None, scales=None):
    """MXFP4((LN(x) (1 + scale[b]) + shift[b]) T): LayerNorm without affine,
    AdaLN modulation per sample, transform and quantizer in one pass."""
    M, d = _adaln_args(x, shift, scale, tokens_per_sample)
    _, _, q, scales = _out_codes(x, q, scales)
    _params(params, d)
    st = lib().kq_quantize_adaln(x.data_ptr(), M, d, shift.data_ptr(), scale.data_ptr(),
                                 int(tokens_per_sample), float(eps), params.data_ptr(),
                                 q.data_ptr(), scales.data_ptr(), _stream(x.device))
    _check("kq_quantize_adaln", st)
    return q, scales


def quantize_adaln_tiled(x: torch.Tensor, shift: torch.Tensor, scale: torch.Tensor,
                         tokens_per_sample: int, params: torch.Tensor, eps: float = 1e-6,
                         q=None, scales=None):
    """quantize_adaln with the scales in the tiled layout of gemm_mxfp4_tiled."""
    M, d = _adaln_args(x, shift, scale, tokens_per_sample)
    _params(params, d)
    if q is None:
        q = torch.empty((M, d // 2), dtype=torch.uint8, device=x.device)
    n = int(lib().kq_scales_tiled_bytes(M, d))
    if scales is None:
        scales = torch.zeros((n,), dtype=torch.uint8, device=x.device)
    _dev_tensor(q, torch.uint8, "q")
    _dev_tensor(scales, torch.uint8, "scales")
    if tuple(q.shape) != (M, d // 2) or scales.numel() < n:
        raise ValueError("q must be [M, d/2] and scales hold kq_scales_tiled_bytes(M, d) bytes")
    st = lib().kq_quantize_adaln_tiled(x.data_ptr(), M, d, shift.data_ptr(), scale.data_ptr(),
                                       int(tokens_per_sample), float(eps), params.data_ptr(),
                                       q.data_ptr(), scales.data_ptr(), _stream(x.device))
    _check("kq_quantize_adaln_tiled", st)
    return q, scales


def transform_adaln(x: torch.Tensor, shift: torch.Tensor, scale: torch.Tensor,
                    tokens_per_sample: int, params: torch.Tensor, eps: float = 1e-6, y=None):
    """(LN(x) (1 + scale[b]) + shift[b]) T in float32."""
    M, d = _adaln_args(x, shift, scale, tokens_per_sample)
    _params(params, d)
    if y is None:
        y = torch.empty((M, d), dtype=torch.float32, device=x.device)
    _dev_tensor(y, torch.float32, "y")
    st = lib().kq_transform_adaln(x.data_ptr(), M, d, shift.data_ptr(), scale.data_ptr(),
                                  int(tokens_per_sample), float(eps), params.data_ptr(),
                                  y.data_ptr(), _stream(x.device))
    _check("kq_transform_adaln", st)
    return y


def transform_params_grad(z: torch.Tensor, zq: torch.Tensor, g: torch.Tensor,
                          params: torch.Tensor, inverse_transpose: bool, lam: float,
                          workspace: torch.Tensor, dparams=None, reg=None):
    """dL/dtheta of Z = X K(theta) (K = T, or T^-T for the weight side) with
    dL/dZ = g + 2 lam (Z - Zq); returns (dparams [d/32, 5, 3], reg [1])."""
    for t, n in ((z, "z"), (zq, "zq"), (g, "g")):
        _dev_tensor(t, torch.float32, n)
    M, d = _shape(z)
    if zq.shape != z.shape or g.shape != z.shape:
        raise ValueError("z, zq and g must have the same [M, d] shape")
    _params(params, d)
    if dparams is None:
        dparams = torch.empty((d // 32, 5, 3), dtype=torch.float32, device=z.device)
    if reg is None:
        reg = torch.empty((1,), dtype=torch.float32, device=z.device)
    _dev_tensor(workspace, torch.uint8, "workspace")
    st = lib().kq_transform_params_grad(z.data_ptr(), zq.data_ptr(), g.data_ptr(), M, d,
                                        params.data_ptr(), int(bool(inverse_transpose)),
                                        float(lam), dparams.data_ptr(), reg.data_ptr(),
                                        workspace.data_ptr(), workspace.numel(),
                                        _stream(z.device))
    _check("kq_transform_params_grad", st)
    return dparams, reg


def params_grad_workspace_bytes(M: int, d: int) -> int:
    return int(lib().kq_transform_params_grad_workspace_bytes(M, d))


def residual(y: torch.Tensor, y_ref: torch.Tensor, scale: float, workspace: torch.Tensor,
             out=None, sumsq=None):
    """(scale (y - y_ref), sum (y - y_ref)^2 as a float64 [1] tensor)."""
    _dev_tensor(y, torch.float32, "y")
    _dev_tensor(y_ref, torch.float32, "y_ref")
    if y.shape != y_ref.shape:
        raise ValueError("y and y_ref must have the same shape")
    if out is None:
        out = torch.empty_like(y)
    if sumsq is None:
        sumsq = torch.empty((1,), dtype=torch.float64, device=y.device)
    _dev_tensor(workspace, torch.uint8, "workspace")
    st = lib().kq_residual(y.data_ptr(), y_ref.data_ptr(), y.numel(), float(scale),
                           out.data_ptr(), sumsq.data_ptr(), workspace.data_ptr(),
                           workspace.numel(), _stream(y.device))
    _check("kq_residual", st)
    return out, sumsq


def residual_workspace_bytes() -> int:
    return int(lib().kq_residual_workspace_bytes())


def adam_step(params: torch.Tensor, grad0: torch.Tensor, grad1, m: torch.Tensor,
              v: torch.Tensor, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
              eps: float = 1e-8):
    for t, n in ((params, "params"), (grad0, "grad0"), (m, "m"), (v, "v")):
        _dev_tensor(t, torch.float32, n)
    if grad1 is not None:
        _dev_tensor(grad1, torch.float32, "grad1")
    st = lib().kq_adam_step(params.data_ptr(), grad0.data_ptr(),
                            grad1.data_ptr() if grad1 is not None else None, m.data_ptr(),
                            v.data_ptr(), params.numel(), int(step), float(lr), float(beta1),
                            float(beta2), float(eps), _stream(params.device))
    _check("kq_adam_step", st)
    return params


def scales_to_tiled(scales: torch.Tensor, K: int, out=None):
    """Row-major scale bytes [rows, K/32] -> the tiled layout the tensor-core
    product reads (1-D uint8 of kq_scales_tiled_bytes(rows, K) bytes)."""
    _dev_tensor(scales, torch.uint8, "scales")
    rows = scales.shape[0]
    if scales.dim() != 2 or scales.shape[1] != K // 32:
        raise ValueError("scales must be [rows, K/32]")
    n = int(lib().kq_scales_tiled_bytes(rows, K))
    if out is None:
        out = torch.empty((n,), dtype=torch.uint8, device=scales.device)
    _dev_tensor(out, torch.uint8, "out")
    if out.numel() < n:
        raise ValueError("out is too small")
    st = lib().kq_scales_to_tiled(scales.data_ptr(), rows, K, out.data_ptr(),
                                  _stream(scales.device))
    _check("kq_scales_to_tiled", st)
    return out


def _quantize_tiled(fn: str, x: torch.Tensor, params: torch.Tensor, q=None, scales=None):
    _dev_tensor(x, torch.bfloat16, "x")
    M, d = _shape(x)
    _params(params, d)
    if q is None:
        q = torch.empty((M, d // 2), dtype=torch.uint8, device=x.device)
    n = int(lib().kq_scales_tiled_bytes(M, d))
    if scales is None:
        scales = torch.zeros((n,), dtype=torch.uint8, device=x.device)
    _dev_tensor(q, torch.uint8, "q")
    _dev_tensor(scales, torch.uint8, "scales")
    if tuple(q.shape) != (M, d // 2) or scales.numel() < n:
        raise ValueError("q must be [M, d/2] and scales hold kq_scales_tiled_bytes(M, d) bytes")
    st = getattr(lib(), fn)(x.data_ptr(), M, d, params.data_ptr(), q.data_ptr(),
                            scales.data_ptr(), _stream(x.device))
    _check(fn, st)
    return q, scales


def quantize_tiled(x: torch.Tensor, params: torch.Tensor, q=None, scales=None):
    """MXFP4(x T) with the scales in the tiled layout of the tensor-core product."""
    return _quantize_tiled("kq_quantize_tiled", x, params, q, scales)


def quantize_weight_tiled(w: torch.Tensor, params: torch.Tensor, q=None, scales=None):
    """MXFP4(W T^-T) with the scales in the tiled layout."""
    return _quantize_tiled("kq_quantize_weight_tiled", w, params, q, scales)


def gemm_mxfp4_tiled(qa: torch.Tensor, sa_tiled: torch.Tensor, qb: torch.Tensor,
                     sb_tiled: torch.Tensor, out=None, out_dtype=torch.float32):
    """C = A B^T with both operands' scales in the tiled layout."""
    for t, n in ((qa, "qa"), (sa_tiled, "sa_tiled"), (qb, "qb"), (sb_tiled, "sb_tiled")):
        _dev_tensor(t, torch.uint8, n)
    M, K = qa.shape[0], 2 * qa.shape[1]
    N = qb.shape[0]
    if tuple(qb.shape) != (N, K // 2):
        raise ValueError("qb must be [N, K/2]")
    if sa_tiled.numel() < lib().kq_scales_tiled_bytes(M, K) or \
            sb_tiled.numel() < lib().kq_scales_tiled_bytes(N, K):
        raise ValueError("tiled scale arrays are too small")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=qa.device)
    _dev_tensor(out, out_dtype, "out")
    code = KQ_OUT_F32 if out_dtype == torch.float32 else KQ_OUT_BF16
    st = lib().kq_gemm_mxfp4_tiled(qa.data_ptr(), sa_tiled.data_ptr(), qb.data_ptr(),
                                   sb_tiled.data_ptr(), M, N, K, out.data_ptr(), code,
                                   _stream(qa.device))
    _check("kq_gemm_mxfp4_tiled", st)
    return out


def inverse_transform(y: torch.Tensor, params: torch.Tensor, x=None):
    """x = y T^-1 in float32."""
    _dev_tensor(y, torch.float32, "y")
    M, d = _shape(y)
    _params(params, d)
    if x is None:
        x = torch.empty((M, d), dtype=torch.float32, device=y.device)
    _dev_tensor(x, torch.float32, "x")
    st = lib().kq_inverse_transform(y.data_ptr(), M, d, params.data_ptr(), x.data_ptr(),
                                    _stream(y.device))
    _check("kq_inverse_transform", st)
    return x


def dequantize(q: torch.Tensor, scales: torch.Tensor, y=None):
    """float32 [M, d] = E2M1(code) * 2^(scale - 127)."""
    _dev_tensor(q, torch.uint8, "q")
    _dev_tensor(scales, torch.uint8, "scales")
    M, half = q.shape
    d = 2 * half
    if tuple(scales.shape) != (M, d // 32):
        raise ValueError("scales must be [M, d/32]")
    if y is None:
        y = torch.empty((M, d), dtype=torch.float32, device=q.device)
    _dev_tensor(y, torch.float32, "y")
    st = lib().kq_dequantize(q.data_ptr(), scales.data_ptr(), M, d, y.data_ptr(), _stream(q.device))
    _check("kq_dequantize", st)
    return y


def host_workspace_bytes(d: int, rows_per_chunk: int) -> int:
    """Device workspace bytes quantize_host needs for chunks of that many rows."""
    return int(lib().kq_quantize_host_workspace_bytes(d, rows_per_chunk))


def _host_tensor(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor")
    return t


def quantize_host(x: torch.Tensor, params: torch.Tensor, q: torch.Tensor, scales: torch.Tensor,
                  workspace: torch.Tensor, stream=None):
    """MXFP4(x T) for host-resident x (pinned bf16 [M, d]) into host q / scales
    (pinned uint8), streamed through a device ``workspace`` (uint8 CUDA
    tensor).  Asynchronous on ``stream`` (default: the current stream of the
    workspace's device)."""
    _host_tensor(x, torch.bfloat16, "x")
    M, d = _shape(x)
    _host_tensor(q, torch.uint8, "q")
    _host_tensor(scales, torch.uint8, "scales")
    if tuple(q.shape) != (M, d // 2) or tuple(scales.shape) != (M, d // 32):
        raise ValueError("output shapes must be [M, d/2] and [M, d/32]")
    _dev_tensor(workspace, torch.uint8, "workspace")
    _params(params, d)
    st = stream if stream is not None else _stream(workspace.device)
    rc = lib().kq_quantize_host(x.data_ptr(), M, d, params.data_ptr(), q.data_ptr(),
                                scales.data_ptr(), workspace.data_ptr(), workspace.numel(), st)
    _check("kq_quantize_host", rc)
    return q, scales


def quantize_host_static(x: torch.Tensor, params: torch.Tensor, q: torch.Tensor,
                         scales: torch.Tensor, stream=None):
    """quantize_host without a workspace, for callers that cannot allocate
    device memory: the rows pass through a 16 MiB staging area built into the
    library.  Calls that overlap on the GPU share that area and must be
    serialised.  Runs on ``stream`` (default: the current CUDA stream of
    ``params``' device), with that device made current for the call.  The
    call is asynchronous: the host outputs are complete once the stream has
    reached this point, and every host buffer must stay alive until then."""
    _host_tensor(x, torch.bfloat16, "x")
    M, d = _shape(x)
    _host_tensor(q, torch.uint8, "q")
    _host_tensor(scales, torch.uint8, "scales")
    if tuple(q.shape) != (M, d // 2) or tuple(scales.shape) != (M, d // 32):
        raise ValueError("output shapes must be [M, d/2] and [M, d/32]")
    _params(params, d)
    # The staging area is looked up on the current device: make it the one
    # that holds the parameters and the stream.
    with torch.cuda.device(params.device):
        st = stream if stream is not None else _stream(params.device)
        rc = lib().kq_quantize_host_static(x.data_ptr(), M, d, params.data_ptr(),
                                           q.data_ptr(), scales.data_ptr(), st)
    _check("kq_quantize_host_static", rc)
    return q, scales


def device_status() -> int:
    """Synchronise and return (and clear) the device-side wait-timeout flags."""
    flags = _int(0)
    _check("kq_device_status", lib().kq_device_status(ctypes.byref(flags)))
    return flags.value
