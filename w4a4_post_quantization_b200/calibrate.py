"""Straight-through calibration of the Kronecker transform on one linear layer
``y = x W^T`` (KroQuant review, "What carries the argument" and the
free-parameter ledger: the 15 parameters of every 32x32 block are learned per
layer by minimizing the quantized output error with auxiliary per-operand
regularization, Adam with a straight-through estimator, 100 steps at lr 1e-2,
from the Hadamard initialization; the regularization weights come from the
loss ratios at the initialization).

Loss at parameters theta (A = X T, B = W T^-T, Q = MXFP4):

    L = |Q(A) Q(B)^T - X W^T|^2 / |X W^T|^2 + lam_A |Q(A) - A|^2 + lam_W |Q(B) - B|^2

with lam_A, lam_W making each auxiliary term equal to the output term at
the initialization.  Every step runs in the library's kernels: the transform,
the weight fold and both quantizers, the W4A4 product on the tensor cores,
the residual, the parameter gradients through the Kronecker factors and the
Adam update; the two float32 products R Q(B) and R^T Q(A) that carry the
output gradient back to the operands, and the reference X W^T, are plain
cuBLAS GEMMs.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import _lib as L

HADAMARD_INIT = (-1.0, 1.0 / math.sqrt(2.0), 1.0 / math.sqrt(2.0))


def hadamard_params(nb: int, device) -> torch.Tensor:
    """[nb, 5, 3] float32 at the Hadamard initialization: every factor is the
    45-degree rotation (a, b, c) = (-1, 1/sqrt2, 1/sqrt2), so each block is a
    Hadamard matrix up to row signs (the unit-determinant form cannot hold
    H2/sqrt2 itself)."""
    p = torch.empty((nb, 5, 3), dtype=torch.float32, device=device)
    p[:, :, 0], p[:, :, 1], p[:, :, 2] = HADAMARD_INIT
    return p


class LayerCalibrator:
    """Buffers and kernel sequence of the calibration of one layer.

    ``x``: bf16 activations [M, d]; ``w``: bf16 weights [N, d] (rows are
    output channels); both on the same CUDA device.
    """

    def __init__(self, x: torch.Tensor, w: torch.Tensor, params0: Optional[torch.Tensor] = None):
        dev = x.device
        M, d = x.shape
        N = w.shape[0]
        if w.shape[1] != d or d % 32:
            raise ValueError("x [M, d] and w [N, d] with d a multiple of 32")
        self.x, self.w = x, w
        self.params = (hadamard_params(d // 32, dev) if params0 is None
                       else params0.to(dev, torch.float32).clone().contiguous())
        f32 = dict(dtype=torch.float32, device=dev)
        u8 = dict(dtype=torch.uint8, device=dev)
        self.A, self.Aq = torch.empty((M, d), **f32), torch.empty((M, d), **f32)
        self.B, self.Bq = torch.empty((N, d), **f32), torch.empty((N, d), **f32)
        self.qa, self.sa = torch.empty((M, d // 2), **u8), torch.empty((M, d // 32), **u8)
        self.qb, self.sb = torch.empty((N, d // 2), **u8), torch.empty((N, d // 32), **u8)
        self.Y, self.R = torch.empty((M, N), **f32), torch.empty((M, N), **f32)
        self.dpa, self.dpb = torch.empty((d // 32, 5, 3), **f32), torch.empty((d // 32, 5, 3), **f32)
        self.rega, self.regb = torch.empty((1,), **f32), torch.empty((1,), **f32)
        self.sumsq = torch.empty((1,), dtype=torch.float64, device=dev)
        self.m, self.v = torch.zeros_like(self.params), torch.zeros_like(self.params)
        self.ws_a = torch.zeros((L.params_grad_workspace_bytes(M, d),), **u8)
        self.ws_b = torch.zeros((L.params_grad_workspace_bytes(N, d),), **u8)
        self.ws_r = torch.zeros((L.residual_workspace_bytes(),), **u8)
        # Reference output X W^T (float32 products of the bf16 operands).
        self.y_ref = torch.matmul(x.float(), w.float().t())
        zero = torch.zeros_like(self.y_ref)
        _, ss = L.residual(self.y_ref, zero, 1.0, self.ws_r, out=torch.empty_like(zero))
        self.s = float(ss.item())
        self.t = 0
        self.lam_a = self.lam_w = None

    def forward(self) -> None:
        """A, B, their quantized values and codes, Y = Q(A) Q(B)^T, and
        R = 2 (Y - X W^T) / |X W^T|^2 (the output term's gradient in Y)."""
        p = self.params
        L.transform(self.x, p, y=self.A)
        L.quantize(self.x, p, self.qa, self.sa)
        L.dequantize(self.qa, self.sa, y=self.Aq)
        L.fold_weight(self.w, p, out=self.B)
        L.quantize_weight(self.w, p, self.qb, self.sb)
        L.dequantize(self.qb, self.sb, y=self.Bq)
        L.gemm_mxfp4(self.qa, self.sa, self.qb, self.sb, out=self.Y)
        L.residual(self.Y, self.y_ref, 2.0 / self.s, self.ws_r, out=self.R, sumsq=self.sumsq)

    def losses(self):
        """(L_out, L_A, L_W) at the current parameters (synchronizes)."""
        self.forward()
        l_out = float(self.sumsq.item()) / self.s
        tmp = torch.empty_like(self.A)
        _, la = L.residual(self.Aq, self.A, 1.0, self.ws_r, out=tmp)
        l_a = float(la.item())
        tmp = torch.empty_like(self.B)
        _, lw = L.residual(self.Bq, self.B, 1.0, self.ws_r, out=tmp)
        return l_out, l_a, float(lw.item())

    def gradient(self, lam_a: float, lam_w: float):
        """Forward pass, then the straight-through gradient of L into
        ``dpa`` (activation side) and ``dpb`` (weight side); returns the
        device scalars (|Y - X W^T|^2, |Q(A) - A|^2, |Q(B) - B|^2)."""
        self.forward()
        ga = torch.matmul(self.R, self.Bq)          # dL_out / dQ(A)
        gb = torch.matmul(self.R.t(), self.Aq)      # dL_out / dQ(B)
        L.transform_params_grad(self.A, self.Aq, ga, self.params, False, lam_a, self.ws_a,
                                self.dpa, self.rega)
        L.transform_params_grad(self.B, self.Bq, gb, self.params, True, lam_w, self.ws_b,
                                self.dpb, self.regb)
        return self.sumsq, self.rega, self.regb

    def run(self, steps: int = 100, lr: float = 1e-2):
        """Adam from the current parameters; returns the total loss before
        each step (one synchronization at the end)."""
        if self.lam_a is None:
            l_out, l_a, l_w = self.losses()
            self.lam_a, self.lam_w = l_out / l_a, l_out / l_w
        hist = torch.empty((steps,), dtype=torch.float64, device=self.params.device)
        for i in range(steps):
            ss, ra, rb = self.gradient(self.lam_a, self.lam_w)
            hist[i] = ss[0] / self.s + self.lam_a * ra[0].double() + self.lam_w * rb[0].double()
            self.t += 1
            L.adam_step(self.params, self.dpa, self.dpb, self.m, self.v, self.t, lr)
        return hist.cpu().tolist()


def calibrate_layer(x: torch.Tensor, w: torch.Tensor, steps: int = 100, lr: float = 1e-2,
                    params0: Optional[torch.Tensor] = None):
    """Calibrated parameters [d/32, 5, 3] and the loss before each step."""
    cal = LayerCalibrator(x, w, params0)
    hist = cal.run(steps, lr)
    return cal.params, hist, (cal.lam_a, cal.lam_w)
