"""CPU oracle for the calibration of the Kronecker transform on one linear
layer (float64, numpy).

TEST INFRASTRUCTURE ONLY, like ``oracle.kq_oracle``: the GPU calibration is
checked against it and it is never on the product path.

What it follows (KroQuant review, pith.science: "What carries the argument",
the axiom and free-parameter ledger, "What would settle it"):

* each layer's transform is fitted by driving down the mean squared error
  of the quantized layer output, plus one extra penalty term for each of the
  two quantized operands (Eq. 2, 7, 9), with a
  straight-through estimator through the quantizer (Section 3.3);
* the regularization weights are set from the loss ratios at the
  initialization (Eq. 10); the optimizer is Adam, 100 steps, lr 1e-2
  (Appendix D.1 as the ledger quotes it);
* the initialization is the Hadamard transform.

Readings where the pages print no formula:

* loss ``L = L_out + lam_A L_A + lam_W L_W`` with
  ``L_out = |Q(A) Q(B)^T - X W^T|^2 / |X W^T|^2``, ``A = X T``,
  ``B = W T^-T``, ``L_A = |Q(A) - A|^2``, ``L_W = |Q(B) - B|^2`` (sums of
  squares over all elements);
* ``lam_A = L_out(theta0) / L_A(theta0)`` and likewise ``lam_W``: each
  auxiliary term starts equal to the output loss;
* straight-through estimator: the quantizer's Jacobian is the identity in
  ``L_out``; in ``L_A`` and ``L_W`` the quantized operand is a constant (the
  gradient pulls an operand toward its own quantized value);
* the Hadamard initialization in the unit-determinant form is
  ``(a, b, c) = (-1, 1/sqrt2, 1/sqrt2)`` for every factor, the rotation by
  45 degrees (a Hadamard matrix up to the signs of its rows; the form cannot
  hold ``H2/sqrt2`` itself, whose determinant is -1);
* Adam with the usual ``beta1 = 0.9``, ``beta2 = 0.999``, ``eps = 1e-8`` and
  bias correction.
"""
from __future__ import annotations

import math

import numpy as np

from oracle import kq_oracle as o

HADAMARD_INIT = (-1.0, 1.0 / math.sqrt(2.0), 1.0 / math.sqrt(2.0))
ADAM_BETA1, ADAM_BETA2, ADAM_EPS = 0.9, 0.999, 1e-8


def hadamard_params(nb: int, n_factors: int = o.N_FACTORS) -> np.ndarray:
    """``[nb, n_factors, 3]`` float32 parameters at the Hadamard initialization."""
    p = np.empty((nb, n_factors, 3), dtype=np.float32)
    p[:, :, 0], p[:, :, 1], p[:, :, 2] = HADAMARD_INIT
    return p


def fake_quant(v64: np.ndarray) -> np.ndarray:
    """``Q(v)``: MXFP4 quantize then dequantize (the value the codes stand
    for), the decision taken on float32 values."""
    codes, scales = o.mxfp4_quantize(v64)
    return o.dequantize(o.pack_codes(codes), scales)


# ----------------------------------------------------------------- factors
def factor_entries(a, b, c):
    """``G = [[b, c], [a b, a c + 1/b]]`` (row-vector form)."""
    return np.array([[b, c], [a * b, a * c + 1.0 / b]])


def factor_partials(a, b, c):
    """``dG/da``, ``dG/db``, ``dG/dc``."""
    return (np.array([[0.0, 0.0], [b, c]]),
            np.array([[1.0, 0.0], [a, -1.0 / (b * b)]]),
            np.array([[0.0, 1.0], [0.0, a]]))


def inverse_transpose_entries(a, b, c):
    """``(G^-1)^T = [[g11, -g10], [-g01, g00]]`` (det G = 1)."""
    g = factor_entries(a, b, c)
    return np.array([[g[1, 1], -g[1, 0]], [-g[0, 1], g[0, 0]]])


def inverse_transpose_partials(a, b, c):
    """Partials of ``(G^-1)^T`` with respect to ``a``, ``b``, ``c``."""
    return (np.array([[c, -b], [0.0, 0.0]]),
            np.array([[-1.0 / (b * b), -a], [0.0, 1.0]]),
            np.array([[a, 0.0], [-1.0, 0.0]]))


def block_grad_params(dK: np.ndarray, p_j: np.ndarray, inverse_transpose: bool) -> np.ndarray:
    """Gradient of a loss with respect to one block's ``[5, 3]`` parameters,
    from its gradient with respect to the dense block ``dK`` (32x32):
    ``dL/dtheta = sum_rc dL/dK[r,c] dK[r,c]/dtheta`` with
    ``K = F1 (x) ... (x) F5`` and ``F_k = G_k`` or ``(G_k^-1)^T``."""
    p_j = np.asarray(p_j, dtype=np.float64)
    ent = inverse_transpose_entries if inverse_transpose else factor_entries
    par = inverse_transpose_partials if inverse_transpose else factor_partials
    F = [ent(*p_j[k]) for k in range(p_j.shape[0])]
    out = np.zeros(p_j.shape)
    for k in range(p_j.shape[0]):
        for t, dF in enumerate(par(*p_j[k])):
            dK_k = o.kron_factors(F[:k] + [dF] + F[k + 1:])
            out[k, t] = np.sum(dK * dK_k)
    return out


def transform_params_grad(x64: np.ndarray, g64: np.ndarray, params: np.ndarray,
                          inverse_transpose: bool = False) -> np.ndarray:
    """Gradient with respect to the parameters of ``Z = x K`` (per 32-block:
    ``K = T`` blocks, or ``T^-T`` blocks with ``inverse_transpose``) given
    ``g = dL/dZ``: ``dL/dK_j = x_j^T g_j`` contracted with ``dK_j/dtheta``."""
    params = np.asarray(params, dtype=np.float64)
    out = np.zeros(params.shape)
    for j in range(params.shape[0]):
        sl = slice(32 * j, 32 * (j + 1))
        out[j] = block_grad_params(x64[:, sl].T @ g64[:, sl], params[j], inverse_transpose)
    return out


def abs_transform_params_grad(x64, g64, params, inverse_transpose=False):
    """The same contraction with every term replaced by its magnitude: the
    size of the sum each gradient entry is, for stating tolerances."""
    params = np.asarray(params, dtype=np.float64)
    out = np.zeros(params.shape)
    ent = inverse_transpose_entries if inverse_transpose else factor_entries
    par = inverse_transpose_partials if inverse_transpose else factor_partials
    for j in range(params.shape[0]):
        sl = slice(32 * j, 32 * (j + 1))
        dK = np.abs(x64[:, sl]).T @ np.abs(g64[:, sl])
        F = [np.abs(ent(*params[j, k])) for k in range(params.shape[1])]
        for k in range(params.shape[1]):
            for t, dF in enumerate(par(*params[j, k])):
                out[j, k, t] = np.sum(dK * o.kron_factors(F[:k] + [np.abs(dF)] + F[k + 1:]))
    return out


# ------------------------------------------------------------ loss and step
def layer_terms(x64: np.ndarray, w64: np.ndarray, params: np.ndarray):
    """Forward pass of the transformed layer: ``A = X T``, ``B = W T^-T``,
    their fake-quantized values and the quantized output ``Y = Q(A) Q(B)^T``."""
    A = o.transform(x64, params)
    B = o.fold_weight(w64, params)
    Aq, Bq = fake_quant(A), fake_quant(B)
    return A, B, Aq, Bq, Aq @ Bq.T


def losses(x64, w64, params, y_ref=None):
    """``(L_out, L_A, L_W)`` at ``params`` (``y_ref = X W^T``)."""
    if y_ref is None:
        y_ref = x64 @ w64.T
    A, B, Aq, Bq, Y = layer_terms(x64, w64, params)
    return (np.sum((Y - y_ref) ** 2) / np.sum(y_ref ** 2), np.sum((Aq - A) ** 2),
            np.sum((Bq - B) ** 2))


def regularization_weights(x64, w64, params0):
    """Eq. 10 reading: each auxiliary term starts equal to the output loss."""
    l_out, l_a, l_w = losses(x64, w64, params0)
    return l_out / l_a, l_out / l_w


def loss_and_grad(x64, w64, params, lam_a, lam_w, y_ref=None):
    """Total loss and its straight-through gradient with respect to the
    ``[nb, 5, 3]`` parameters."""
    if y_ref is None:
        y_ref = x64 @ w64.T
    s = np.sum(y_ref ** 2)
    A, B, Aq, Bq, Y = layer_terms(x64, w64, params)
    R = Y - y_ref
    l_out = np.sum(R ** 2) / s
    l_a, l_w = np.sum((Aq - A) ** 2), np.sum((Bq - B) ** 2)
    gA = 2.0 * (R @ Bq) / s + lam_a * 2.0 * (A - Aq)
    gB = 2.0 * (R.T @ Aq) / s + lam_w * 2.0 * (B - Bq)
    grad = transform_params_grad(x64, gA, params) + \
        transform_params_grad(w64, gB, params, inverse_transpose=True)
    return l_out + lam_a * l_a + lam_w * l_w, (l_out, l_a, l_w), grad


def adam_step(params, grad, m, v, t, lr):
    """One Adam update (step number ``t`` from 1), float64."""
    m = ADAM_BETA1 * m + (1.0 - ADAM_BETA1) * grad
    v = ADAM_BETA2 * v + (1.0 - ADAM_BETA2) * grad * grad
    mhat = m / (1.0 - ADAM_BETA1 ** t)
    vhat = v / (1.0 - ADAM_BETA2 ** t)
    return params - lr * mhat / (np.sqrt(vhat) + ADAM_EPS), m, v


def calibrate(x64, w64, steps: int = 100, lr: float = 1e-2, params0=None):
    """Adam on the straight-through gradient from the Hadamard
    initialization; returns the final parameters (float32, as the library
    stores them) and the total loss before each step."""
    nb = x64.shape[1] // o.BLOCK
    p = (hadamard_params(nb) if params0 is None else np.asarray(params0, np.float32))
    p = p.astype(np.float64)
    y_ref = x64 @ w64.T
    lam_a, lam_w = regularization_weights(x64, w64, p.astype(np.float32))
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    history = []
    for t in range(1, steps + 1):
        # The transform is evaluated at the float32 parameters the kernels use.
        total, _, g = loss_and_grad(x64, w64, p.astype(np.float32), lam_a, lam_w, y_ref)
        history.append(total)
        p, m, v = adam_step(p, g, m, v, t, lr)
    return p.astype(np.float32), history, (lam_a, lam_w)

