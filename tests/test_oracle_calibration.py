"""Pins for the calibration oracle (``oracle.kq_calibration``): each check
ties a step to something other than its own code -- central finite
differences, closed forms, textbook identities -- so that a wrong partial, a
dropped transpose or a mis-signed term fails here."""
import math

import numpy as np

from oracle import kq_calibration as c
from oracle import kq_oracle as o


def _params(nb, seed):
    rng = np.random.default_rng(seed)
    p = np.empty((nb, 5, 3))
    p[:, :, 0] = rng.uniform(-1, 1, (nb, 5))
    p[:, :, 1] = 2.0 ** rng.uniform(-0.5, 0.5, (nb, 5))
    p[:, :, 2] = rng.uniform(-1, 1, (nb, 5))
    return p


def _fd(f, p, h=1e-6):
    g = np.zeros_like(p)
    for idx in np.ndindex(p.shape):
        e = np.zeros_like(p)
        e[idx] = h
        g[idx] = (f(p + e) - f(p - e)) / (2 * h)
    return g


def test_param_gradient_of_the_transform_matches_finite_differences():
    """L = sum(g * (x T)) is linear in T, so dL/dtheta is exactly the
    transform gradient; central differences agree to O(h^2)."""
    rng = np.random.default_rng(1)
    x, g = rng.standard_normal((7, 64)), rng.standard_normal((7, 64))
    p = _params(2, 2)
    got = c.transform_params_grad(x, g, p)
    ref = _fd(lambda q: np.sum(g * o.transform(x, q)), p)
    np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-7)


def test_param_gradient_of_the_weight_fold_matches_finite_differences():
    rng = np.random.default_rng(3)
    w, g = rng.standard_normal((5, 64)), rng.standard_normal((5, 64))
    p = _params(2, 4)
    got = c.transform_params_grad(w, g, p, inverse_transpose=True)
    ref = _fd(lambda q: np.sum(g * o.fold_weight(w, q)), p)
    np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-7)


def test_ste_gradient_is_the_gradient_of_the_linearized_loss():
    """With the quantization offsets frozen at theta0 (Q(v) = v + delta0 in
    the output term, Q(v) = const in the regularizers), the surrogate loss's
    finite-difference gradient at theta0 equals the oracle's STE gradient."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((12, 64))
    x[:, 3] *= 20
    w = rng.standard_normal((9, 64)) / 8
    p0 = _params(2, 6)
    lam_a, lam_w = 0.3, 0.7
    y_ref = x @ w.T
    s = np.sum(y_ref ** 2)
    A0, B0, Aq0, Bq0, _ = c.layer_terms(x, w, p0)
    dA, dB = Aq0 - A0, Bq0 - B0

    def surrogate(q):
        A, B = o.transform(x, q), o.fold_weight(w, q)
        R = (A + dA) @ (B + dB).T - y_ref
        return np.sum(R ** 2) / s + lam_a * np.sum((Aq0 - A) ** 2) + \
            lam_w * np.sum((Bq0 - B) ** 2)

    _, _, got = c.loss_and_grad(x, w, p0, lam_a, lam_w)
    ref = _fd(surrogate, p0, h=1e-6)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-8)


def test_adam_first_step_is_lr_times_the_sign():
    """Bias-corrected Adam's first update is lr g / (|g| + eps)."""
    g = np.array([3.0, -2e-3, 0.5, -7.0])
    p, m, v = c.adam_step(np.zeros(4), g, np.zeros(4), np.zeros(4), 1, 1e-2)
    np.testing.assert_allclose(p, -1e-2 * g / (np.abs(g) + c.ADAM_EPS), rtol=1e-12)
    np.testing.assert_allclose(m, 0.1 * g)
    np.testing.assert_allclose(v, 0.001 * g * g)


def test_hadamard_initialization_is_an_orthonormal_signed_hadamard():
    K = o.kron_block(c.hadamard_params(1)[0])
    np.testing.assert_allclose(K @ K.T, np.eye(32), atol=1e-6)
    np.testing.assert_allclose(np.abs(K), 1 / math.sqrt(32), atol=1e-7)
    # orthonormal: the weight fold equals the transform itself
    w = np.random.default_rng(7).standard_normal((3, 32))
    np.testing.assert_allclose(o.fold_weight(w, c.hadamard_params(1)), o.transform(
        w, c.hadamard_params(1)), atol=1e-6)


def test_regularization_weights_equalize_the_terms_at_init():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((16, 64))
    w = rng.standard_normal((8, 64)) / 8
    p0 = c.hadamard_params(2)
    lam_a, lam_w = c.regularization_weights(x, w, p0)
    l_out, l_a, l_w = c.losses(x, w, p0)
    assert math.isclose(lam_a * l_a, l_out, rel_tol=1e-12)
    assert math.isclose(lam_w * l_w, l_out, rel_tol=1e-12)


def test_abs_gradient_bounds_the_gradient():
    rng = np.random.default_rng(9)
    x, g = rng.standard_normal((6, 64)), rng.standard_normal((6, 64))
    p = _params(2, 10)
    for inv in (False, True):
        assert (np.abs(c.transform_params_grad(x, g, p, inv)) <=
                c.abs_transform_params_grad(x, g, p, inv) * (1 + 1e-12)).all()


def test_calibration_loop_starts_at_three_output_losses_and_steps_by_adam():
    """The loop's first recorded loss is L_out + lam_a L_A + lam_w L_W at the
    Hadamard start, which the Eq. 10 weights make exactly 3 L_out; its first
    step is bias-corrected Adam's, a move of lr g / (|g| + eps) against the
    straight-through gradient, and its parameters come back in float32."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((16, 64))
    x[:, 7] *= 30
    w = rng.standard_normal((8, 64)) / 8
    p0 = c.hadamard_params(2)
    l_out, _, _ = c.losses(x, w, p0)
    p1, hist, (lam_a, lam_w) = c.calibrate(x, w, steps=1, lr=1e-3)
    assert len(hist) == 1 and math.isclose(hist[0], 3 * l_out, rel_tol=1e-12)
    assert p1.dtype == np.float32 and p1.shape == p0.shape
    _, _, g = c.loss_and_grad(x, w, p0, lam_a, lam_w)
    step = p1.astype(np.float64) - p0.astype(np.float64)
    np.testing.assert_allclose(step, -1e-3 * g / (np.abs(g) + c.ADAM_EPS), rtol=0, atol=1e-7)
    # a second step continues from the first, with the moments carried over
    p2, hist2, _ = c.calibrate(x, w, steps=2, lr=1e-3)
    assert hist2[0] == hist[0] and np.array_equal(
        c.calibrate(x, w, steps=1, lr=1e-3, params0=p0)[0], p1)
    assert not np.array_equal(p2, p1)
