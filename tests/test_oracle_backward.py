"""Pins of the frame-step backward in oracle/vda_oracle.py against central finite
differences of the forward frame step, and against special cases in which a
gradient vanishes. The differences use the forward oracle only; the backward's
algebra is not retyped here."""
import numpy as np
import pytest

from oracle import vda_oracle as vo


def _case(seed, U=5, d_k=4, d_v=3, beta_scale=1.0):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((U, d_k))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((U, d_v))
    beta = beta_scale / (1 + np.exp(-rng.standard_normal(U)))
    alpha = 1 / (1 + np.exp(-(rng.standard_normal(d_k) + 2)))
    S_prev = rng.standard_normal((d_v, d_k))
    dS = rng.standard_normal((d_v, d_k))
    return S_prev, K, V, beta, alpha, dS


def _fd(fn, x, direction, h=1e-6):
    return (fn(x + h * direction) - fn(x - h * direction)) / (2 * h)


NAMES = ["S_prev", "K", "V", "beta", "alpha"]


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("which", NAMES)
def test_backward_matches_finite_differences(seed, which):
    args = list(_case(seed))
    dS = args.pop()
    grads = vo.frame_step_backward(*args, dS)
    key = {"S_prev": "dS_prev", "K": "dK", "V": "dV", "beta": "dbeta", "alpha": "dalpha"}[which]
    i = NAMES.index(which)
    rng = np.random.default_rng(100 + seed)
    for _ in range(3):
        direction = rng.standard_normal(args[i].shape)

        def loss(x):
            a = list(args)
            a[i] = x
            return float(np.sum(dS * vo.frame_step(*a)))

        want = _fd(loss, args[i], direction)
        got = float(np.sum(grads[key] * direction))
        assert abs(got - want) <= 1e-6 * (1 + abs(want)), (which, got, want)


def test_backward_on_a_wider_frame():
    """d = 8, U = 12: every entry's gradient by coordinate-wise differences."""
    S_prev, K, V, beta, alpha, dS = _case(7, U=12, d_k=8, d_v=8)
    grads = vo.frame_step_backward(S_prev, K, V, beta, alpha, dS)
    args = [S_prev, K, V, beta, alpha]
    for i, key in enumerate(["dS_prev", "dK", "dV", "dbeta", "dalpha"]):
        x = args[i]
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            e = np.zeros_like(x)
            e[idx] = 1.0

            def loss(y):
                a = list(args)
                a[i] = y
                return float(np.sum(dS * vo.frame_step(*a)))

            num[idx] = _fd(loss, x, e)
        np.testing.assert_allclose(grads[key], num, rtol=1e-6, atol=1e-8)


def test_zero_write_strength_freezes_keys_and_values():
    """beta = 0: the frame writes nothing, so K and V get no gradient, and the
    step reduces to S_prev Diag(alpha): dS_prev = dS Diag(alpha)."""
    S_prev, K, V, beta, alpha, dS = _case(3)
    g = vo.frame_step_backward(S_prev, K, V, np.zeros_like(beta), alpha, dS)
    assert np.all(g["dK"] == 0) and np.all(g["dV"] == 0)
    np.testing.assert_allclose(g["dS_prev"], dS * alpha[None, :], rtol=1e-14)
    np.testing.assert_allclose(g["dalpha"], np.sum(S_prev * dS, axis=0), rtol=1e-12)


def test_zero_decay_cuts_the_state_path():
    S_prev, K, V, beta, alpha, dS = _case(4)
    g = vo.frame_step_backward(S_prev, K, V, beta, np.zeros_like(alpha), dS)
    assert np.all(g["dS_prev"] == 0)


def test_planted_sign_error_is_caught():
    """A backward with dL/dA's sign flipped fails the finite-difference pin."""
    S_prev, K, V, beta, alpha, dS = _case(5)
    good = vo.frame_step_backward(S_prev, K, V, beta, alpha, dS)
    A, B = vo.frame_stats(K, V, beta)
    P = np.linalg.inv(np.eye(A.shape[0]) + A)
    Gx = dS @ P
    S = (S_prev * alpha + B) @ P
    GA_wrong = +(S.T @ Gx)
    dK_wrong = beta[:, None] * (K @ (GA_wrong + GA_wrong.T).T + V @ Gx)
    direction = np.random.default_rng(0).standard_normal(K.shape)

    def loss(x):
        return float(np.sum(dS * vo.frame_step(S_prev, x, V, beta, alpha)))

    want = _fd(loss, K, direction)
    assert abs(np.sum(good["dK"] * direction) - want) <= 1e-6 * (1 + abs(want))
    assert abs(np.sum(dK_wrong * direction) - want) > 1e-3
