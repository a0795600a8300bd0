"""Pins of the Adam oracle against closed forms that the published algorithm
implies (bias-corrected Adam, Kingma and Ba 2015; decoupled weight decay,
Loshchilov and Hutter 2019), chosen so that a dropped bias correction, a
swapped beta, a missing square root, epsilon under the root, coupled weight
decay or a wrong sign each fail one of them."""
import numpy as np
import pytest

from oracle import adam, nf4

rng = np.random.default_rng(20260)


def _state(n):
    theta = rng.standard_normal(n) * 0.02
    g = rng.standard_normal(n) * 1e-3
    return theta, g


def test_first_step_from_zero_state_is_sign_like():
    # m_1 = (1-b1) g, v_1 = (1-b2) g^2; after bias correction m_hat = g, v_hat = g^2,
    # so the step is lr * g / (|g| + eps)
    theta, g = _state(1000)
    g[:10] = 1e-8                                   # |g| = eps: epsilon outside the root matters
    lr, eps = 3e-4, 1e-8
    out = adam.adam_step(theta, np.zeros_like(g), np.zeros_like(g), g, t=1, lr=lr, eps=eps)
    expect = theta - lr * g / (np.abs(g) + eps)
    np.testing.assert_allclose(out["theta"], expect, rtol=0, atol=1e-15)
    np.testing.assert_allclose(out["m"], 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(out["v"], 0.001 * g * g, rtol=1e-12)


@pytest.mark.parametrize("b1,b2", [(0.9, 0.999), (0.5, 0.9), (0.0, 0.99)])
def test_constant_gradient_moves_by_lr_per_step(b1, b2):
    # with a constant gradient, m_t = (1 - b1^t) g and v_t = (1 - b2^t) g^2 exactly,
    # so the bias-corrected ratio is g / |g| at every step
    theta, g = _state(256)
    lr, eps = 1e-3, 0.0
    m = np.zeros_like(g)
    v = np.zeros_like(g)
    th = theta.copy()
    for t in range(1, 41):
        out = adam.adam_step(th, m, v, g, t=t, lr=lr, beta1=b1, beta2=b2, eps=eps)
        th, m, v = out["theta"], out["m"], out["v"]
        np.testing.assert_allclose(m, (1 - b1 ** t) * g, rtol=1e-12, atol=1e-300)
        np.testing.assert_allclose(v, (1 - b2 ** t) * g * g, rtol=1e-12)
    np.testing.assert_allclose(th, theta - 40 * lr * np.sign(g), rtol=0, atol=1e-13)


def test_decoupled_weight_decay_shrinks_geometrically():
    # zero gradient and zero state: theta_t = theta (1 - lr wd)^t exactly in real arithmetic
    theta, _ = _state(128)
    z = np.zeros_like(theta)
    lr, wd = 1e-2, 0.1
    th, m, v = theta.copy(), z, z
    for t in range(1, 11):
        out = adam.adam_step(th, m, v, z, t=t, lr=lr, weight_decay=wd)
        th, m, v = out["theta"], out["m"], out["v"]
    np.testing.assert_allclose(th, theta * (1 - lr * wd) ** 10, rtol=1e-13)
    assert np.all(m == 0) and np.all(v == 0)


def test_scale_invariance_without_epsilon():
    # m_hat / sqrt(v_hat) does not change when every gradient is scaled by c > 0
    theta, g = _state(512)
    m = rng.standard_normal(512) * 1e-4
    v = rng.random(512) * 1e-6
    a = adam.adam_step(theta, m, v, g, t=7, lr=1e-3, eps=0.0)
    b = adam.adam_step(theta, 64.0 * m, 4096.0 * v, 64.0 * g, t=7, lr=1e-3, eps=0.0)
    np.testing.assert_allclose(a["theta"], b["theta"], rtol=0, atol=1e-15)


def test_bf16_copy_is_the_rounded_master():
    theta, g = _state(300)
    out = adam.adam_step(theta, np.zeros_like(g), np.zeros_like(g), g, t=3, lr=1e-4)
    back = nf4.bf16_to_f64(out["theta_bf16"])
    # nearest bf16: within half a bf16 ulp of the master value
    ulp = np.ldexp(1.0, np.frexp(np.abs(out["theta"]))[1] - 8)
    assert np.all(np.abs(back - out["theta"]) <= ulp / 2)


def test_rejects_step_zero():
    with pytest.raises(ValueError):
        adam.adam_step(np.zeros(2), np.zeros(2), np.zeros(2), np.zeros(2), t=0, lr=1e-3)


def test_state_bytes_match_the_pages_accounting():
    # [P2] "The LoRA hypothesis": a rank-8 adapter on 4096 x 4096 has 65,536 parameters;
    # master + m + v in fp32 and the bf16 copy: 14 bytes each
    n = 4096 * 8 + 8 * 4096
    assert n == 65536
    assert adam.optimizer_state_bytes(n) == 14 * 65536
