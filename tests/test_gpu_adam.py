"""GPU parity of lora_adam_step against the float64 Adam oracle."""
import numpy as np
import pytest
import torch

from oracle import adam
from tests.gpu_helpers import bf16_host_bits

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def _state(n, seed):
    rng = np.random.Generator(np.random.Philox(key=seed))
    theta = (rng.standard_normal(n) * 0.02).astype(np.float32)
    m = (rng.standard_normal(n) * 1e-4).astype(np.float32)
    v = (rng.random(n) * 1e-7).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    return theta, m, v, g


def f32(x):
    """The hyperparameters cross the C ABI as fp32: give the oracle the same values."""
    return float(np.float32(x))


B1, B2, EPS = f32(0.9), f32(0.999), f32(1e-8)


def step_bound(ref, theta_prev, m_prev, g, t, lr, wd=0.0):
    """lr (|beta1 m| + |(1-beta1) g|) / (1-beta1^t) / (sqrt(v_hat) + eps) + lr wd |theta|:
    the terms of the step before any cancellation (in m, or between the Adam
    term and the decay); the fp32 error of a step is a few roundings of these."""
    m_terms = B1 * np.abs(m_prev) + (1 - B1) * np.abs(g)
    v_hat = ref["v"] / (1 - B2 ** t)
    return lr * (m_terms / (1 - B1 ** t) / (np.sqrt(v_hat) + EPS) + wd * np.abs(theta_prev))


def _dev(x, dtype=torch.float32):
    return torch.from_numpy(x).to("cuda", dtype)


def _check(ref, theta_g, m_g, v_g, w16_g, step_size, steps=1):
    """step_size: bound on the terms of the steps over the run (step_bound); the
    error of each fp32 step is a few roundings of those terms."""
    th = theta_g.cpu().numpy().astype(np.float64)
    mm = m_g.cpu().numpy().astype(np.float64)
    vv = v_g.cpu().numpy().astype(np.float64)
    f32 = 2.0 ** -23
    # m can cancel to near zero: its error is relative to the terms, not the sum
    np.testing.assert_allclose(mm, ref["m"], rtol=4 * steps * f32,
                               atol=8 * steps * f32 * np.abs(ref["m"]).max())
    np.testing.assert_allclose(vv, ref["v"], rtol=4 * steps * f32, atol=1e-30)
    tol = 2 * steps * f32 * np.abs(ref["theta"]) + 16 * f32 * step_size
    assert np.all(np.abs(th - ref["theta"]) <= tol)
    # the bf16 copy is the GPU master rounded to nearest, bit for bit
    assert torch.equal(w16_g.view(torch.int16), theta_g.to(torch.bfloat16).view(torch.int16))
    # and within one bf16 ulp of the oracle's rounding of its own master
    got = bf16_host_bits(w16_g).astype(np.int32)
    assert np.all(np.abs(got - ref["theta_bf16"].astype(np.int32)) <= 1)


@pytest.mark.parametrize("n", [1, 4, 7, 1000003])
@pytest.mark.parametrize("t", [1, 10, 1000])
def test_one_step(n, t):
    theta, m, v, g = _state(n, 11 * n + t)
    lr, wd = f32(2e-4), f32(0.01)
    th_g, m_g, v_g, g_g = _dev(theta), _dev(m), _dev(v), _dev(g)
    w16 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    q4.lora_adam_step(th_g, w16, m_g, v_g, g_g, step=t, lr=lr, beta1=B1, beta2=B2, eps=EPS, weight_decay=wd)
    torch.cuda.synchronize()
    ref = adam.adam_step(theta, m, v, g, t=t, lr=lr, beta1=B1, beta2=B2, eps=EPS, weight_decay=wd)
    _check(ref, th_g, m_g, v_g, w16, step_bound(ref, theta, m, g, t, lr, wd))


def test_twenty_five_steps_from_zero_state():
    n = 65536 + 3
    theta, _, _, _ = _state(n, 5)
    rng = np.random.Generator(np.random.Philox(key=6))
    th_g = _dev(theta)
    m_g = torch.zeros(n, device="cuda")
    v_g = torch.zeros(n, device="cuda")
    w16 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    ref = {"theta": theta.astype(np.float64), "m": np.zeros(n), "v": np.zeros(n)}
    lr = f32(1e-3)
    moved = np.zeros(n)
    for t in range(1, 26):
        g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
        q4.lora_adam_step(th_g, w16, m_g, v_g, _dev(g), step=t, lr=lr, beta1=B1, beta2=B2, eps=EPS)
        prev, m_prev = ref["theta"], ref["m"]
        ref = adam.adam_step(ref["theta"], ref["m"], ref["v"], g, t=t, lr=lr, beta1=B1, beta2=B2, eps=EPS)
        moved += step_bound(ref, prev, m_prev, g, t, lr)
    torch.cuda.synchronize()
    _check(ref, th_g, m_g, v_g, w16, moved, steps=25)


def test_adapter_shapes_in_place():
    # A (r x k) and B (d x r) of the 4096 x 11008 projection, r = 16, one step each
    for shape in ((16, 4096), (11008, 16)):
        n = shape[0] * shape[1]
        theta, m, v, g = _state(n, n)
        th_g, m_g, v_g, g_g = (_dev(x).view(shape) for x in (theta, m, v, g))
        w16 = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        q4.lora_adam_step(th_g, w16, m_g, v_g, g_g, step=3, lr=f32(1e-4), beta1=B1, beta2=B2, eps=EPS)
        torch.cuda.synchronize()
        ref = adam.adam_step(theta, m, v, g, t=3, lr=f32(1e-4), beta1=B1, beta2=B2, eps=EPS)
        _check(ref, th_g.view(-1), m_g.view(-1), v_g.view(-1), w16.view(-1), step_bound(ref, theta, m, g, 3, f32(1e-4)))


def test_rejects_bad_arguments():
    x = torch.zeros(8, device="cuda")
    w = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    for kw in ({"step": 0, "lr": 1e-3}, {"step": 1, "lr": 1e-3, "beta1": 1.0},
               {"step": 1, "lr": -1.0}):
        with pytest.raises(q4.QloraError) as e:
            q4.lora_adam_step(x, w, x.clone(), x.clone(), x.clone(), **kw)
        assert e.value.status == 1
