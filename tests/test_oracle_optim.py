"""Pins for the oracle's AdamW update: torch.optim.AdamW (the library routine
the textbook definition reduces to), the closed form of the first step, and
pure decoupled decay when the gradient is zero."""
import numpy as np
import torch

import oracle


def test_adamw_matches_library_over_several_steps():
    rng = np.random.default_rng(3)
    n = 1000
    theta0 = rng.standard_normal(n)
    grads = [rng.standard_normal(n) * (0.1 + k) for k in range(5)]
    hp = dict(lr=3e-3, betas=(0.8, 0.95), eps=1e-6, weight_decay=0.1)
    p = torch.nn.Parameter(torch.from_numpy(theta0.copy()))
    opt = torch.optim.AdamW([p], **hp)
    theta, m, v = theta0.copy(), np.zeros(n), np.zeros(n)
    for k, g in enumerate(grads):
        p.grad = torch.from_numpy(g.copy())
        opt.step()
        oracle.adamw_step(theta, g, m, v, k + 1, lr=hp["lr"], beta1=hp["betas"][0], beta2=hp["betas"][1],
                          eps=hp["eps"], weight_decay=hp["weight_decay"])
        np.testing.assert_allclose(theta, p.detach().numpy(), rtol=1e-12, atol=1e-14)
    st = opt.state[p]
    np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-12)
    np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-12)


def test_adamw_first_step_closed_form():
    """At t = 1, m_hat = g and v_hat = g^2 exactly, so the step is
    lr (wd theta + g / (|g| + eps)): a sign step of size lr for |g| >> eps."""
    rng = np.random.default_rng(4)
    theta0 = rng.standard_normal(64)
    g = rng.standard_normal(64)
    theta, m, v = theta0.copy(), np.zeros(64), np.zeros(64)
    lr, wd, eps = 0.01, 0.05, 1e-8
    oracle.adamw_step(theta, g, m, v, 1, lr=lr, beta1=0.9, beta2=0.99, eps=eps, weight_decay=wd)
    np.testing.assert_allclose(theta, theta0 - lr * (wd * theta0 + g / (np.abs(g) + eps)), rtol=1e-13)
    np.testing.assert_allclose(m, 0.1 * g, rtol=1e-14)
    np.testing.assert_allclose(v, 0.01 * g * g, rtol=1e-14)


def test_adamw_zero_gradient_is_pure_decoupled_decay():
    theta0 = np.linspace(-2, 2, 17)
    theta, m, v = theta0.copy(), np.zeros(17), np.zeros(17)
    oracle.adamw_step(theta, np.zeros(17), m, v, 3, lr=0.1, weight_decay=0.2)
    np.testing.assert_allclose(theta, theta0 * (1 - 0.1 * 0.2), rtol=1e-15)
