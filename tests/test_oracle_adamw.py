"""Pins of the oracle's AdamW step for the adapter (the page "QLoRA: put the large model
in memory, then change it with a small adapter", section 3: every batch ends with an
update of the LoRA parameters by a paged optimizer; section 2: its state lives in unified
memory). The oracle's fp32 step is checked against things that do not depend on it:
torch.optim.AdamW run in float64 (the same recurrence, decoupled weight decay), the closed
form of the first step from a zero state, and the zero-gradient case."""
import numpy as np
import pytest
import torch

import oracle


def _state(n, seed):
    rng = np.random.default_rng(seed)
    theta = rng.normal(0, 0.02, n).astype(np.float32)
    grads = [rng.normal(0, 1e-3, n).astype(np.float32) * np.float32(10.0 ** rng.uniform(-1, 1)) for _ in range(12)]
    return theta, grads


def _f32(x):
    return float(np.float32(x))      # hyperparameters as the fp32 step sees them


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_matches_torch_adamw_in_float64(wd):
    n, lr, b1, b2, eps, wd = 4099, _f32(2e-3), _f32(0.9), _f32(0.999), _f32(1e-8), _f32(wd)
    theta, grads = _state(n, 3)
    p = torch.nn.Parameter(torch.from_numpy(theta.astype(np.float64)))
    opt = torch.optim.AdamW([p], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    th, m, v = theta.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    for t, g in enumerate(grads, start=1):
        p.grad = torch.from_numpy(g.astype(np.float64))
        opt.step()
        oracle.adamw_step(th, g, m, v, t, lr, b1, b2, eps, wd)
        ref = p.detach().numpy()
        # fp32 rounding of a dozen steps: a few ulps of the parameter, far below a step (lr)
        assert np.max(np.abs(th.astype(np.float64) - ref)) < 16 * np.spacing(np.float32(np.max(np.abs(ref))))
        st = opt.state[p]
        assert np.allclose(m, st["exp_avg"].numpy(), rtol=0, atol=2e-6 * np.max(np.abs(m)))   # m can cancel
        assert np.allclose(v, st["exp_avg_sq"].numpy(), rtol=2e-6, atol=0)


def test_first_step_closed_form():
    # from m = v = 0 at t = 1 the bias-corrected moments are g and g^2, so the step is
    # lr (g / (|g| + eps) + wd theta)
    n, lr, eps, wd = 1000, 1e-3, 1e-8, 0.05
    theta, grads = _state(n, 5)
    g = grads[0]
    th, m, v = theta.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    bits = oracle.adamw_step(th, g, m, v, 1, lr, 0.9, 0.999, eps, wd, want_bf16=True)
    g64, t64 = g.astype(np.float64), theta.astype(np.float64)
    ref = t64 - lr * (g64 / (np.abs(g64) + eps) + wd * t64)
    assert np.max(np.abs(th - ref)) < 2e-9
    assert np.allclose(m, 0.1 * g64, rtol=1e-6) and np.allclose(v, 0.001 * g64 * g64, rtol=1e-5)
    # the adapter copy the layer multiplies with: bf16 round-to-nearest-even of theta
    assert np.array_equal(bits, torch.from_numpy(th).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_zero_gradient_only_decays():
    n, lr, wd = 512, 1e-2, 0.1
    theta, _ = _state(n, 7)
    th, m, v = theta.copy(), np.full(n, 0.5, np.float32), np.full(n, 2.0, np.float32)
    oracle.adamw_step(th, np.zeros(n, np.float32), m, v, 4, lr, 0.9, 0.999, 1e-8, wd)
    assert np.all(m == np.float32(0.9) * np.float32(0.5)) and np.all(v == np.float32(0.999) * np.float32(2.0))
    # the moment-driven part still moves theta (m > 0); with wd alone the change is lr wd theta
    th2, m2, v2 = theta.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    oracle.adamw_step(th2, np.zeros(n, np.float32), m2, v2, 1, lr, 0.9, 0.999, 1e-8, wd)
    ref = theta.astype(np.float64) - np.float32(lr) * np.float64(np.float32(np.float32(wd) * theta))
    assert np.max(np.abs(th2 - ref) / np.spacing(np.abs(th2))) <= 1.0


def test_bias_corrections():
    ib1, ib2 = oracle.adamw_bias_corrections(0.9, 0.999, 1)
    b1, b2 = np.float64(np.float32(0.9)), np.float64(np.float32(0.999))
    assert ib1 == np.float32(1 / (1 - b1)) and ib2 == np.float32(1 / (1 - b2))
    ib1, ib2 = oracle.adamw_bias_corrections(0.9, 0.999, 1000)
    assert ib1 == np.float32(1 / (1 - b1 ** 1000)) and abs(ib2 - 1 / (1 - b2 ** 1000)) <= np.spacing(np.float32(ib2))
