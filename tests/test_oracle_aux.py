"""Pins for the auxiliary oracle functions (no GPU)."""
import numpy as np
import pytest
import torch

from oracle import aux


def test_average_exact_on_dyadic_values():
    """Six checkpoints of small dyadic values: the average is exact."""
    thetas = [np.array([1.0, -2.0, 0.5, 3.0]) * (i + 1) for i in range(6)]
    assert np.array_equal(aux.checkpoint_average(thetas), np.array([1.0, -2.0, 0.5, 3.0]) * 3.5)


def test_average_of_identical_checkpoints_is_the_checkpoint():
    x = np.random.default_rng(0).standard_normal(1000)
    assert np.allclose(aux.checkpoint_average([x] * 6), x, rtol=0, atol=1e-15)


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_adamw_matches_the_library_routine(wd):
    """torch.optim.AdamW (decoupled weight decay, bias correction) on the CPU
    in float64, several steps."""
    rng = np.random.default_rng(1)
    p0 = rng.standard_normal(257)
    grads = [rng.standard_normal(257) * 10 ** (-k) for k in range(5)]
    tp = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=3e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros(257), np.zeros(257)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = aux.adamw_step(p, m, v, g, t, 3e-3, 0.9, 0.95, 1e-8, wd)
        assert np.allclose(p, tp.detach().numpy(), rtol=0, atol=1e-15)


def test_adamw_first_step_is_a_sign_step():
    """At t = 1 the bias-corrected ratio is g/(|g| + eps): a step of lr sign(g)."""
    g = np.array([3.0, -0.5, 1e-3])
    p, _, _ = aux.adamw_step(np.zeros(3), np.zeros(3), np.zeros(3), g, 1, 0.01, eps=0.0, weight_decay=0.0)
    assert np.allclose(p, -0.01 * np.sign(g), rtol=0, atol=1e-15)
