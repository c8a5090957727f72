"""Pins for the oracle's AdamW step: PyTorch's own AdamW in fp64 on the CPU over several steps, and the
closed forms of the first step (the update is lr * g / (|g| + eps)) and of a pure weight-decay step."""
import numpy as np
import pytest
import torch

from oracle.adamw import adamw_step
import synth


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_matches_torch_adamw_in_fp64(wd):
    n = 1000
    p0 = synth.normal_f32(n, 0.02, 1, 1).astype(np.float64)
    grads = [synth.normal_f32(n, 1e-3 * (k + 1), 1, 10 + k).astype(np.float64) for k in range(5)]
    tp = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([tp], lr=2e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.from_numpy(g.copy())
        opt.step()
        p, m, v = adamw_step(p, g, m, v, t, 2e-4, wd=wd)
        st = opt.state[tp]
        assert np.allclose(p, tp.detach().numpy(), rtol=0, atol=1e-15)
        # torch forms m by lerp (m + (1 - beta1)(g - m)): the same value up to fp64 rounding
        em, ev = st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()
        assert np.allclose(m, em, rtol=1e-12, atol=1e-15 * np.abs(em).max())
        assert np.allclose(v, ev, rtol=1e-12, atol=1e-15 * np.abs(ev).max())


def test_first_step_closed_form():
    """From zero moments the bias corrections cancel: m_hat = g, v_hat = g^2, so the step is
    lr * g / (|g| + eps), close to lr * sign(g)."""
    g = np.array([3e-3, -2e-5, 0.0, 1.0, -7.0])
    p, m, v = adamw_step(np.ones(5), g, np.zeros(5), np.zeros(5), 1, 1e-3, eps=1e-8)
    assert np.allclose(p, 1.0 - 1e-3 * g / (np.abs(g) + 1e-8), rtol=0, atol=1e-16)
    assert np.allclose(m, 0.1 * g) and np.allclose(v, 0.001 * g * g)


def test_weight_decay_alone_scales_the_parameter():
    p, m, v = adamw_step(np.array([2.0, -4.0]), np.zeros(2), np.zeros(2), np.zeros(2), 3, 0.01, wd=0.5)
    assert np.array_equal(p, np.array([2.0, -4.0]) * (1 - 0.01 * 0.5))
    assert np.all(m == 0) and np.all(v == 0)


def test_step_count_starts_at_one():
    with pytest.raises(ValueError):
        adamw_step(np.zeros(1), np.zeros(1), np.zeros(1), np.zeros(1), 0, 1e-3)
