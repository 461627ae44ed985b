"""Pins of the oracle's LUT update (AdamW, SGD, gradient averaging).

The pages train the LUT values but name no optimizer; the oracle writes out
plain AdamW (decoupled weight decay) and SGD.  They are pinned against the
library optimizers of PyTorch (float64 on the CPU) over several steps with
changing gradients, against closed forms of special cases, and the averaging
variant (SpaLLM section 2.1: the gradient of a shared value averaged over the
virtual parameters that share it) against the bin counts.
"""
import numpy as np
import pytest
import torch

import oracle
from compressive_fine_tuning_b200 import synth


def _grads(rng, shape, steps):
    return [rng.standard_normal(shape) * 10.0 ** rng.uniform(-4, 0) for _ in range(steps)]


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_adamw_matches_torch_over_several_steps(wd):
    rng = synth.rng_for(41000)
    shape = (2, 5, 3, 16)
    p0 = rng.standard_normal(shape) * 0.02
    grads = _grads(rng, shape, 5)
    lr, b1, b2, eps = 1e-3, 0.9, 0.98, 1e-8
    ref = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([ref], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros(shape), np.zeros(shape)
    for t, g in enumerate(grads, start=1):
        ref.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = oracle.adamw_step(p, m, v, g, t, lr, b1, b2, eps, wd)
        np.testing.assert_allclose(p, ref.detach().numpy(), rtol=1e-12, atol=1e-15)


def test_sgd_matches_torch():
    rng = synth.rng_for(41001)
    shape = (1, 4, 2, 8)
    p0 = rng.standard_normal(shape)
    ref = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.SGD([ref], lr=0.05)
    p = p0.copy()
    for g in _grads(rng, shape, 3):
        ref.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p = oracle.sgd_step(p, g, 0.05)
        np.testing.assert_allclose(p, ref.detach().numpy(), rtol=1e-14, atol=0)


def test_adamw_closed_forms():
    rng = synth.rng_for(41002)
    shape = (1, 3, 2, 4)
    p0 = rng.standard_normal(shape)
    # a constant gradient: the bias-corrected moments are exactly g and g^2
    g = rng.standard_normal(shape)
    p, m, v = p0.copy(), np.zeros(shape), np.zeros(shape)
    for t in range(1, 6):
        p, m, v = oracle.adamw_step(p, m, v, g, t, 0.01, 0.9, 0.999, 1e-8, 0.0)
    np.testing.assert_allclose(p, p0 - 5 * 0.01 * g / (np.abs(g) + 1e-8), rtol=1e-12)
    # a zero gradient with weight decay: pure multiplicative decay, moments stay zero
    p, m, v = oracle.adamw_step(p0, np.zeros(shape), np.zeros(shape), np.zeros(shape), 1, 0.1, 0.9, 0.999,
                                1e-8, 0.5)
    np.testing.assert_array_equal(m, 0.0)
    np.testing.assert_array_equal(v, 0.0)
    np.testing.assert_allclose(p, p0 * (1 - 0.1 * 0.5), rtol=1e-15)


def test_averaging_divides_by_bin_counts():
    c = synth.layer_case(41003, n=6, d=64, bits=2, gpr=2, T=3)
    counts = oracle.bin_counts(c.idx, c.gpr, c.k)
    g = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k)
    avg = oracle.averaged_gradient(g, counts)
    # the mean over the virtual parameters of each bin, computed column by column
    gs = c.d // c.gpr
    G = c.dy.T @ c.x
    for i in range(c.n):
        for gi in range(c.gpr):
            for cc in range(c.k):
                cols = [j for j in range(gi * gs, (gi + 1) * gs) if c.idx[i, j] == cc]
                want = np.mean(G[i, cols]) if cols else 0.0
                assert abs(avg[i, gi, cc] - want) <= 1e-12 * (abs(want) + 1e-300)
    # without counts the gradient is the sum (unchanged)
    np.testing.assert_array_equal(oracle.averaged_gradient(g, None), g)
