"""The oracle's AdamW against torch.optim.AdamW (binary64), a library routine.

Model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct", section
"Calibration": AdamW, betas 0.9/0.999, weight decay 0, constant learning rate
5e-3 for m and 1e-3 for q.  eps is not given: 1e-8 (the usual default).
"""
import numpy as np
import pytest
import torch

import oracle

F = np.float32


@pytest.mark.parametrize("lr,wd", [(5e-3, 0.0), (1e-3, 0.0), (1e-3, 0.05)])
def test_adamw_against_torch(lr, wd):
    rng = np.random.default_rng(17)
    n = 4096
    p = rng.normal(6.0, 2.0, n).astype(F)
    v1 = np.zeros(n, F); v2 = np.zeros(n, F)
    tp = torch.tensor(p.astype(np.float64), requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=lr, betas=(0.9, 0.999), eps=1e-8, weight_decay=wd, foreach=False)
    for t in range(1, 6):
        g = (rng.normal(0, 1e-4, n) * rng.choice([1e-4, 1.0, 100.0], n)).astype(F)
        oracle.adamw(p, g, v1, v2, lr, t, weight_decay=wd)
        tp.grad = torch.tensor(g.astype(np.float64))
        opt.step()
        st = opt.state[tp]
        if t in (1, 2, 5):
            np.testing.assert_allclose(p, tp.detach().numpy(), rtol=1e-6, atol=1e-9)
            # the oracle keeps its moments in binary32 between steps (torch here in binary64):
            # near-cancelling sums are compared on the scale of the whole vector
            ea, eas = st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()
            np.testing.assert_allclose(v1, ea, rtol=1e-6, atol=1e-6 * np.abs(ea).max())
            np.testing.assert_allclose(v2, eas, rtol=1e-6, atol=1e-6 * np.abs(eas).max())


def test_first_step_is_sign_step():
    n = 64
    p = np.ones(n, F)
    g = np.where(np.arange(n) % 2 == 0, 1e-3, -2e-2).astype(F)
    v1 = np.zeros(n, F); v2 = np.zeros(n, F)
    oracle.adamw(p, g, v1, v2, 5e-3, 1)
    # step 1: v1/(1-b1) = g and sqrt(v2/(1-b2)) = |g|, so the update is lr*g/(|g|+eps)
    want = 1.0 - 5e-3 * g / (np.abs(g) + 1e-8)
    np.testing.assert_allclose(p, want.astype(F), rtol=0, atol=2e-7)
    np.testing.assert_allclose(v1, 0.1 * g, rtol=1e-6)
    np.testing.assert_allclose(v2, 0.001 * g.astype(np.float64) ** 2, rtol=1e-6)


def test_zero_gradient_keeps_parameter():
    p = np.full(8, 6.0, F); v1 = np.zeros(8, F); v2 = np.zeros(8, F)
    oracle.adamw(p, np.zeros(8, F), v1, v2, 1e-3, 1)
    assert np.all(p == 6.0) and not v1.any() and not v2.any()


def test_rejects_bad_hyperparameters():
    p = np.zeros(4, F); z = np.zeros(4, F)
    with pytest.raises(oracle.OracleError):
        oracle.adamw(p, z, z.copy(), z.copy(), 1e-3, 0)
    with pytest.raises(oracle.OracleError):
        oracle.adamw(p, z, z.copy(), z.copy(), -1e-3, 1)
    with pytest.raises(oracle.OracleError):
        oracle.adamw(p, z, z.copy(), z.copy(), 1e-3, 1, beta1=1.0)
