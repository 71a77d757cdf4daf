"""bcjr_qat_step (self-reconstruction QAT step) against the oracle, and the
driver's descent property; every call goes through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from bcjr_sum_product_b200 import inputs as I
from bcjr_sum_product_b200 import lib, qat
from helpers import assert_grad, assert_soft

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("L,k,V,T", [(8, 2, 1, 0.3), (10, 2, 2, 0.1), (16, 2, 1, 0.05), (16, 2, 2, 0.05)])
def test_qat_step_matches_oracle(L, k, V, T):
    n_seq = 12 if L < 16 else 3
    target, c, _ = I.random_case(L, k, V, n_seq, 32 * V, seed=400 + L + V)
    noise = torch.randn(target.shape, generator=torch.Generator().manual_seed(9)) * 0.2
    w0 = target + noise
    lr_w, lr_c = 1e-2, 1e-3
    w = w0.to(DEV).contiguous()
    cd = c.to(DEV).contiguous()
    soft, loss, gw, gc = lib.qat_step(w, target.to(DEV), cd, L, k, V, T, lr_w, lr_c)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    ref = oracle.soft(w0, c, L, k, V, T)
    assert_soft(soft.cpu().numpy(), ref["soft"], c)
    d = ref["soft"] - target.numpy().astype(np.float64)
    loss_ref = (d ** 2).sum(axis=1)
    np.testing.assert_allclose(loss.cpu().numpy(), loss_ref, rtol=1e-4, atol=1e-5 * float(np.abs(c.numpy()).max()))
    rv = oracle.vjp(w0, c, L, k, V, T, torch.from_numpy(2.0 * d).float())
    assert_grad(gw.cpu().numpy(), rv["grad_w"], "grad_w")
    assert_grad(gc.cpu().numpy().reshape(rv["grad_c"].shape), rv["grad_c"], "grad_c")
    # in-place updates
    w_ref = w0.numpy().astype(np.float64) - lr_w * rv["grad_w"]
    c_ref = c.numpy().astype(np.float64) - lr_c * rv["grad_c"].reshape(c.shape)
    tol_w = lr_w * 1e-4 * float(np.abs(rv["grad_w"]).max()) + 1e-6 * float(np.abs(w_ref).max())
    tol_c = lr_c * 1e-4 * float(np.abs(rv["grad_c"]).max()) + 1e-6 * float(np.abs(c_ref).max())
    assert float(np.abs(w.cpu().numpy() - w_ref).max()) <= tol_w
    assert float(np.abs(cd.cpu().numpy() - c_ref).max()) <= tol_c


def test_qat_step_without_codebook_update_leaves_codebook():
    target, c, _ = I.random_case(8, 2, 1, 4, 16, seed=5)
    cd = c.to(DEV)
    before = cd.clone()
    lib.qat_step(target.to(DEV).clone(), target.to(DEV), cd, 8, 2, 1, 0.2, 1e-2, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(cd, before)


def test_descent_at_fixed_temperature():
    """Small steps of gradient descent lower the self-reconstruction loss."""
    target, c, _ = I.random_case(12, 2, 1, 32, 64, seed=6)
    t, cd = target.to(DEV), c.to(DEV)
    w = (target + 0.3 * torch.randn(target.shape, generator=torch.Generator().manual_seed(2))).to(DEV)
    losses = []
    for _ in range(4):
        _, loss, _, _ = lib.qat_step(w, t, cd, 12, 2, 1, 0.2, 2e-3)
        losses.append(float(loss.sum()))
    assert all(b < a for a, b in zip(losses, losses[1:])), losses


def test_driver_reports_drift_and_codes():
    target, c, _ = I.random_case(12, 2, 1, 16, 64, seed=8)
    out = qat.run(target.to(DEV), c.to(DEV), 12, 2, 1, 0.3, 0.01, 6, 1e-3)
    assert out["steps"] == 6 and len(out["loss"]) == 6
    assert 0.0 <= out["code_changed_fraction"] <= 1.0
    assert out["drift_budget"] >= out["max_drift"] - 1e-6
    # the PTQ code is the minimum-energy path of the target: no code has a lower hard MSE
    assert out["hard_mse_qat"] >= out["hard_mse_ptq"] - 1e-3 * out["hard_mse_ptq"]
