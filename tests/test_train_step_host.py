"""Host-side checks of the training-step module (no GPU).

The group-LASSO penalty of the dense baseline is the sum of the m x m blocks' Frobenius norms
(page "kronecker-layer-benchmark", section "The baselines"). It is pinned on a weight whose
block norms are known by construction. The Kronecker MLP refuses CPU tensors: the library has
no CPU path.
"""
import math

import pytest
import torch

from kronecker_factored_structured_b200.train_step import DenseMLP, KronMLP


def test_group_lasso_is_sum_of_block_frobenius_norms():
    m = 4
    model = DenseMLP(d=8, classes=2, block=m, group_lasso=True, device="cpu")
    with torch.no_grad():
        for lin, vals in ((model.l1, (3.0, 0.0, 1.0, 2.0)), (model.l2, (0.5, 0.5, 0.0, 4.0))):
            w = torch.zeros(8, 8)
            # block (r, c) filled with a constant v: Frobenius norm = |v| * m
            for (r, c), v in zip(((0, 0), (0, 1), (1, 0), (1, 1)), vals):
                w[r * m:(r + 1) * m, c * m:(c + 1) * m] = v
            lin.weight.copy_(w)
    expect = m * (3.0 + 0.0 + 1.0 + 2.0) + m * (0.5 + 0.5 + 0.0 + 4.0)
    # an all-zero block contributes sqrt(1e-12) (the page's guard against a zero norm)
    expect += 2 * math.sqrt(1e-12)
    assert abs(float(model.penalty().detach()) - expect) < 1e-5


def test_dense_without_group_lasso_has_no_penalty():
    assert DenseMLP(d=8, classes=2, block=4, group_lasso=False, device="cpu").penalty() is None


def test_kron_mlp_refuses_cpu_tensors():
    model = KronMLP(d=64, classes=10, block=8, rank=2, path="f32", device="cpu")
    assert model.l1.S.shape == (8, 8) and model.l1.A.shape == (2, 8, 8)
    # the l1 penalty on both layers' S (all ones at initialisation)
    assert float(model.penalty().detach()) == pytest.approx(2 * 64)
    with pytest.raises((ValueError, RuntimeError)):
        model(torch.randn(4, 64))


def test_kron_mlp_fused_penalty_is_a_value_only():
    """With the penalty's gradient fused into the layers' backward, penalty() carries no
    gradient of its own (else S would get lam * sign(S) twice), and the layers hold lam."""
    model = KronMLP(d=64, classes=10, block=8, rank=2, path="f32", device="cpu", fused_l1=0.25)
    pen = model.penalty()
    assert not pen.requires_grad and float(pen) == pytest.approx(2 * 64)
    assert model.l1.l1 == 0.25 and model.l2.l1 == 0.25
    assert KronMLP(d=64, classes=10, block=8, rank=2, path="f32", device="cpu").l1.l1 == 0.0


def test_time_model_refuses_mismatched_penalty_weight():
    from kronecker_factored_structured_b200.train_step import time_model
    model = KronMLP(d=64, classes=10, block=8, rank=2, path="f32", device="cpu", fused_l1=0.25)
    with pytest.raises(ValueError):
        time_model(model, 4, 64, 10, 0.5, warmup=0, steps=1, dtype=torch.float32)
