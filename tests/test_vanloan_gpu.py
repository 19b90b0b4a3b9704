"""GPU parity of the Van Loan rank-r Kronecker fit (kron_vanloan_fit, through the C ABI)
against the fp64 oracle (page "LLM Compression via Kronecker Product Decomposition",
sections "Van Loan Rearrangement (1993)", "Rank-K" and "Adaptive Normalization").

The factors of one term are fixed only up to a common sign (and equal singular values mix
terms), so the comparison is on what is unique: the fitted sum of Kronecker products, the
singular values and alpha."""
import numpy as np
import pytest
import torch

import oracle
from kronecker_factored_structured_b200 import native

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _kron_sum(A, B):
    A, B = np.asarray(A, np.float64), np.asarray(B, np.float64)
    return oracle.weight(np.ones(A.shape[1:]), A, B)


def _low_rank_w(rng, p, q, m1, m2, r, noise=0.0):
    C = rng.standard_normal((r, p, q)) * (2.0 ** -np.arange(r))[:, None, None]
    B = rng.standard_normal((r, m1, m2))
    W = sum(np.kron(C[i], B[i]) for i in range(r))
    if noise:
        W = W + noise * np.abs(W).max() * rng.standard_normal(W.shape)
    return W.astype(np.float32).astype(np.float64)


def _fit(W, shape, r, **kw):
    p, q, m1, m2 = shape
    f = native.vanloan_fit(torch.from_numpy(W.astype(np.float32)).to(DEV), p, q, m1, m2, r, **kw)
    torch.cuda.synchronize()
    return {k: v.double().cpu().numpy() for k, v in f.items()}


@pytest.mark.parametrize("shape,r", [((32, 32, 32, 32), 4), ((24, 48, 32, 64), 4),
                                     ((48, 24, 64, 32), 1), ((64, 64, 64, 64), 8),
                                     ((5, 3, 4, 6), 2)],
                         ids=["tutorial", "gpt2_c_fc", "gpt2_c_proj", "stress", "odd"])
def test_exact_kronecker_rank_is_recovered(shape, r):
    """W = sum of r Kronecker products (fp32): the GPU fit reproduces it, alpha = 1, and its
    singular values match the oracle's (those past r vanish)."""
    rng = np.random.default_rng(sum(shape) + r)
    p, q, m1, m2 = shape
    W = _low_rank_w(rng, p, q, m1, m2, r)
    g = _fit(W, shape, r)
    ref = oracle.vanloan_fit(W, p, q, m1, m2, r)
    scale = np.abs(W).max()
    assert np.abs(_kron_sum(g["A"], g["B"]) - W).max() <= 1e-5 * scale
    assert abs(g["alpha"][0] - ref["alpha"]) <= 1e-5
    k = g["sigma"].shape[0]
    assert np.abs(g["sigma"][:r] - ref["sigma"][:r]).max() <= 1e-5 * ref["sigma"][0]
    assert np.all(g["sigma"][r:k] <= 1e-5 * ref["sigma"][0])


@pytest.mark.parametrize("normalize", [False, True])
def test_noisy_low_rank_matches_oracle_fit(normalize):
    """Kronecker rank 4 plus 1e-3 noise: the rank-4 fit (unique: a wide gap to sigma_5) and
    alpha match the oracle's exact truncated SVD."""
    rng = np.random.default_rng(17)
    shape, r = (32, 32, 32, 32), 4
    W = _low_rank_w(rng, *shape, r, noise=1e-3)
    g = _fit(W, shape, r, power_iters=3, normalize=normalize)
    ref = oracle.vanloan_fit(W, *shape, r, normalize=normalize)
    got, want = _kron_sum(g["A"], g["B"]), _kron_sum(ref["A"], ref["B"])
    assert np.abs(got - want).max() <= 1e-4 * np.abs(want).max()
    assert abs(g["alpha"][0] - ref["alpha"]) <= 1e-5 * ref["alpha"]
    if normalize:
        assert abs(np.linalg.norm(got) - np.linalg.norm(W)) <= 1e-5 * np.linalg.norm(W)


def test_fit_is_deterministic():
    rng = np.random.default_rng(5)
    W = torch.from_numpy(_low_rank_w(rng, 24, 48, 32, 64, 4, noise=1e-2).astype(np.float32)).to(DEV)
    runs = [native.vanloan_fit(W, 24, 48, 32, 64, 4) for _ in range(2)]
    torch.cuda.synchronize()
    for k in runs[0]:
        assert torch.equal(runs[0][k], runs[1][k]), k


def test_fitted_factors_drive_the_layer():
    """The fitted (S = 1, A, B) as layer factors: the layer's forward (TF32 path) gives x W
    for the dense W the factors were fitted to (exact Kronecker rank)."""
    import kronecker_factored_structured_b200 as kfs
    rng = np.random.default_rng(9)
    W = _low_rank_w(rng, 32, 32, 32, 32, 4)
    f = native.vanloan_fit(torch.from_numpy(W.astype(np.float32)).to(DEV), 32, 32, 32, 32, 4)
    x = torch.randn(300, 1024, device=DEV)
    y = kfs.forward(x, f["S"], f["A"], f["B"], None, dtype="tf32")
    torch.cuda.synchronize()
    ref = x.double().cpu().numpy() @ W
    assert np.abs(y.double().cpu().numpy() - ref).max() <= 5e-3 * np.abs(ref).max()
