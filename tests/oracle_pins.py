"""Pins for the fp64 oracle: checks against facts that do not come from the oracle.

Each ``pin_*`` function takes an oracle object (``oracle.Oracle``) and raises
AssertionError when the oracle disagrees with something the pages or plain
mathematics fix.  ``test_oracle_pins.py`` runs them on the real oracle and
``test_oracle_mutations.py`` runs them on deliberately broken copies of it, to
show that a dropped term, a swapped index or a transposed operand is caught.

Sources of truth used here (none of them is the oracle's own loop):
  * numpy's ``np.kron`` and ``@`` (library routines),
  * pure-Python scalar sums on tiny inputs (brute force),
  * Kronecker algebra: mixed product, transpose, block structure, rank one,
  * the Van Loan rearrangement of a sum of r Kronecker products has rank <= r
    (page "LLM Compression via Kronecker Product Decomposition", section
    "Van Loan Rearrangement (1993)"),
  * special shapes that reduce to a plain GEMM,
  * central finite differences of L = <G, y> (exact here: L is affine in each
    single parameter coordinate), and Euler's identity for functions that are
    linear in one argument,
  * for the l1 penalty lam * sum|S| on S: central differences away from the kink at
    0, and torch's autograd of abs() for the value taken at S = 0,
  * for the Kronecker-sparse factor (page "Fast Inference with Kronecker-Sparse
    Matrices", abstract: supports that are Kronecker products of identity and all-ones
    blocks): its support against numpy's kron of eye and ones, scipy's block_diag and
    hadamard, numpy's kron for tied values, and the two-factor Kronecker layer as a
    product of two KS factors.
"""
from __future__ import annotations

import itertools

import numpy as np


def _rand_layer(rng, p, q, m1, m2, r, s_zero=0.25, N=3):
    S = np.ones((p, q))
    S[rng.random((p, q)) < s_zero] = 0.0
    A = rng.standard_normal((r, p, q))
    B = rng.standard_normal((r, m1, m2))
    bias = rng.standard_normal(q * m2)
    x = rng.standard_normal((N, p * m1))
    G = rng.standard_normal((N, q * m2))
    return S, A, B, bias, x, G


def pin_weight_is_sum_of_numpy_krons(orc):
    """W equals sum_i np.kron(S*A_i, B_i) (page "kronecker-layer-benchmark", KronLinear.weight)."""
    rng = np.random.default_rng(101)
    for (p, q, m1, m2, r) in [(2, 3, 4, 5, 2), (3, 2, 1, 3, 3), (4, 4, 2, 2, 1), (1, 2, 3, 1, 2)]:
        S, A, B, *_ = _rand_layer(rng, p, q, m1, m2, r)
        ref = sum(np.kron(S * A[i], B[i]) for i in range(r))
        W = orc.weight(S, A, B)
        assert W.shape == (p * m1, q * m2)
        assert np.allclose(W, ref, rtol=0, atol=1e-13), (p, q, m1, m2, r)


def pin_forward_brute_force(orc):
    """Tiny case: y[n, c*m2+k] = bias + sum_{i,a,j} x[n, a*m1+j] S[a,c] A_i[a,c] B_i[j,k]."""
    rng = np.random.default_rng(102)
    p, q, m1, m2, r, N = 2, 3, 2, 3, 2, 2
    S, A, B, bias, x, _ = _rand_layer(rng, p, q, m1, m2, r, N=N)
    y = orc.forward(x, S, A, B, bias)
    for n, c, k in itertools.product(range(N), range(q), range(m2)):
        s = bias[c * m2 + k]
        for i, a, j in itertools.product(range(r), range(p), range(m1)):
            s += x[n, a * m1 + j] * S[a, c] * A[i, a, c] * B[i, j, k]
        assert abs(y[n, c * m2 + k] - s) < 1e-12, (n, c, k)


def pin_forward_vec_trick(orc):
    """The row-wise vec trick Y_n = sum_i C_i^T X_n B_i gives the same y
    (page "kronecker-layer-benchmark", section "2. The vec trick": all variants agree)."""
    rng = np.random.default_rng(103)
    for (p, q, m1, m2, r, N) in [(8, 8, 8, 8, 2, 16), (3, 5, 4, 2, 3, 7), (6, 4, 2, 5, 1, 5)]:
        S, A, B, bias, x, _ = _rand_layer(rng, p, q, m1, m2, r, N=N)
        X = x.reshape(N, p, m1)
        Y = np.zeros((N, q, m2))
        for i in range(r):
            Y += np.swapaxes(S * A[i], 0, 1)[None] @ (X @ B[i])
        ref = Y.reshape(N, q * m2) + bias
        assert np.allclose(orc.forward(x, S, A, B, bias), ref, rtol=0, atol=1e-12)


def pin_forward_is_gemm_with_numpy_weight(orc):
    """y = x @ W + bias with numpy's matmul on the numpy-built W (larger, ragged shapes)."""
    rng = np.random.default_rng(104)
    p, q, m1, m2, r, N = 5, 3, 3, 4, 3, 37
    S, A, B, bias, x, _ = _rand_layer(rng, p, q, m1, m2, r, N=N)
    W = sum(np.kron(S * A[i], B[i]) for i in range(r))
    assert np.allclose(orc.forward(x, S, A, B, bias), x @ W + bias, rtol=0, atol=1e-11)
    assert np.allclose(orc.forward(x, S, A, B, None), x @ W, rtol=0, atol=1e-11)


def pin_mixed_product(orc):
    """(C kron B)(C' kron B') = (C C') kron (B B') (r = 1, S = 1)."""
    rng = np.random.default_rng(105)
    p, q, s, m1, m2, m3 = 3, 4, 2, 2, 3, 5
    C1, C2 = rng.standard_normal((p, q)), rng.standard_normal((q, s))
    B1, B2 = rng.standard_normal((m1, m2)), rng.standard_normal((m2, m3))
    W1 = orc.weight(np.ones((p, q)), C1[None], B1[None])
    W2 = orc.weight(np.ones((q, s)), C2[None], B2[None])
    W12 = orc.weight(np.ones((p, s)), (C1 @ C2)[None], (B1 @ B2)[None])
    assert np.allclose(W1 @ W2, W12, rtol=0, atol=1e-12)


def pin_transpose(orc):
    """(sum_i C_i kron B_i)^T = sum_i C_i^T kron B_i^T; also maps the out x in convention."""
    rng = np.random.default_rng(106)
    p, q, m1, m2, r = 3, 5, 2, 4, 2
    S, A, B, *_ = _rand_layer(rng, p, q, m1, m2, r)
    W = orc.weight(S, A, B)
    Wt = orc.weight(S.T, np.swapaxes(A, 1, 2), np.swapaxes(B, 1, 2))
    assert np.allclose(W.T, Wt, rtol=0, atol=1e-13)


def pin_block_structure(orc):
    """S[a,c] = 0 makes the m1 x m2 block (a, c) of W exactly zero, other blocks are not
    (page "kronecker-layer-benchmark", introduction: sparse S gives a block-sparse W)."""
    rng = np.random.default_rng(107)
    p, q, m1, m2, r = 6, 5, 3, 2, 3
    S, A, B, *_ = _rand_layer(rng, p, q, m1, m2, r, s_zero=0.4)
    W = orc.weight(S, A, B)
    for a, c in itertools.product(range(p), range(q)):
        blk = W[a * m1:(a + 1) * m1, c * m2:(c + 1) * m2]
        if S[a, c] == 0:
            assert np.all(blk == 0.0), (a, c)
        else:
            assert np.abs(blk).max() > 1e-6, (a, c)


def pin_rank_one(orc):
    """r = 1, S = ones: W = A kron B exactly."""
    rng = np.random.default_rng(108)
    A = rng.standard_normal((1, 4, 3))
    B = rng.standard_normal((1, 2, 5))
    W = orc.weight(np.ones((4, 3)), A, B)
    assert np.array_equal(W, np.kron(A[0], B[0]))


def pin_van_loan_rank(orc):
    """The rearranged W~ (rows (a,c), columns (j,k)) equals sum_i vec(C_i) vec(B_i)^T and
    has exactly r non-zero singular values (page "LLM Compression via Kronecker Product
    Decomposition", section "Core Algorithm -- Van Loan Kronecker Decomposition")."""
    rng = np.random.default_rng(109)
    p, q, m1, m2, r = 4, 3, 3, 4, 3
    S, A, B, *_ = _rand_layer(rng, p, q, m1, m2, r, s_zero=0.0)
    W = orc.weight(S, A, B)
    Wt = W.reshape(p, m1, q, m2).transpose(0, 2, 1, 3).reshape(p * q, m1 * m2)
    outer = sum(np.outer((S * A[i]).ravel(), B[i].ravel()) for i in range(r))
    assert np.allclose(Wt, outer, rtol=0, atol=1e-12)
    sv = np.linalg.svd(Wt, compute_uv=False)
    assert sv[r - 1] > 1e-6 * sv[0]
    assert np.all(sv[r:] < 1e-10 * sv[0])


def pin_special_shapes(orc):
    """Shapes that reduce to a plain GEMM: m1 = m2 = 1 (W = S (.) sum_i b_i A_i, b_i the
    1 x 1 block B_i),
    p = q = 1 (W = S * sum_i A_i B_i) and C = I, r = 1 (W = blockdiag(B, ..., B))."""
    rng = np.random.default_rng(110)
    N = 6
    # m1 = m2 = 1
    p, q, r = 5, 4, 3
    S, A, B, bias, x, _ = _rand_layer(rng, p, q, 1, 1, r, N=N)
    assert np.allclose(orc.forward(x, S, A, B, bias),
                       x @ (S * (B[:, 0, 0, None, None] * A).sum(0)) + bias, atol=1e-12)
    # p = q = 1
    m1, m2, r = 3, 4, 2
    S, A, B, bias, x, _ = _rand_layer(rng, 1, 1, m1, m2, r, s_zero=0.0, N=N)
    W = S[0, 0] * sum(A[i, 0, 0] * B[i] for i in range(r))
    assert np.allclose(orc.forward(x, S, A, B, bias), x @ W + bias, atol=1e-12)
    # C = I, r = 1: block-diagonal copy of B
    p, m1, m2 = 4, 3, 2
    B = rng.standard_normal((1, m1, m2))
    x = rng.standard_normal((N, p * m1))
    y = orc.forward(x, np.ones((p, p)), np.eye(p)[None], B, None)
    for c in range(p):
        assert np.allclose(y[:, c * m2:(c + 1) * m2], x[:, c * m1:(c + 1) * m1] @ B[0], atol=1e-12)


def _loss(orc, x, S, A, B, bias, G):
    return float(np.sum(G * orc.forward(x, S, A, B, bias)))


def pin_finite_differences(orc):
    """Central differences of L = <G, y>.  L is affine in every single coordinate of
    x, S, A, B and bias, so the difference quotient is exact up to rounding."""
    rng = np.random.default_rng(111)
    p, q, m1, m2, r, N = 3, 2, 2, 3, 2, 4
    S, A, B, bias, x, G = _rand_layer(rng, p, q, m1, m2, r, N=N)
    g = orc.backward(x, S, A, B, G)
    h = 0.5
    for name, arr in (("dX", x), ("dS", S), ("dA", A), ("dB", B), ("dbias", bias)):
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            lp = _loss(orc, x, S, A, B, bias, G)
            arr[idx] = old - h
            lm = _loss(orc, x, S, A, B, bias, G)
            arr[idx] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[name][idx]) < 1e-9 * (1 + abs(fd)), (name, idx, fd, g[name][idx])


def pin_linearity_identities(orc):
    """y - bias is linear in each of x, S, A and B, so by Euler's identity
    <dX, x> = <dS, S> = <dA, A> = <dB, B> = <G, y - bias>, and <dbias, 1> = sum G."""
    rng = np.random.default_rng(112)
    p, q, m1, m2, r, N = 6, 5, 4, 3, 3, 29
    S, A, B, bias, x, G = _rand_layer(rng, p, q, m1, m2, r, N=N)
    S = S * rng.standard_normal((p, q))          # a general (not 0/1) S
    g = orc.backward(x, S, A, B, G)
    ref = float(np.sum(G * orc.forward(x, S, A, B, None)))
    tol = 1e-10 * (1 + abs(ref))
    assert abs(np.sum(g["dX"] * x) - ref) < tol
    assert abs(np.sum(g["dS"] * S) - ref) < tol
    assert abs(np.sum(g["dA"] * A) - ref) < tol
    assert abs(np.sum(g["dB"] * B) - ref) < tol
    assert np.allclose(g["dbias"], G.sum(0), atol=1e-12)


def pin_backward_numpy_chain_rule(orc):
    """dX = G W^T and dW = x^T G with numpy on the numpy-built W; dC, dB by contracting dW
    with the other factor; dA = dC (.) S and dS = sum_i dC_i (.) A_i."""
    rng = np.random.default_rng(113)
    p, q, m1, m2, r, N = 4, 3, 2, 5, 2, 11
    S, A, B, bias, x, G = _rand_layer(rng, p, q, m1, m2, r, N=N)
    W = sum(np.kron(S * A[i], B[i]) for i in range(r))
    dW = (x.T @ G).reshape(p, m1, q, m2)
    dC = np.einsum("ajck,ijk->iac", dW, B)
    dB = np.einsum("ajck,iac->ijk", dW, S[None] * A)
    g = orc.backward(x, S, A, B, G)
    assert np.allclose(g["dX"], G @ W.T, atol=1e-11)
    assert np.allclose(g["dA"], dC * S[None], atol=1e-11)
    assert np.allclose(g["dS"], (dC * A).sum(0), atol=1e-11)
    assert np.allclose(g["dB"], dB, atol=1e-11)
    assert np.allclose(g["dbias"], G.sum(0), atol=1e-12)


def pin_zero_s_gradient(orc):
    """Where S[a,c] = 0, dA is zero but dS is in general not (sum_i dC_i (.) A_i)."""
    rng = np.random.default_rng(114)
    p, q, m1, m2, r, N = 4, 4, 2, 2, 2, 9
    S, A, B, bias, x, G = _rand_layer(rng, p, q, m1, m2, r, s_zero=0.5, N=N)
    assert (S == 0).any()
    g = orc.backward(x, S, A, B, G)
    z = S == 0
    assert np.all(g["dA"][:, z] == 0.0)
    assert np.abs(g["dS"][z]).min() > 1e-8


def pin_l1_grad_finite_differences(orc):
    """Gradient of the penalty lam * sum|S| (page "kronecker-layer-benchmark", introduction:
    an l1 term on S).  Away from 0, |.| is linear on [v - h, v + h] when h < |v|, so the
    central difference of the penalty is exact; the entries that are 0 get 0, the
    subgradient torch's autograd returns for abs() there (checked with torch itself)."""
    import torch
    rng = np.random.default_rng(115)
    p, q, lam = 7, 5, 0.37
    S = rng.standard_normal((p, q))
    S[rng.random((p, q)) < 0.3] = 0.0
    S[0, 0], S[0, 1] = 0.0, -2.5
    g = orc.l1_grad(S, lam)
    pen = lambda M: lam * float(np.abs(M).sum())
    for idx in np.ndindex(S.shape):
        v = S[idx]
        if v == 0.0:
            continue
        h = 0.5 * abs(v)
        Sp, Sm = S.copy(), S.copy()
        Sp[idx], Sm[idx] = v + h, v - h
        fd = (pen(Sp) - pen(Sm)) / (2 * h)
        assert abs(fd - g[idx]) < 1e-12 * (1 + abs(fd)), (idx, fd, g[idx])
    St = torch.tensor(S, dtype=torch.float64, requires_grad=True)
    (lam * St.abs().sum()).backward()
    z = S == 0.0
    assert z.sum() >= 1
    assert np.array_equal(g[z], St.grad.numpy()[z])
    assert np.all(g[z] == 0.0)
    assert np.array_equal(orc.l1_grad(S, 0.0), np.zeros_like(S))


# ---------------------------------------------------------------- Van Loan rank-r fit
# (page "LLM Compression via Kronecker Product Decomposition", sections "Van Loan
# Rearrangement (1993)" and "Adaptive Normalization")

def pin_vanloan_rearrangement_of_krons(orc):
    """R(sum_i kron(C_i, B_i)) = sum_i vec(C_i) vec(B_i)^T, with W built by numpy's kron and
    the outer products by numpy (the identity the fit rests on), for rectangular blocks; and
    R is the page's block permutation (numpy reshape / transpose route)."""
    rng = np.random.default_rng(211)
    for (p, q, m1, m2, r) in [(3, 4, 2, 5, 2), (2, 5, 4, 3, 3), (1, 3, 3, 1, 1)]:
        C = rng.standard_normal((r, p, q))
        B = rng.standard_normal((r, m1, m2))
        W = sum(np.kron(C[i], B[i]) for i in range(r))
        Wt = orc.vanloan_rearrange(W, p, q, m1, m2)
        outer = sum(np.outer(C[i].ravel(), B[i].ravel()) for i in range(r))
        assert np.allclose(Wt, outer, rtol=0, atol=1e-12), (p, q, m1, m2)
        perm = W.reshape(p, m1, q, m2).transpose(0, 2, 1, 3).reshape(p * q, m1 * m2)
        assert np.array_equal(Wt, perm)


def pin_vanloan_fit_recovers_exact_rank(orc):
    """W of Kronecker rank r: the rank-r fit reproduces W (to rounding), alpha = 1 and the
    singular values past r vanish; the fit of a smaller rank does not reproduce it."""
    rng = np.random.default_rng(223)
    p, q, m1, m2, r = 4, 3, 5, 2, 3
    C = rng.standard_normal((r, p, q))
    B = rng.standard_normal((r, m1, m2))
    W = sum(np.kron(C[i], B[i]) for i in range(r))
    f = orc.vanloan_fit(W, p, q, m1, m2, r)
    Wr = sum(np.kron(f["A"][i], f["B"][i]) for i in range(r))
    assert np.abs(Wr - W).max() <= 1e-12 * np.abs(W).max()
    assert abs(f["alpha"] - 1.0) <= 1e-12
    assert np.all(f["sigma"][r:] <= 1e-12 * f["sigma"][0]) and f["sigma"][r - 1] > 1e-6
    f1 = orc.vanloan_fit(W, p, q, m1, m2, r - 1, normalize=False)
    W1 = sum(np.kron(f1["A"][i], f1["B"][i]) for i in range(r - 1))
    assert np.abs(W1 - W).max() > 1e-3 * np.abs(W).max()


def pin_vanloan_rank_one_closed_form(orc):
    """W = kron(A, B): R(W) = vec(A) vec(B)^T has the single singular value |A|_F |B|_F, and
    the rank-1 fit gives back kron(A, B) exactly."""
    rng = np.random.default_rng(227)
    A = rng.standard_normal((3, 6))
    B = rng.standard_normal((4, 2))
    W = np.kron(A, B)
    f = orc.vanloan_fit(W, 3, 6, 4, 2, 1)
    assert abs(f["sigma"][0] - np.linalg.norm(A) * np.linalg.norm(B)) <= 1e-12 * f["sigma"][0]
    assert np.allclose(np.kron(f["A"][0], f["B"][0]), W, rtol=0, atol=1e-12)


def pin_vanloan_best_approximation(orc):
    """Eckart-Young on R(W): the squared Frobenius error of the rank-r fit of a random W is
    the sum of the discarded squared singular values, and nudging the fitted factors in
    random directions never lowers the error (the fit is the best Kronecker sum of r
    terms)."""
    rng = np.random.default_rng(229)
    p, q, m1, m2, r = 3, 4, 4, 3, 2
    W = rng.standard_normal((p * m1, q * m2))
    f = orc.vanloan_fit(W, p, q, m1, m2, r, normalize=False)
    Wr = sum(np.kron(f["A"][i], f["B"][i]) for i in range(r))
    err2 = np.sum((W - Wr) ** 2)
    assert abs(err2 - np.sum(f["sigma"][r:] ** 2)) <= 1e-10 * np.sum(W ** 2)
    for t in range(20):
        dA = 1e-3 * rng.standard_normal(f["A"].shape)
        dB = 1e-3 * rng.standard_normal(f["B"].shape)
        Wp = sum(np.kron(f["A"][i] + dA[i], f["B"][i] + dB[i]) for i in range(r))
        assert np.sum((W - Wp) ** 2) >= err2 - 1e-12


def pin_vanloan_alpha_restores_energy(orc):
    """alpha = |W|_F / |sum_i kron(C_i, B_i)|_F; after scaling both factors by sqrt(alpha) the
    fit has the Frobenius norm of W."""
    rng = np.random.default_rng(233)
    p, q, m1, m2 = 3, 3, 4, 4
    W = rng.standard_normal((p * m1, q * m2))
    for r in (1, 2):
        f0 = orc.vanloan_fit(W, p, q, m1, m2, r, normalize=False)
        f1 = orc.vanloan_fit(W, p, q, m1, m2, r, normalize=True)
        W0 = sum(np.kron(f0["A"][i], f0["B"][i]) for i in range(r))
        W1 = sum(np.kron(f1["A"][i], f1["B"][i]) for i in range(r))
        assert abs(f1["alpha"] - np.linalg.norm(W) / np.linalg.norm(W0)) <= 1e-12 * f1["alpha"]
        assert abs(np.linalg.norm(W1) - np.linalg.norm(W)) <= 1e-12 * np.linalg.norm(W)
        assert f1["alpha"] > 1.0


# ---------------------------------------------------------------- triple Kronecker layer
# (page "LLM Compression via Kronecker Product Decomposition", section "Triple Kronecker --
# AxBxC (Extreme Compression)")

def _rand_triple(rng, p, q, m1, m2, s1, s2, r, N=3):
    A = rng.standard_normal((r, p, q))
    B = rng.standard_normal((r, m1, m2))
    C = rng.standard_normal((r, s1, s2))
    x = rng.standard_normal((N, p * m1 * s1))
    G = rng.standard_normal((N, q * m2 * s2))
    bias = rng.standard_normal(q * m2 * s2)
    return A, B, C, x, G, bias


def pin_kron3_weight_is_numpy_triple_kron(orc):
    """W = sum_i kron(A_i, kron(B_i, C_i)) by numpy's kron, rectangular factors; numpy's kron
    is associative, so this is also sum_i kron(kron(A_i, B_i), C_i)."""
    rng = np.random.default_rng(311)
    A, B, C, *_ = _rand_triple(rng, 2, 3, 3, 2, 2, 4, 2)
    W = orc.weight3(A, B, C)
    ref = sum(np.kron(A[i], np.kron(B[i], C[i])) for i in range(2))
    assert np.allclose(W, ref, rtol=0, atol=1e-12)
    ref2 = sum(np.kron(np.kron(A[i], B[i]), C[i]) for i in range(2))
    assert np.allclose(W, ref2, rtol=0, atol=1e-12)


def pin_kron3_forward_brute_force(orc):
    """y[n][(c,k,v)] = sum_{a,j,u} x[n][(a,j,u)] A[a,c] B[j,k] C[u,v] + bias, scalar loops."""
    rng = np.random.default_rng(313)
    p, q, m1, m2, s1, s2, r = 2, 2, 2, 3, 3, 2, 2
    A, B, C, x, G, bias = _rand_triple(rng, p, q, m1, m2, s1, s2, r, N=2)
    y = orc.forward3(x, A, B, C, bias)
    for n in range(2):
        for c, k, v in itertools.product(range(q), range(m2), range(s2)):
            s = bias[(c * m2 + k) * s2 + v]
            for a, j, u, i in itertools.product(range(p), range(m1), range(s1), range(r)):
                s += x[n][(a * m1 + j) * s1 + u] * A[i, a, c] * B[i, j, k] * C[i, u, v]
            assert abs(y[n][(c * m2 + k) * s2 + v] - s) <= 1e-12 * max(1.0, abs(s))


def pin_kron3_finite_differences(orc):
    """Central differences of L = <G, y> in every input (exact up to rounding: L is affine in
    each single coordinate)."""
    rng = np.random.default_rng(317)
    p, q, m1, m2, s1, s2, r = 2, 3, 2, 2, 2, 3, 2
    A, B, C, x, G, bias = _rand_triple(rng, p, q, m1, m2, s1, s2, r)
    g = orc.backward3(x, A, B, C, G)
    L = lambda x_, A_, B_, C_, b_: float(np.sum(G * orc.forward3(x_, A_, B_, C_, b_)))
    h = 1e-3
    args = {"x": x, "A": A, "B": B, "C": C, "bias": bias}
    names = {"x": "dX", "A": "dA", "B": "dB", "C": "dC", "bias": "dbias"}
    for key, grad in names.items():
        base = args[key]
        for idx in list(np.ndindex(base.shape))[:: max(1, base.size // 9)]:
            up_, dn_ = base.copy(), base.copy()
            up_[idx] += h
            dn_[idx] -= h
            a_up = dict(args, **{key: up_})
            a_dn = dict(args, **{key: dn_})
            num = (L(a_up["x"], a_up["A"], a_up["B"], a_up["C"], a_up["bias"]) -
                   L(a_dn["x"], a_dn["A"], a_dn["B"], a_dn["C"], a_dn["bias"])) / (2 * h)
            assert abs(num - g[grad][idx]) <= 1e-7 * max(1.0, abs(num)), (key, idx)


# ---- Kronecker-sparse factor (pattern (a, b, c, d), values w [a][d][b][c]) ----

KS_PATTERNS = [(2, 3, 4, 5), (1, 4, 2, 3), (3, 2, 5, 1), (2, 1, 1, 3), (1, 3, 3, 1), (4, 2, 2, 2)]


def _ks_values(rng, a, b, c, d):
    """Values bounded away from zero, so the support shows in K != 0."""
    return rng.uniform(0.5, 1.5, (a, d, b, c)) * rng.choice([-1.0, 1.0], (a, d, b, c))


def pin_ks_support_is_kron_of_identity_and_ones(orc):
    """supp K = kron(I_a, kron(1_{b x c}, I_d)) (numpy's kron of eye and ones), K is
    (a*b*d) x (a*c*d) and holds exactly a*b*c*d non-zeros, each value once."""
    rng = np.random.default_rng(401)
    for a, b, c, d in KS_PATTERNS:
        w = _ks_values(rng, a, b, c, d)
        K = orc.ks_dense(w)
        mask = np.kron(np.eye(a), np.kron(np.ones((b, c)), np.eye(d)))
        assert K.shape == mask.shape == (a * b * d, a * c * d)
        assert np.array_equal(K != 0, mask != 0), (a, b, c, d)
        assert np.array_equal(np.sort(K[K != 0]), np.sort(w.ravel()))


def pin_ks_block_diagonal(orc):
    """d = 1: K is block-diagonal with the a blocks w[al][0] (scipy's block_diag)."""
    from scipy.linalg import block_diag
    rng = np.random.default_rng(403)
    for a, b, c in ((3, 2, 4), (1, 5, 3), (4, 3, 3)):
        w = rng.standard_normal((a, 1, b, c))
        assert np.array_equal(orc.ks_dense(w), block_diag(*[w[i, 0] for i in range(a)]))


def pin_ks_diagonal(orc):
    """b = c = 1: K = diag(w) with the values in (al, de) order (numpy's diag)."""
    rng = np.random.default_rng(409)
    w = rng.standard_normal((3, 4, 1, 1))
    assert np.array_equal(orc.ks_dense(w), np.diag(w.reshape(12)))


def pin_ks_tied_values_are_numpy_kron(orc):
    """All a*d blocks equal to one rectangular M: K = kron(I_a, kron(M, I_d)); in particular
    a = 1 gives kron(M, I_d) and d = 1 gives kron(I_a, M) (numpy's kron)."""
    rng = np.random.default_rng(419)
    for a, b, c, d in ((1, 3, 2, 4), (3, 2, 4, 1), (2, 3, 2, 3)):
        M = rng.standard_normal((b, c))
        w = np.broadcast_to(M, (a, d, b, c))
        ref = np.kron(np.eye(a), np.kron(M, np.eye(d)))
        assert np.array_equal(orc.ks_dense(w), ref), (a, b, c, d)


def pin_ks_chain_is_kronecker_layer(orc):
    """The vec trick as two KS factors: x -> KS(p, m1, m2, 1) with every block B_i, then
    KS(1, p, q, m2) with every block C_i, summed over i, equals x kron(C_i, B_i) summed over
    i (numpy's kron) -- the two-factor layer's W with S = ones."""
    rng = np.random.default_rng(421)
    p, q, m1, m2, r, N = 3, 2, 2, 4, 2, 5
    C = rng.standard_normal((r, p, q))
    B = rng.standard_normal((r, m1, m2))
    x = rng.standard_normal((N, p * m1))
    y = np.zeros((N, q * m2))
    for i in range(r):
        t = orc.ks_forward(x, np.broadcast_to(B[i], (p, 1, m1, m2)))
        y += orc.ks_forward(t, np.broadcast_to(C[i], (1, m2, p, q)))
    ref = x @ sum(np.kron(C[i], B[i]) for i in range(r))
    assert np.allclose(y, ref, rtol=0, atol=1e-12)


def pin_ks_hadamard_chain(orc):
    """The Walsh-Hadamard transform as a chain of KS factors: with every 2 x 2 block
    [[1, 1], [1, -1]], the product over l = 1..L of the patterns (2^(l-1), 2, 2, 2^(L-l))
    is Sylvester's Hadamard matrix of order 2^L (scipy's hadamard)."""
    from scipy.linalg import hadamard
    L = 4
    n = 1 << L
    H2 = np.array([[1.0, 1.0], [1.0, -1.0]])
    y = np.eye(n)
    for l in range(1, L + 1):
        a, d = 1 << (l - 1), 1 << (L - l)
        y = orc.ks_forward(y, np.broadcast_to(H2, (a, d, 2, 2)))
    assert np.array_equal(y, hadamard(n).astype(np.float64))


def pin_ks_forward_is_numpy_matmul(orc):
    """y = x K + bias with numpy's matmul on the oracle's dense K; bias None means 0."""
    rng = np.random.default_rng(431)
    a, b, c, d, N = 2, 3, 4, 3, 7
    w = rng.standard_normal((a, d, b, c))
    x = rng.standard_normal((N, a * b * d))
    bias = rng.standard_normal(a * c * d)
    K = orc.ks_dense(w)
    assert np.allclose(orc.ks_forward(x, w, bias), x @ K + bias, rtol=0, atol=1e-12)
    assert np.allclose(orc.ks_forward(x, w), x @ K, rtol=0, atol=1e-12)


def pin_ks_finite_differences(orc):
    """Central differences of L = <G, y> in x, w and bias (exact up to rounding: L is affine
    in each single coordinate), on a pattern with a, b, c, d all > 1 and b != c."""
    rng = np.random.default_rng(433)
    a, b, c, d, N = 2, 3, 2, 2, 3
    w = rng.standard_normal((a, d, b, c))
    x = rng.standard_normal((N, a * b * d))
    G = rng.standard_normal((N, a * c * d))
    bias = rng.standard_normal(a * c * d)
    g = orc.ks_backward(x, w, G)
    Lf = lambda x, w, bias: float(np.sum(G * orc.ks_forward(x, w, bias)))
    h = 1e-3
    args = {"x": x, "w": w, "bias": bias}
    for key, grad in (("x", "dX"), ("w", "dw"), ("bias", "dbias")):
        base = args[key]
        for idx in np.ndindex(base.shape):
            up_, dn_ = base.copy(), base.copy()
            up_[idx] += h
            dn_[idx] -= h
            num = (Lf(**dict(args, **{key: up_})) - Lf(**dict(args, **{key: dn_}))) / (2 * h)
            assert abs(num - g[grad][idx]) <= 1e-8 * max(1.0, abs(num)), (key, idx)


def pin_ks_linearity_identities(orc):
    """y - bias is linear in x and in w, so <dX, x> = <dw, w> = <G, y - bias> (Euler)."""
    rng = np.random.default_rng(439)
    a, b, c, d, N = 3, 2, 3, 2, 6
    w = rng.standard_normal((a, d, b, c))
    x = rng.standard_normal((N, a * b * d))
    G = rng.standard_normal((N, a * c * d))
    g = orc.ks_backward(x, w, G)
    ref = float(np.sum(G * orc.ks_forward(x, w)))
    assert abs(float(np.sum(g["dX"] * x)) - ref) <= 1e-11 * max(1.0, abs(ref))
    assert abs(float(np.sum(g["dw"] * w)) - ref) <= 1e-11 * max(1.0, abs(ref))
    assert np.allclose(g["dbias"], G.sum(axis=0), rtol=0, atol=1e-12)


ALL_PINS = [
    pin_weight_is_sum_of_numpy_krons,
    pin_forward_brute_force,
    pin_forward_vec_trick,
    pin_forward_is_gemm_with_numpy_weight,
    pin_mixed_product,
    pin_transpose,
    pin_block_structure,
    pin_rank_one,
    pin_van_loan_rank,
    pin_vanloan_rearrangement_of_krons,
    pin_vanloan_fit_recovers_exact_rank,
    pin_vanloan_rank_one_closed_form,
    pin_vanloan_best_approximation,
    pin_vanloan_alpha_restores_energy,
    pin_kron3_weight_is_numpy_triple_kron,
    pin_kron3_forward_brute_force,
    pin_kron3_finite_differences,
    pin_special_shapes,
    pin_finite_differences,
    pin_linearity_identities,
    pin_backward_numpy_chain_rule,
    pin_zero_s_gradient,
    pin_l1_grad_finite_differences,
    pin_ks_support_is_kron_of_identity_and_ones,
    pin_ks_block_diagonal,
    pin_ks_diagonal,
    pin_ks_tied_values_are_numpy_kron,
    pin_ks_chain_is_kronecker_layer,
    pin_ks_hadamard_chain,
    pin_ks_forward_is_numpy_matmul,
    pin_ks_finite_differences,
    pin_ks_linearity_identities,
]
