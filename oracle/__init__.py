"""fp64 CPU oracle for the sum-of-Kronecker-products linear layer.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library never calls it and shares no code with it.

The arithmetic lives in ``kron_oracle.c`` (plain C, double precision): it builds
W = sum_i kron(S (.) A_i, B_i) entry by entry and multiplies naively, as the
page "kronecker-layer-benchmark", section "1. Build W, then multiply" defines
the layer; the backward is the chain rule through that explicit W.  This module
only marshals numpy arrays into that library, except for the Van Loan fit,
whose SVD step is numpy's (a library routine serving as one step of the
algorithm as the page gives it).  The same library holds the Kronecker-sparse
factor of the page "Fast Inference with Kronecker-Sparse Matrices" (its dense
matrix built entry by entry from the pattern, then the same naive multiply).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kron_oracle.c")
_LIB = os.path.join(_HERE, "_kron_oracle.so")


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile a C source of the oracle into a shared library (gcc, OpenMP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", tmp, src]
        )
        os.replace(tmp, out)
    return out


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shapes(S, A, B):
    r, p, q = A.shape
    r2, m1, m2 = B.shape
    if S.shape != (p, q) or r2 != r:
        raise ValueError(f"inconsistent factor shapes S{S.shape} A{A.shape} B{B.shape}")
    return p, q, m1, m2, r


class Oracle:
    """numpy front end of one compiled copy of kron_oracle.c."""

    def __init__(self, so_path: str):
        lib = ctypes.CDLL(so_path)
        dp = ctypes.POINTER(ctypes.c_double)
        L, I = ctypes.c_long, ctypes.c_int
        lib.oracle_build_weight.argtypes = [dp, dp, dp, I, I, I, I, I, dp]
        lib.oracle_matmul_bias.argtypes = [dp, dp, dp, L, L, L, dp]
        lib.oracle_forward.argtypes = [dp, dp, dp, dp, dp, L, I, I, I, I, I, dp]
        lib.oracle_backward.argtypes = [dp, dp, dp, dp, dp, L, I, I, I, I, I,
                                        dp, dp, dp, dp, dp]
        lib.oracle_l1_grad.argtypes = [dp, I, I, ctypes.c_double, dp]
        lib.oracle_vanloan_rearrange.argtypes = [dp, I, I, I, I, dp]
        lib.oracle_build_weight3.argtypes = [dp, dp, dp, I, I, I, I, I, I, I, dp]
        lib.oracle_forward3.argtypes = [dp, dp, dp, dp, dp, L, I, I, I, I, I, I, I, dp]
        lib.oracle_backward3.argtypes = [dp, dp, dp, dp, dp, L, I, I, I, I, I, I, I,
                                         dp, dp, dp, dp, dp]
        lib.oracle_ks_build.argtypes = [dp, I, I, I, I, dp]
        lib.oracle_ks_forward.argtypes = [dp, dp, dp, L, I, I, I, I, dp]
        lib.oracle_ks_backward.argtypes = [dp, dp, dp, L, I, I, I, I, dp, dp, dp]
        lib.oracle_set_threads.argtypes = [I]
        lib.oracle_get_threads.restype = I
        self._lib = lib

    def set_threads(self, n: int) -> None:
        self._lib.oracle_set_threads(int(n))

    def get_threads(self) -> int:
        return int(self._lib.oracle_get_threads())

    def weight(self, S, A, B) -> np.ndarray:
        """Dense W = sum_i kron(S (.) A_i, B_i), shape (p*m1, q*m2)."""
        S, A, B = _f64(S), _f64(A), _f64(B)
        p, q, m1, m2, r = _shapes(S, A, B)
        W = np.empty((p * m1, q * m2), dtype=np.float64)
        self._lib.oracle_build_weight(_ptr(S), _ptr(A), _ptr(B), p, q, m1, m2, r, _ptr(W))
        return W

    def forward(self, x, S, A, B, bias=None) -> np.ndarray:
        """y = x W + bias for x of shape (N, p*m1); returns (N, q*m2) float64."""
        x, S, A, B = _f64(x), _f64(S), _f64(A), _f64(B)
        p, q, m1, m2, r = _shapes(S, A, B)
        N = x.shape[0]
        if x.shape != (N, p * m1):
            raise ValueError(f"x has shape {x.shape}, expected (N, {p * m1})")
        bias = None if bias is None else _f64(bias)
        y = np.empty((N, q * m2), dtype=np.float64)
        self._lib.oracle_forward(_ptr(x), _ptr(S), _ptr(A), _ptr(B), _ptr(bias),
                                 N, p, q, m1, m2, r, _ptr(y))
        return y

    def backward(self, x, S, A, B, G, need_dx: bool = True, need_params: bool = True) -> dict:
        """Gradients of <G, y> with respect to x, S, A, B and bias (float64).

        Returns a dict with keys dX, dS, dA, dB, dbias (None where not requested).
        """
        x, S, A, B, G = _f64(x), _f64(S), _f64(A), _f64(B), _f64(G)
        p, q, m1, m2, r = _shapes(S, A, B)
        N = x.shape[0]
        if x.shape != (N, p * m1) or G.shape != (N, q * m2):
            raise ValueError("x / G shapes do not match the factors")
        dX = np.empty_like(x) if need_dx else None
        dS = np.empty((p, q)) if need_params else None
        dA = np.empty((r, p, q)) if need_params else None
        dB = np.empty((r, m1, m2)) if need_params else None
        dbias = np.empty((q * m2,)) if need_params else None
        self._lib.oracle_backward(_ptr(x), _ptr(S), _ptr(A), _ptr(B), _ptr(G),
                                  N, p, q, m1, m2, r,
                                  _ptr(dX), _ptr(dS), _ptr(dA), _ptr(dB), _ptr(dbias))
        return {"dX": dX, "dS": dS, "dA": dA, "dB": dB, "dbias": dbias}

    def l1_grad(self, S, lam: float) -> np.ndarray:
        """Gradient lam * sign(S) of the penalty lam * sum|S| (0 where S is 0)."""
        S = _f64(S)
        if S.ndim != 2:
            raise ValueError("S must be p x q")
        out = np.empty_like(S)
        self._lib.oracle_l1_grad(_ptr(S), S.shape[0], S.shape[1], float(lam), _ptr(out))
        return out


    def vanloan_rearrange(self, W, p, q, m1, m2) -> np.ndarray:
        """Wt[(a, c)][(j, k)] = W[a*m1 + j][c*m2 + k], shape (p*q, m1*m2)."""
        W = _f64(W)
        if W.shape != (p * m1, q * m2):
            raise ValueError(f"W has shape {W.shape}, expected ({p * m1}, {q * m2})")
        Wt = np.empty((p * q, m1 * m2), dtype=np.float64)
        self._lib.oracle_vanloan_rearrange(_ptr(W), p, q, m1, m2, _ptr(Wt))
        return Wt

    def vanloan_fit(self, W, p, q, m1, m2, r, normalize: bool = True) -> dict:
        """Rank-r Kronecker fit of a dense W, in the steps of the page "LLM Compression via
        Kronecker Product Decomposition" (sections "Van Loan Rearrangement (1993)" and
        "Adaptive Normalization"):

          1. Wt = R(W), the rearrangement above;
          2. Wt = U diag(s) V^T (numpy's SVD: the library routine is this step);
          3. C_i = sqrt(s_i) reshape(u_i, p, q),  B_i = sqrt(s_i) reshape(v_i, m1, m2), i < r;
          4. alpha = ||W||_F / ||sum_i kron(C_i, B_i)||_F, and with normalize each factor is
             scaled by sqrt(alpha) (so the fit carries the energy of W).

        Returns dict(A = C stacked [r][p][q], B [r][m1][m2], sigma = s (all of them), alpha).
        With S = ones, (S, A, B) are factors of this layer.  The sum of r terms is unique
        when s_{r-1} > s_r; each pair (C_i, B_i) is fixed up to a common sign."""
        Wt = self.vanloan_rearrange(W, p, q, m1, m2)
        U, s, Vt = np.linalg.svd(Wt, full_matrices=False)
        C = np.stack([np.sqrt(s[i]) * U[:, i].reshape(p, q) for i in range(r)])
        B = np.stack([np.sqrt(s[i]) * Vt[i].reshape(m1, m2) for i in range(r)])
        Wr = self.weight(np.ones((p, q)), C, B)
        alpha = float(np.sqrt(np.sum(_f64(W) ** 2)) / np.sqrt(np.sum(Wr ** 2)))
        if normalize:
            C, B = C * np.sqrt(alpha), B * np.sqrt(alpha)
        return {"A": C, "B": B, "sigma": s, "alpha": alpha}


    # ---- triple Kronecker layer: W = sum_i kron(A_i, kron(B_i, C_i)) ----
    @staticmethod
    def _shapes3(A, B, C):
        r, p, q = A.shape
        r2, m1, m2 = B.shape
        r3, s1, s2 = C.shape
        if r2 != r or r3 != r:
            raise ValueError("A, B, C must hold the same number of terms")
        return p, q, m1, m2, s1, s2, r

    def weight3(self, A, B, C) -> np.ndarray:
        """Dense W = sum_i kron(A_i, kron(B_i, C_i)), shape (p*m1*s1, q*m2*s2)."""
        A, B, C = _f64(A), _f64(B), _f64(C)
        p, q, m1, m2, s1, s2, r = self._shapes3(A, B, C)
        W = np.empty((p * m1 * s1, q * m2 * s2))
        self._lib.oracle_build_weight3(_ptr(A), _ptr(B), _ptr(C), p, q, m1, m2, s1, s2, r, _ptr(W))
        return W

    def forward3(self, x, A, B, C, bias=None) -> np.ndarray:
        x, A, B, C = _f64(x), _f64(A), _f64(B), _f64(C)
        p, q, m1, m2, s1, s2, r = self._shapes3(A, B, C)
        N = x.shape[0]
        if x.shape != (N, p * m1 * s1):
            raise ValueError(f"x has shape {x.shape}, expected (N, {p * m1 * s1})")
        bias = None if bias is None else _f64(bias)
        y = np.empty((N, q * m2 * s2))
        self._lib.oracle_forward3(_ptr(x), _ptr(A), _ptr(B), _ptr(C), _ptr(bias), N, p, q, m1, m2,
                                  s1, s2, r, _ptr(y))
        return y

    def backward3(self, x, A, B, C, G) -> dict:
        """Gradients of <G, y> for the triple layer: dict(dX, dA, dB, dC, dbias)."""
        x, A, B, C, G = _f64(x), _f64(A), _f64(B), _f64(C), _f64(G)
        p, q, m1, m2, s1, s2, r = self._shapes3(A, B, C)
        N = x.shape[0]
        dX, dA, dB, dC = np.empty_like(x), np.empty_like(A), np.empty_like(B), np.empty_like(C)
        dbias = np.empty(q * m2 * s2)
        self._lib.oracle_backward3(_ptr(x), _ptr(A), _ptr(B), _ptr(C), _ptr(G), N, p, q, m1, m2,
                                   s1, s2, r, _ptr(dX), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dbias))
        return {"dX": dX, "dA": dA, "dB": dB, "dC": dC, "dbias": dbias}


    # ---- Kronecker-sparse factor: support kron(I_a, kron(1_{b x c}, I_d)) ----
    @staticmethod
    def _ks_pattern(w):
        if w.ndim != 4:
            raise ValueError("w must have shape (a, d, b, c)")
        a, d, b, c = w.shape
        return a, b, c, d

    def ks_dense(self, w) -> np.ndarray:
        """Dense KS matrix K ((a*b*d) x (a*c*d)) of the values w [a][d][b][c]:
        K[(al*b + be)*d + de][(al*c + ga)*d + de] = w[al][de][be][ga], zero elsewhere."""
        w = _f64(w)
        a, b, c, d = self._ks_pattern(w)
        K = np.empty((a * b * d, a * c * d))
        self._lib.oracle_ks_build(_ptr(w), a, b, c, d, _ptr(K))
        return K

    def ks_forward(self, x, w, bias=None) -> np.ndarray:
        """y = x K + bias for x of shape (N, a*b*d); returns (N, a*c*d)."""
        x, w = _f64(x), _f64(w)
        a, b, c, d = self._ks_pattern(w)
        N = x.shape[0]
        if x.shape != (N, a * b * d):
            raise ValueError(f"x has shape {x.shape}, expected (N, {a * b * d})")
        bias = None if bias is None else _f64(bias)
        y = np.empty((N, a * c * d))
        self._lib.oracle_ks_forward(_ptr(x), _ptr(w), _ptr(bias), N, a, b, c, d, _ptr(y))
        return y

    def ks_backward(self, x, w, G) -> dict:
        """Gradients of <G, y>: dict(dX, dw, dbias)."""
        x, w, G = _f64(x), _f64(w), _f64(G)
        a, b, c, d = self._ks_pattern(w)
        N = x.shape[0]
        if x.shape != (N, a * b * d) or G.shape != (N, a * c * d):
            raise ValueError("x / G shapes do not match the pattern")
        dX, dw, dbias = np.empty_like(x), np.empty_like(w), np.empty(a * c * d)
        self._lib.oracle_ks_backward(_ptr(x), _ptr(w), _ptr(G), N, a, b, c, d, _ptr(dX),
                                     _ptr(dw), _ptr(dbias))
        return {"dX": dX, "dw": dw, "dbias": dbias}


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def set_threads(n: int) -> None:
    default().set_threads(n)


def get_threads() -> int:
    return default().get_threads()


def weight(S, A, B) -> np.ndarray:
    return default().weight(S, A, B)


def forward(x, S, A, B, bias=None) -> np.ndarray:
    return default().forward(x, S, A, B, bias)


def backward(x, S, A, B, G, need_dx: bool = True, need_params: bool = True) -> dict:
    return default().backward(x, S, A, B, G, need_dx, need_params)


def l1_grad(S, lam: float) -> np.ndarray:
    return default().l1_grad(S, lam)


def vanloan_rearrange(W, p, q, m1, m2) -> np.ndarray:
    return default().vanloan_rearrange(W, p, q, m1, m2)


def vanloan_fit(W, p, q, m1, m2, r, normalize: bool = True) -> dict:
    return default().vanloan_fit(W, p, q, m1, m2, r, normalize)


def weight3(A, B, C) -> np.ndarray:
    return default().weight3(A, B, C)


def forward3(x, A, B, C, bias=None) -> np.ndarray:
    return default().forward3(x, A, B, C, bias)


def backward3(x, A, B, C, G) -> dict:
    return default().backward3(x, A, B, C, G)


def ks_dense(w) -> np.ndarray:
    return default().ks_dense(w)


def ks_forward(x, w, bias=None) -> np.ndarray:
    return default().ks_forward(x, w, bias)


def ks_backward(x, w, G) -> dict:
    return default().ks_backward(x, w, G)
