"""ctypes binding of libkronlinear.so (include/kron_linear.h, include/ks_linear.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current CUDA stream.  If the
library has not been built, or a call fails, this module raises -- it never
computes anything itself.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkronlinear.so")

KRON_F32, KRON_TF32, KRON_BF16 = 0, 1, 2
DTYPES = {"f32": KRON_F32, "tf32": KRON_TF32, "bf16": KRON_BF16}
KRON_FLAG_SKIP_ZERO_BLOCKS = 1
KRON_NOALLOC_SCRATCH_BYTES = 8 << 20   # fixed scratch of kron_linear_backward_noalloc

# Paths whose kernels are built into the library.
IMPLEMENTED_PATHS = ("f32", "tf32", "bf16")

STATUS = {0: "KRON_OK", 1: "KRON_ERR_INVALID_ARG", 2: "KRON_ERR_UNSUPPORTED",
          3: "KRON_ERR_ALIGNMENT", 4: "KRON_ERR_WORKSPACE", 5: "KRON_ERR_CUDA",
          6: "KRON_ERR_TIMEOUT"}

# Every symbol include/kron_linear.h declares.
EXPORTS = ("kron_linear_forward", "kron_linear_backward", "kron_linear_backward_l1",
           "kron_linear_backward_noalloc",
           "kron_linear_workspace_size", "kron_vanloan_fit", "kron_vanloan_workspace_size",
           "kron3_linear_forward", "kron3_linear_backward", "kron3_linear_workspace_size",
           "kron_status_string", "kron_last_error", "kron_linear_device_error",
           "kron_linear_abi_version",
           "ks_linear_forward", "ks_linear_backward", "ks_linear_workspace_size")


class KronError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{self.name}: {detail}")


_lib = None


def load(path: str = LIB_PATH):
    """Load the shared library (raises if it is missing: no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing; build it with `python -m kronecker_factored_structured_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, I, U, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
    lib.kron_linear_forward.argtypes = [vp, vp, vp, vp, vp, vp, i64, I, I, I, I, I, I, U, vp]
    lib.kron_linear_forward.restype = I
    lib.kron_linear_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                         i64, I, I, I, I, I, I, U, vp, sz, vp]
    lib.kron_linear_backward.restype = I
    lib.kron_linear_backward_l1.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                            i64, I, I, I, I, I, I, U, ctypes.c_double,
                                            vp, sz, vp]
    lib.kron_linear_backward_l1.restype = I
    lib.kron_linear_backward_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                 i64, I, I, I, I, I, I, U, vp]
    lib.kron_linear_backward_noalloc.restype = I
    lib.kron_vanloan_workspace_size.argtypes = [I, I, I, I, I]
    lib.kron_vanloan_workspace_size.restype = sz
    lib.kron_vanloan_fit.argtypes = [vp, I, I, I, I, I, vp, I, I, I, vp, vp, vp, vp, vp, sz, vp]
    lib.kron_vanloan_fit.restype = I
    lib.kron3_linear_workspace_size.argtypes = [i64, I, I, I, I, I, I, I, I, I]
    lib.kron3_linear_workspace_size.restype = sz
    lib.kron3_linear_forward.argtypes = [vp, vp, vp, vp, vp, vp, i64, I, I, I, I, I, I, I, I, U,
                                         vp, sz, vp]
    lib.kron3_linear_forward.restype = I
    lib.kron3_linear_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, I, I, I,
                                          I, I, I, I, I, U, vp, sz, vp]
    lib.kron3_linear_backward.restype = I
    lib.kron_linear_workspace_size.argtypes = [i64, I, I, I, I, I, I]
    lib.kron_linear_workspace_size.restype = sz
    lib.kron_status_string.argtypes = [I]
    lib.kron_status_string.restype = ctypes.c_char_p
    lib.kron_last_error.argtypes = []
    lib.kron_last_error.restype = ctypes.c_char_p
    lib.kron_linear_device_error.argtypes = [I]
    lib.kron_linear_device_error.restype = I
    lib.kron_linear_abi_version.argtypes = []
    lib.kron_linear_abi_version.restype = I
    lib.ks_linear_forward.argtypes = [vp, vp, vp, vp, i64, I, I, I, I, I, U, vp]
    lib.ks_linear_forward.restype = I
    lib.ks_linear_backward.argtypes = [vp, vp, vp, vp, vp, vp, i64, I, I, I, I, I, U, vp, sz, vp]
    lib.ks_linear_backward.restype = I
    lib.ks_linear_workspace_size.argtypes = [i64, I, I, I, I, I]
    lib.ks_linear_workspace_size.restype = sz
    _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        detail = load().kron_last_error().decode()
        raise KronError(status, detail)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def io_dtype(dtype: str) -> torch.dtype:
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def _expect(t, name, dtype, shape):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def shapes(S, A, B):
    r, p, q = A.shape
    r2, m1, m2 = B.shape
    if tuple(S.shape) != (p, q) or r2 != r:
        raise ValueError(f"inconsistent factor shapes S{tuple(S.shape)} A{tuple(A.shape)} "
                         f"B{tuple(B.shape)}")
    return p, q, m1, m2, r


def device_error(clear: bool = False) -> None:
    """Raise KronError(KRON_ERR_TIMEOUT) if a kernel's bounded wait gave up."""
    _check(load().kron_linear_device_error(1 if clear else 0))


def workspace_size(N, p, q, m1, m2, r, dtype="tf32") -> int:
    return int(load().kron_linear_workspace_size(N, p, q, m1, m2, r, DTYPES[dtype]))


def forward(x, S, A, B, bias=None, dtype="tf32", flags=0, out=None, stream=None):
    """y = x W + bias with W = sum_i kron(S*A_i, B_i), on the library's kernels."""
    p, q, m1, m2, r = shapes(S, A, B)
    N = x.shape[0]
    t = io_dtype(dtype)
    _expect(x, "x", t, (N, p * m1))
    for name, v, shp in (("S", S, (p, q)), ("A", A, (r, p, q)), ("B", B, (r, m1, m2))):
        _expect(v, name, t, shp)
    if bias is not None:
        _expect(bias, "bias", t, (q * m2,))
    if out is None:
        out = torch.empty(N, q * m2, dtype=t, device=x.device)
    _expect(out, "y", t, (N, q * m2))
    _check(load().kron_linear_forward(_ptr(x), _ptr(S), _ptr(A), _ptr(B), _ptr(bias), _ptr(out),
                                      N, p, q, m1, m2, r, DTYPES[dtype], flags, _stream(stream)))
    return out


def backward(x, S, A, B, dY, dtype="tf32", flags=0, need_dx=True, need_dbias=True,
             workspace=None, grads=None, stream=None, l1=0.0):
    """Gradients of <dY, y>: returns dict(dX, dS, dA, dB, dbias).

    dX has the I/O dtype; dS, dA, dB and dbias are float32.  ``grads`` may hold
    preallocated outputs (same keys); ``workspace`` a preallocated uint8 buffer.
    ``l1`` > 0 adds the gradient l1 * sign(S) of the penalty l1 * sum|S| to dS inside the
    library's dS epilogue (kron_linear_backward_l1).
    """
    p, q, m1, m2, r = shapes(S, A, B)
    N = x.shape[0]
    t = io_dtype(dtype)
    _expect(x, "x", t, (N, p * m1))
    _expect(dY, "dY", t, (N, q * m2))
    for name, v, shp in (("S", S, (p, q)), ("A", A, (r, p, q)), ("B", B, (r, m1, m2))):
        _expect(v, name, t, shp)
    dev = x.device
    g = dict(grads or {})
    f32 = torch.float32
    if need_dx and g.get("dX") is None:
        g["dX"] = torch.empty(N, p * m1, dtype=t, device=dev)
    if not need_dx:
        g["dX"] = None
    for k, shp in (("dS", (p, q)), ("dA", (r, p, q)), ("dB", (r, m1, m2))):
        if g.get(k) is None:
            g[k] = torch.empty(shp, dtype=f32, device=dev)
        _expect(g[k], k, f32, shp)
    if need_dbias and g.get("dbias") is None:
        g["dbias"] = torch.empty(q * m2, dtype=f32, device=dev)
    if not need_dbias:
        g["dbias"] = None
    ws_bytes = workspace_size(N, p, q, m1, m2, r, dtype)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    ptrs = (_ptr(x), _ptr(S), _ptr(A), _ptr(B), _ptr(dY), _ptr(g["dX"]), _ptr(g["dS"]),
            _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dbias"]), N, p, q, m1, m2, r, DTYPES[dtype],
            flags)
    tail = (_ptr(workspace), workspace.numel(), _stream(stream))
    if l1:
        _check(load().kron_linear_backward_l1(*ptrs, float(l1), *tail))
    else:
        _check(load().kron_linear_backward(*ptrs, *tail))
    return g


def vanloan_fit(W, p, q, m1, m2, r, k=None, power_iters=2, normalize=True, omega=None,
                seed=0, stream=None):
    """Rank-r Kronecker fit of a dense float32 CUDA matrix W ((p*m1) x (q*m2)) by the
    library's kron_vanloan_fit; returns dict(S = ones, A [r][p][q], B [r][m1][m2],
    sigma [k], alpha).  ``omega`` ([k][m1*m2] float32) is the random test matrix; by default
    it is drawn here with torch (seeded), k = r + 8 capped by the sizes."""
    if k is None:
        k = min(r + 8, 64, p * q, m1 * m2)
    _expect(W, "W", torch.float32, (p * m1, q * m2))
    dev = W.device
    if omega is None:
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        omega = torch.randn(k, m1 * m2, device=dev, generator=g)
    _expect(omega, "omega", torch.float32, (k, m1 * m2))
    A = torch.empty(r, p, q, device=dev)
    B = torch.empty(r, m1, m2, device=dev)
    sigma = torch.empty(k, device=dev)
    alpha = torch.empty(4, device=dev)
    lib = load()
    wsb = int(lib.kron_vanloan_workspace_size(p, q, m1, m2, k))
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
    _check(lib.kron_vanloan_fit(_ptr(W), p, q, m1, m2, r, _ptr(omega), k, power_iters,
                                1 if normalize else 0, _ptr(A), _ptr(B), _ptr(sigma), _ptr(alpha),
                                _ptr(ws), ws.numel(), _stream(stream)))
    return {"S": torch.ones(p, q, device=dev), "A": A, "B": B, "sigma": sigma,
            "alpha": alpha[:1]}


def _shapes3(A, B, C):
    r, p, q = A.shape
    r2, m1, m2 = B.shape
    r3, s1, s2 = C.shape
    if r2 != r or r3 != r:
        raise ValueError("A, B and C must hold the same number of terms")
    return p, q, m1, m2, s1, s2, r


def forward3(x, A, B, C, bias=None, dtype="tf32", flags=0, stream=None):
    """Triple Kronecker layer y = x W + bias, W = sum_i kron(A_i, kron(B_i, C_i))."""
    p, q, m1, m2, s1, s2, r = _shapes3(A, B, C)
    N = x.shape[0]
    t = io_dtype(dtype)
    _expect(x, "x", t, (N, p * m1 * s1))
    for name, v, shp in (("A", A, (r, p, q)), ("B", B, (r, m1, m2)), ("C", C, (r, s1, s2))):
        _expect(v, name, t, shp)
    y = torch.empty(N, q * m2 * s2, dtype=t, device=x.device)
    lib = load()
    n = int(lib.kron3_linear_workspace_size(N, p, q, m1, m2, s1, s2, r, DTYPES[dtype], 0))
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device=x.device)
    _check(lib.kron3_linear_forward(_ptr(x), _ptr(A), _ptr(B), _ptr(C), _ptr(bias), _ptr(y), N, p,
                                    q, m1, m2, s1, s2, r, DTYPES[dtype], flags, _ptr(ws),
                                    ws.numel(), _stream(stream)))
    return y


def backward3(x, A, B, C, dY, dtype="tf32", flags=0, stream=None):
    """Gradients of <dY, y> for the triple layer: dict(dX, dA, dB, dC, dbias)."""
    p, q, m1, m2, s1, s2, r = _shapes3(A, B, C)
    N = x.shape[0]
    t = io_dtype(dtype)
    _expect(x, "x", t, (N, p * m1 * s1))
    _expect(dY, "dY", t, (N, q * m2 * s2))
    dev = x.device
    g = {"dX": torch.empty(N, p * m1 * s1, dtype=t, device=dev),
         "dA": torch.empty(r, p, q, device=dev), "dB": torch.empty(r, m1, m2, device=dev),
         "dC": torch.empty(r, s1, s2, device=dev), "dbias": torch.empty(q * m2 * s2, device=dev)}
    lib = load()
    n = int(lib.kron3_linear_workspace_size(N, p, q, m1, m2, s1, s2, r, DTYPES[dtype], 1))
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device=dev)
    _check(lib.kron3_linear_backward(_ptr(x), _ptr(A), _ptr(B), _ptr(C), _ptr(dY), _ptr(g["dX"]),
                                     _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dbias"]),
                                     N, p, q, m1, m2, s1, s2, r, DTYPES[dtype], flags, _ptr(ws),
                                     ws.numel(), _stream(stream)))
    return g


# ---- Kronecker-sparse factor (include/ks_linear.h) ----

def ks_pattern(w):
    """(a, b, c, d) of the values w, laid out [a][d][b][c]."""
    if w.dim() != 4:
        raise ValueError(f"w must have shape (a, d, b, c), got {tuple(w.shape)}")
    a, d, b, c = w.shape
    return a, b, c, d


def ks_workspace_size(N, a, b, c, d) -> int:
    return int(load().ks_linear_workspace_size(N, a, b, c, d, KRON_F32))


def ks_forward(x, w, bias=None, out=None, stream=None):
    """y = x K + bias for the KS matrix K of pattern (a, b, c, d) with values w."""
    a, b, c, d = ks_pattern(w)
    N = x.shape[0]
    f32 = torch.float32
    _expect(x, "x", f32, (N, a * b * d))
    _expect(w, "w", f32, (a, d, b, c))
    if bias is not None:
        _expect(bias, "bias", f32, (a * c * d,))
    if out is None:
        out = torch.empty(N, a * c * d, dtype=f32, device=x.device)
    _expect(out, "y", f32, (N, a * c * d))
    _check(load().ks_linear_forward(_ptr(x), _ptr(w), _ptr(bias), _ptr(out), N, a, b, c, d,
                                    KRON_F32, 0, _stream(stream)))
    return out


def ks_backward(x, w, dY, need_dx=True, need_dbias=True, workspace=None, grads=None,
                stream=None):
    """Gradients of <dY, y> for the KS factor: dict(dX, dw, dbias) (None where not asked)."""
    a, b, c, d = ks_pattern(w)
    N = x.shape[0]
    f32 = torch.float32
    _expect(x, "x", f32, (N, a * b * d))
    _expect(w, "w", f32, (a, d, b, c))
    _expect(dY, "dY", f32, (N, a * c * d))
    dev = x.device
    g = dict(grads or {})
    if need_dx and g.get("dX") is None:
        g["dX"] = torch.empty(N, a * b * d, dtype=f32, device=dev)
    if not need_dx:
        g["dX"] = None
    if g.get("dw") is None:
        g["dw"] = torch.empty(a, d, b, c, dtype=f32, device=dev)
    _expect(g["dw"], "dw", f32, (a, d, b, c))
    if need_dbias and g.get("dbias") is None:
        g["dbias"] = torch.empty(a * c * d, dtype=f32, device=dev)
    if not need_dbias:
        g["dbias"] = None
    if workspace is None:
        workspace = torch.empty(ks_workspace_size(N, a, b, c, d), dtype=torch.uint8, device=dev)
    _check(load().ks_linear_backward(_ptr(x), _ptr(w), _ptr(dY), _ptr(g["dX"]), _ptr(g["dw"]),
                                     _ptr(g["dbias"]), N, a, b, c, d, KRON_F32, 0,
                                     _ptr(workspace), workspace.numel(), _stream(stream)))
    return g
