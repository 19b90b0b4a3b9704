"""The C ABI: the library loads, exports every symbol the header declares, and its
host-side checks reject bad arguments before launching anything (no GPU needed:
every call below fails validation, so no kernel is ever launched)."""
import ctypes
import os
import re

import pytest

import kronecker_factored_structured_b200 as kfs
from kronecker_factored_structured_b200 import native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("kron_linear.h", "ks_linear.h")]


def header_symbols():
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"KRON_API\s+[\w\s\*]*?\b((?:kron3?|ks)_\w+)\s*\(", text)))


def test_every_header_is_scanned():
    assert sorted(os.listdir(os.path.join(ROOT, "include"))) == sorted(
        os.path.basename(h) for h in HEADERS)


def test_library_exports_every_declared_symbol():
    lib = native.load()
    syms = header_symbols()
    assert set(syms) == set(native.EXPORTS), syms
    for s in syms:
        assert hasattr(lib, s), s


def test_abi_version_and_status_strings():
    lib = native.load()
    assert lib.kron_linear_abi_version() == 2
    for code, name in native.STATUS.items():
        assert lib.kron_status_string(code).decode().startswith(name)


def test_workspace_size_depends_on_shape_only():
    a = kfs.workspace_size(20000, 32, 32, 32, 32, 4, "f32")
    assert a > 0 and a % 256 == 0
    assert a == kfs.workspace_size(20000, 32, 32, 32, 32, 4, "f32")
    assert kfs.workspace_size(0, 0, 32, 32, 32, 4, "f32") == 0      # invalid p
    assert kfs.workspace_size(10, 8, 8, 6, 8, 1, "f32") == 0        # m1 not a multiple of 4


V = ctypes.c_void_p
ALIGNED = V(0x10000)          # never dereferenced: each call below fails a host check
MISALIGNED = V(0x10004)


def fwd(x=ALIGNED, S=ALIGNED, A=ALIGNED, B=ALIGNED, bias=None, y=ALIGNED, N=8, p=2, q=2, m1=4,
        m2=4, r=1, dtype=0, flags=0):
    lib = native.load()
    return lib.kron_linear_forward(x, S, A, B, bias, y, N, p, q, m1, m2, r, dtype, flags, None)


def bwd(ws=None, ws_bytes=0, dtype=0, flags=0, dS=ALIGNED, x=ALIGNED, N=8, m1=4):
    lib = native.load()
    return lib.kron_linear_backward(x, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, dS, ALIGNED,
                                    ALIGNED, None, N, 2, 2, m1, 4, 1, dtype, flags, ws, ws_bytes,
                                    None)


@pytest.mark.parametrize("kwargs,status", [
    (dict(dtype=7), 1),
    (dict(flags=4), 1),
    (dict(N=-1), 1),
    (dict(p=0), 1),
    (dict(r=0), 1),
    (dict(x=None), 1),
    (dict(y=None), 1),
    (dict(S=None, N=0), 1),
    (dict(m1=6), 2),               # not a multiple of 4 (F32)
    (dict(m1=4, dtype=2), 2),      # not a multiple of 8 (BF16)
    (dict(x=MISALIGNED), 3),
    (dict(bias=MISALIGNED), 3),
])
def test_forward_rejects(kwargs, status):
    assert fwd(**kwargs) == status
    assert native.load().kron_last_error().decode() != ""


@pytest.mark.parametrize("kwargs,status", [
    (dict(dtype=5), 1),
    (dict(dS=None), 1),
    (dict(x=MISALIGNED), 3),
    (dict(m1=3), 2),
    (dict(ws=None, ws_bytes=0), 4),                 # no workspace
    (dict(ws=ALIGNED, ws_bytes=16), 4),             # too small
])
def test_backward_rejects(kwargs, status):
    assert bwd(**kwargs) == status


def test_backward_rejects_misaligned_workspace():
    need = kfs.workspace_size(8, 2, 2, 4, 4, 1, "f32")
    assert bwd(ws=V(0x10010), ws_bytes=need) == 3


# shapes without a tensor-core kernel: the block-size sweep's 16x16 and 8x8 blocks on TF32,
# and a small odd-sized layer on BF16
NO_TC = [(64, 64, 16, 16, 2, 1), (128, 128, 8, 8, 8, 1), (3, 5, 8, 8, 3, 2)]


@pytest.mark.parametrize("shape", NO_TC, ids=lambda s: "p{}q{}_m{}x{}_r{}_dt{}".format(*s))
def test_tensor_core_paths_refuse_shapes_without_a_kernel(shape):
    """A TF32 or BF16 request on a shape that no tcgen05 kernel covers returns
    KRON_ERR_UNSUPPORTED from every entry point, before anything touches the device; the
    exact-FP32 path takes the same shape."""
    p, q, m1, m2, r, dt = shape
    lib = native.load()
    assert fwd(p=p, q=q, m1=m1, m2=m2, r=r, dtype=dt) == 2
    assert "tensor-core" in lib.kron_last_error().decode()
    assert lib.kron_linear_workspace_size(8, p, q, m1, m2, r, dt) == 0
    st = lib.kron_linear_backward(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
                                  ALIGNED, ALIGNED, None, 8, p, q, m1, m2, r, dt, 0,
                                  V(0x100000), 1 << 24, None)
    assert st == 2
    st = lib.kron_linear_backward_noalloc(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
                                          ALIGNED, ALIGNED, ALIGNED, None, 8, p, q, m1, m2, r,
                                          dt, 0, None)
    assert st == 2
    assert lib.kron_linear_workspace_size(8, p, q, m1, m2, r, 0) > 0


@pytest.mark.parametrize("args,status", [
    (dict(k=0), 1), (dict(k=65), 1), (dict(r=0), 1), (dict(r=9, k=8), 1),
    (dict(power_iters=17), 1), (dict(W=None), 1), (dict(omega=None), 1),
    (dict(p=2, q=2, k=8), 1),              # k > p*q
    (dict(W=MISALIGNED), 3), (dict(ws=None), 4), (dict(ws_bytes=64), 4),
    (dict(ws=V(0x100010)), 3),
])
def test_vanloan_fit_rejects(args, status):
    """kron_vanloan_fit's host checks, before anything is launched."""
    lib = native.load()
    a = dict(W=ALIGNED, p=4, q=4, m1=4, m2=4, r=2, omega=ALIGNED, k=8, power_iters=2,
             normalize=1, ws=V(0x100000), ws_bytes=1 << 24)
    a.update(args)
    st = lib.kron_vanloan_fit(a["W"], a["p"], a["q"], a["m1"], a["m2"], a["r"], a["omega"],
                              a["k"], a["power_iters"], a["normalize"], ALIGNED, ALIGNED, ALIGNED,
                              ALIGNED, a["ws"], a["ws_bytes"], None)
    assert st == status, lib.kron_last_error().decode()
    assert lib.kron_last_error().decode() != ""


def test_kron3_host_checks():
    """The triple Kronecker entry points check sizes, pointers and workspace on the host."""
    lib = native.load()
    assert lib.kron3_linear_workspace_size(64, 32, 32, 4, 4, 8, 8, 4, 1, 1) > 0
    assert lib.kron3_linear_workspace_size(64, 32, 32, 4, 4, 8, 8, 0, 1, 1) == 0     # r = 0
    assert lib.kron3_linear_workspace_size(64, 3, 5, 2, 2, 4, 4, 1, 2, 1) == 0       # no BF16 kernel
    assert lib.kron3_linear_workspace_size(64, 3, 5, 2, 2, 4, 4, 1, 0, 1) > 0        # F32 takes it
    st = lib.kron3_linear_forward(ALIGNED, None, ALIGNED, ALIGNED, None, ALIGNED, 8, 2, 2, 4, 4,
                                  2, 2, 1, 0, 0, V(0x100000), 1 << 20, None)
    assert st == 1                                                                  # A missing
    st = lib.kron3_linear_forward(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, ALIGNED, 8, 2, 2, 4,
                                  4, 2, 2, 1, 0, 0, None, 0, None)
    assert st == 4                                                                  # no workspace
    st = lib.kron3_linear_backward(ALIGNED, ALIGNED, ALIGNED, MISALIGNED, ALIGNED, ALIGNED,
                                   ALIGNED, ALIGNED, ALIGNED, None, 8, 2, 2, 4, 4, 2, 2, 1, 0, 0,
                                   V(0x100000), 1 << 20, None)
    assert st == 3                                                                  # C misaligned


def test_vanloan_workspace_size():
    lib = native.load()
    assert lib.kron_vanloan_workspace_size(32, 32, 32, 32, 12) >= 4 * 1024 * 1024
    assert lib.kron_vanloan_workspace_size(32, 32, 32, 32, 0) == 0
    assert lib.kron_vanloan_workspace_size(2, 2, 32, 32, 8) == 0     # k > p*q


def test_noalloc_checks_arguments_before_the_size_limit():
    """An oversized problem with a missing or misaligned pointer gets the pointer's status,
    not KRON_ERR_WORKSPACE: the argument checks come first."""
    lib = native.load()
    big = (20000, 64, 64, 64, 64, 8)
    assert lib.kron_linear_workspace_size(*big, 0) > native.KRON_NOALLOC_SCRATCH_BYTES

    def call(x=ALIGNED, dS=ALIGNED):
        return lib.kron_linear_backward_noalloc(x, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
                                                dS, ALIGNED, ALIGNED, None, *big, 0, 0, None)
    assert call() == 4
    assert call(dS=None) == 1
    assert call(x=MISALIGNED) == 3


@pytest.mark.parametrize("l1", [-1.0, float("nan"), float("inf"), -1e-300])
def test_backward_l1_rejects_bad_weight(l1):
    """The penalty weight must be finite and >= 0; checked before any pointer is read."""
    lib = native.load()
    need = kfs.workspace_size(8, 2, 2, 4, 4, 1, "f32")
    st = lib.kron_linear_backward_l1(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
                                     ALIGNED, ALIGNED, ALIGNED, None, 8, 2, 2, 4, 4, 1, 0, 0, l1,
                                     ALIGNED, need, None)
    assert st == 1
    assert "l1" in lib.kron_last_error().decode()


def test_backward_l1_runs_the_same_checks():
    lib = native.load()
    st = lib.kron_linear_backward_l1(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
                                     None, ALIGNED, ALIGNED, None, 8, 2, 2, 4, 4, 1, 0, 0, 0.5,
                                     ALIGNED, 1 << 20, None)
    assert st == 1                                  # dS missing
    st = lib.kron_linear_backward_l1(MISALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
                                     ALIGNED, ALIGNED, ALIGNED, None, 8, 2, 2, 4, 4, 1, 0, 0, 0.5,
                                     ALIGNED, 1 << 20, None)
    assert st == 3


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="needs a host without a usable GPU: the CUDA runtime must refuse")
@pytest.mark.parametrize("dtype", [0, 1, 2])
def test_cuda_failure_surfaces_as_kron_err_cuda(dtype):
    """Arguments that pass every host check on a host whose CUDA runtime cannot run anything:
    the first CUDA call fails, nothing is launched, and the status is KRON_ERR_CUDA with the
    failing step in kron_last_error() (the pointers are never dereferenced on the host)."""
    lib = native.load()
    st = lib.kron_linear_forward(ALIGNED, ALIGNED, ALIGNED, ALIGNED, None, ALIGNED, 8, 32, 32,
                                 32, 32, 4, dtype, 0, None)
    assert st == 5
    assert "forward launch" in lib.kron_last_error().decode()
    need = lib.kron_linear_workspace_size(8, 32, 32, 32, 32, 4, dtype)
    st = lib.kron_linear_backward(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
                                  ALIGNED, ALIGNED, None, 8, 32, 32, 32, 32, 4, dtype, 0,
                                  V(0x100000), need, None)
    assert st == 5 and lib.kron_last_error().decode() != ""
    st = lib.kron_linear_backward_noalloc(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
                                          ALIGNED, ALIGNED, ALIGNED, None, 8, 32, 32, 32, 32, 4,
                                          dtype, 0, None)
    assert st == 5
    assert lib.kron_linear_device_error(0) == 5


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU or eager fallback: without the built library every call raises."""
    monkeypatch.setattr(native, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        native.load(str(tmp_path / "libkronlinear.so"))


def test_python_binding_raises_without_cuda_tensors():
    import torch
    x = torch.zeros(4, 8)
    S, A, B = torch.ones(2, 2), torch.zeros(1, 2, 2), torch.zeros(1, 4, 4)
    with pytest.raises(ValueError):
        kfs.forward(x, S, A, B, dtype="f32")


# ---- Kronecker-sparse factor (include/ks_linear.h) ----

def ks_fwd(x=ALIGNED, w=ALIGNED, bias=None, y=ALIGNED, N=8, a=2, b=3, c=4, d=5, dtype=0, flags=0):
    return native.load().ks_linear_forward(x, w, bias, y, N, a, b, c, d, dtype, flags, None)


def ks_bwd(ws=V(0x100000), ws_bytes=1 << 30, N=8, a=2, b=3, c=4, d=5, dtype=0, x=ALIGNED,
           dw=ALIGNED, dbias=None):
    return native.load().ks_linear_backward(x, ALIGNED, ALIGNED, ALIGNED, dw, dbias, N, a, b, c,
                                            d, dtype, 0, ws, ws_bytes, None)


@pytest.mark.parametrize("kwargs,status", [
    (dict(dtype=7), 1),
    (dict(flags=1), 1),
    (dict(N=-1), 1),
    (dict(a=0), 1),
    (dict(d=0), 1),
    (dict(x=None), 1),
    (dict(w=None, N=0), 1),
    (dict(a=1, b=1 << 13, d=1 << 12), 1),     # a*b*d above 2^24
    (dict(dtype=1), 2),                       # TF32: no KS kernel
    (dict(dtype=2), 2),                       # BF16: no KS kernel
    (dict(x=V(0x10002)), 3),
    (dict(bias=V(0x10001)), 3),
])
def test_ks_forward_rejects(kwargs, status):
    assert ks_fwd(**kwargs) == status
    assert native.load().kron_last_error().decode() != ""


@pytest.mark.parametrize("kwargs,status", [
    (dict(dtype=1), 2),
    (dict(dw=None), 1),
    (dict(x=None), 1),
    (dict(ws=None), 4),
    (dict(ws_bytes=16), 4),
    (dict(ws=V(0x100080)), 3),
    (dict(dbias=V(0x10006)), 3),
])
def test_ks_backward_rejects(kwargs, status):
    assert ks_bwd(**kwargs) == status


def test_ks_workspace_size():
    n = native.ks_workspace_size(20000, 1, 32, 32, 32)
    assert n > 0 and n % 256 == 0
    assert n == native.ks_workspace_size(20000, 1, 32, 32, 32)
    n0 = native.ks_workspace_size(0, 1, 32, 32, 32)                  # empty batch: valid
    assert n0 > 0 and n0 % 256 == 0
    assert native.ks_workspace_size(-1, 1, 32, 32, 32) == 0
    assert native.load().ks_linear_workspace_size(100, 1, 2, 2, 1, 1) == 0   # TF32: unsupported
    # the partials grow with the rows until every part has its chunk, then stay fixed
    assert native.ks_workspace_size(10, 32, 32, 32, 1) <= native.ks_workspace_size(20000, 32, 32, 32, 1)


def test_ks_binding_checks_before_any_call():
    """The binding's shape and dtype checks run before the library is called (CPU tensors)."""
    import torch
    w = torch.zeros(2, 5, 3, 4)                      # a = 2, d = 5, b = 3, c = 4
    assert native.ks_pattern(w) == (2, 3, 4, 5)
    with pytest.raises(ValueError):
        native.ks_pattern(torch.zeros(3, 3))
    with pytest.raises(ValueError):
        native.ks_forward(torch.zeros(7, 29), w)     # in = a*b*d = 30
    with pytest.raises(TypeError):
        native.ks_forward(torch.zeros(7, 30, dtype=torch.float64), w)
    with pytest.raises(ValueError):
        native.ks_backward(torch.zeros(7, 30), w, torch.zeros(7, 41))   # out = a*c*d = 40
