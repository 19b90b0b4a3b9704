"""GPU parity of the backward with the l1 penalty on S fused into the dS epilogue
(kron_linear_backward_l1).  The page "kronecker-layer-benchmark" (introduction) trains S
under lam * sum|S|; the library adds that term's gradient lam * sign(S) where it writes dS.

Checked against the fp64 oracle (chain rule through the explicit W, plus the oracle's
l1 gradient) on the CUDA-core path (exact FP32, any shape) and on the tensor-core paths
(TF32, BF16; the tutorial layer's shape), and against the plain backward: every other
output is bit for bit the same, and lam = 0 through the l1 entry point changes nothing."""
import dataclasses
import functools

import numpy as np
import pytest
import torch

import kron_workloads as kw
import oracle
from parity import TOL, rel_err, to_np

import kronecker_factored_structured_b200 as kfs
from kronecker_factored_structured_b200 import native

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

# (workload, rows, path): the tiny layer and a ragged tutorial-shape batch on exact FP32
# (CUDA-core kernels and the separate reduction), the tutorial shape on TF32 and BF16
# (tensor-core kernels with the reduction fused after the grid barrier)
CASES = [("tiny", None, "f32"), ("tutorial", 300, "f32"), ("tutorial", 600, "tf32"),
         ("tutorial", 1001, "bf16"), ("tutorial", None, "tf32")]


def _workload(name, N, path):
    w = kw.get(name)
    if N is not None:
        w = w.with_rows(N)
    return dataclasses.replace(w, dtype="bf16" if path == "bf16" else "f32")


@functools.lru_cache(maxsize=None)
def _inputs(w):
    return kw.inputs(w)


def _backward(d, path, lam):
    g = kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path, l1=lam)
    torch.cuda.synchronize()
    return {k: to_np(v) for k, v in g.items()}


@pytest.mark.parametrize("name,N,path", CASES, ids=lambda v: str(v))
def test_l1_backward_matches_oracle(name, N, path):
    w = _workload(name, N, path)
    inp = _inputs(w)
    d = {k: v.to(DEV) for k, v in inp.items()}
    # every third entry of S negated, so sign = -1 occurs next to +1 and 0
    flip = torch.arange(d["S"].numel(), device=DEV).reshape(d["S"].shape) % 3 == 0
    d["S"] = d["S"] * torch.where(flip, -1.0, 1.0).to(d["S"].dtype)
    Sn = to_np(d["S"].cpu())
    assert (Sn < 0).any() and (Sn == 0).any() and (Sn > 0).any()
    f = {k: to_np(v) for k, v in inp.items()}
    refg = oracle.backward(f["x"], Sn, f["A"], f["B"], f["G"])
    # a weight of the size of dS itself, so a dropped or sign-flipped term shows at any
    # tolerance
    lam = 0.5 * float(np.abs(refg["dS"]).max())
    want_dS = refg["dS"] + oracle.l1_grad(Sn, lam)
    got = _backward(d, path, lam)
    plain = _backward(d, path, 0.0)
    err = rel_err(got["dS"], want_dS)
    assert err <= TOL[path], (path, err)
    # the penalty's term is visible: without it dS is off by far more than the tolerance
    assert rel_err(plain["dS"], want_dS) > 10 * TOL[path]
    for k in ("dX", "dA", "dB", "dbias"):
        assert np.array_equal(got[k], plain[k]), k
        assert rel_err(got[k], refg[k]) <= TOL[path], k


def _raw_l1_call(d, path, lam, g, ws):
    p, q, m1, m2, r = native.shapes(d["S"], d["A"], d["B"])
    N = d["x"].shape[0]
    st = native.load().kron_linear_backward_l1(
        native._ptr(d["x"]), native._ptr(d["S"]), native._ptr(d["A"]), native._ptr(d["B"]),
        native._ptr(d["G"]), native._ptr(g["dX"]), native._ptr(g["dS"]), native._ptr(g["dA"]),
        native._ptr(g["dB"]), native._ptr(g["dbias"]), N, p, q, m1, m2, r, native.DTYPES[path],
        0, float(lam), native._ptr(ws), ws.numel(), native._stream(None))
    torch.cuda.synchronize()
    return st


@pytest.mark.parametrize("path,N", [("f32", 37), ("tf32", 600), ("bf16", 37)])
def test_l1_zero_weight_is_the_plain_backward(path, N):
    """lam = 0 through kron_linear_backward_l1: bit for bit kron_linear_backward."""
    w = _workload("tutorial", N, path)
    d = {k: v.to(DEV) for k, v in _inputs(w).items()}
    plain = _backward(d, path, 0.0)
    g = {k: torch.full_like(torch.from_numpy(v).to(DEV, torch.float32), float("nan"))
         for k, v in plain.items() if v is not None}
    g["dX"] = g["dX"].to(d["x"].dtype)
    p, q, m1, m2, r = native.shapes(d["S"], d["A"], d["B"])
    ws = torch.empty(max(kfs.workspace_size(N, p, q, m1, m2, r, path), 1), dtype=torch.uint8,
                     device=DEV)
    assert _raw_l1_call(d, path, 0.0, g, ws) == 0
    for k, v in g.items():
        assert np.array_equal(to_np(v), plain[k]), k


@pytest.mark.parametrize("path", ["f32", "tf32", "bf16"])
def test_l1_empty_batch(path):
    """N = 0: no rows contribute, so dS = lam * sign(S) and the other gradients are 0."""
    w = _workload("tutorial", 1, path)
    d = {k: v.to(DEV) for k, v in _inputs(w).items()}
    d["x"], d["G"] = d["x"][:0], d["G"][:0]
    d["S"][0, :5] = torch.tensor([1.5, -2.0, 0.0, -0.25, 3.0], dtype=d["S"].dtype, device=DEV)
    lam = 0.125
    g = _backward(d, path, lam)
    want = oracle.l1_grad(to_np(d["S"].cpu()), lam)
    assert np.array_equal(g["dS"], want)
    for k in ("dA", "dB", "dbias"):
        assert not np.any(g[k]), k


def test_l1_module_gradient_is_autograd_of_the_penalty():
    """KronLinear(l1=lam): S.grad equals that of the plain layer plus autograd's gradient of
    lam * sum|S| (fp32 rounding of one addition apart), and A, B, bias grads are unchanged."""
    torch.manual_seed(7)
    lam = 0.05
    fused = kfs.KronLinear(1024, 1024, 32, rank=4, dtype="tf32", device=DEV, l1=lam)
    plain = kfs.KronLinear(1024, 1024, 32, rank=4, dtype="tf32", device=DEV)
    with torch.no_grad():
        fused.S.copy_(torch.randn(32, 32, device=DEV))
        fused.S[fused.S.abs() < 0.3] = 0.0
        for a, b in zip(plain.parameters(), fused.parameters()):
            a.copy_(b)
    x = torch.randn(777, 1024, device=DEV)
    gy = torch.randn(777, 1024, device=DEV)
    (fused(x) * gy).sum().backward()
    ((plain(x) * gy).sum() + lam * plain.S.abs().sum()).backward()
    torch.cuda.synchronize()
    assert torch.equal(fused.A.grad, plain.A.grad)
    assert torch.equal(fused.B.grad, plain.B.grad)
    assert torch.equal(fused.bias.grad, plain.bias.grad)
    diff = (fused.S.grad - plain.S.grad).abs().max().item()
    assert diff <= 1e-6 * plain.S.grad.abs().max().item(), diff
