"""GPU parity of the Kronecker-sparse factor (ks_linear_forward / _backward through the C
ABI) against the fp64 oracle: y = x K + bias with supp K = kron(I_a, kron(1_{b x c}, I_d))
(page "Fast Inference with Kronecker-Sparse Matrices", abstract), exact FP32 on the CUDA
cores.  Small patterns cover ragged row, delta, be and ga tiles and the multi-chunk and
split-row paths; the bench's patterns run at full size with sampled rows (y, dX), exact
column sums (dbias) and Euler's identity (dw), and against the oracle at 2048 rows (dw)."""
import numpy as np
import pytest
import torch

import kron_workloads as kw
import oracle
import kronecker_factored_structured_b200 as kfs
from kronecker_factored_structured_b200 import native
from parity import TOL, rel_err

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
TOL_F32 = TOL["f32"]

SMALL = [(2, 3, 4, 5, 37), (1, 4, 2, 3, 9), (3, 2, 5, 1, 11), (2, 1, 1, 3, 5), (4, 2, 2, 2, 3),
         (1, 9, 6, 10, 13), (2, 5, 3, 12, 40), (1, 33, 17, 1, 70), (2, 2, 2, 16, 100),
         (1, 3, 40, 9, 5), (3, 40, 3, 2, 6), (1, 8, 8, 8, 1), (1, 130, 2, 1, 3),
         (1, 2, 130, 1, 3), (16, 2, 2, 32, 300), (1, 64, 64, 16, 257), (2, 100, 70, 3, 129),
         (4, 16, 16, 4, 1000)]


def _gpu(d, need_dx=True, with_bias=True):
    dd = {k: v.to(DEV) for k, v in d.items()}
    y = native.ks_forward(dd["x"], dd["w"], dd["bias"] if with_bias else None)
    g = native.ks_backward(dd["x"], dd["w"], dd["G"], need_dx=need_dx, need_dbias=with_bias)
    torch.cuda.synchronize()
    out = {"y": y}
    out.update(g)
    return {k: (None if v is None else v.double().cpu().numpy()) for k, v in out.items()}


def _oracle(d, with_bias=True):
    f = {k: v.double().numpy() for k, v in d.items()}
    ref = oracle.ks_backward(f["x"], f["w"], f["G"])
    ref["y"] = oracle.ks_forward(f["x"], f["w"], f["bias"] if with_bias else None)
    return ref


def _compare(got, ref, keys):
    errs = {k: rel_err(got[k], ref[k]) for k in keys}
    bad = {k: e for k, e in errs.items() if not e <= TOL_F32}
    assert not bad, f"relative errors above {TOL_F32}: {bad} (all {errs})"
    return errs


@pytest.mark.parametrize("case", SMALL, ids=lambda s: "a{}_b{}_c{}_d{}_N{}".format(*s))
def test_ks_small(case):
    a, b, c, d, N = case
    inp = kw.ks_inputs(kw.ks_custom(N, a, b, c, d, seed=sum(case)))
    _compare(_gpu(inp), _oracle(inp), ("y", "dX", "dw", "dbias"))


def test_ks_no_bias_no_dx():
    inp = kw.ks_inputs(kw.ks_custom(77, 2, 6, 5, 9, seed=5))
    got = _gpu(inp, need_dx=False, with_bias=False)
    assert got["dX"] is None and got["dbias"] is None
    _compare(got, _oracle(inp, with_bias=False), ("y", "dw"))


def test_ks_empty_batch():
    w = torch.randn(2, 3, 4, 5, device=DEV)
    x = torch.empty(0, 2 * 4 * 3, device=DEV)
    y = native.ks_forward(x, w)
    g = native.ks_backward(x, w, torch.empty(0, 2 * 5 * 3, device=DEV),
                           grads={"dw": torch.full_like(w, 7.0)})
    torch.cuda.synchronize()
    assert y.shape == (0, 30)
    assert torch.count_nonzero(g["dw"]).item() == 0 and torch.count_nonzero(g["dbias"]).item() == 0


def test_ks_bitwise_reproducible():
    inp = {k: v.to(DEV) for k, v in kw.ks_inputs(kw.ks_custom(3000, 1, 32, 32, 32, seed=9)).items()}
    g1 = native.ks_backward(inp["x"], inp["w"], inp["G"])
    g2 = native.ks_backward(inp["x"], inp["w"], inp["G"])
    torch.cuda.synchronize()
    for k in ("dX", "dw", "dbias"):
        assert torch.equal(g1[k], g2[k]), k


def test_ks_chain_reproduces_kronecker_layer():
    """x -> KS(p, m1, m2, 1) with every block B -> KS(1, p, q, m2) with every block C is the
    Kronecker layer x kron(C, B) (S = ones, r = 1): two GPU paths against each other and
    against the oracle."""
    p, q, m1, m2, N = 16, 8, 12, 20, 333
    g = torch.Generator().manual_seed(12)
    C = torch.randn(p, q, generator=g) / 4
    B = torch.randn(m1, m2, generator=g) / 4
    x = torch.randn(N, p * m1, generator=g)
    xd = x.to(DEV)
    t = native.ks_forward(xd, B.expand(p, 1, m1, m2).contiguous().to(DEV))
    y = native.ks_forward(t, C.expand(1, m2, p, q).contiguous().to(DEV))
    yk = kfs.forward(xd, torch.ones(p, q, device=DEV), C[None].to(DEV), B[None].to(DEV),
                     dtype="f32")
    ref = oracle.forward(x.double().numpy(), np.ones((p, q)), C[None].double().numpy(),
                         B[None].double().numpy())
    assert rel_err(y.double().cpu().numpy(), ref) <= TOL_F32
    assert rel_err(yk.double().cpu().numpy(), ref) <= TOL_F32


def test_ks_autograd_module():
    torch.manual_seed(3)
    layer = kfs.KSLinear(4, 8, 6, 3, device=DEV)
    with torch.no_grad():
        layer.bias.normal_()
    x = torch.randn(50, 4 * 8 * 3, device=DEV, requires_grad=True)
    G = torch.randn(50, 4 * 6 * 3, device=DEV)
    (layer(x) * G).sum().backward()
    ref = oracle.ks_backward(x.detach().double().cpu().numpy(),
                             layer.w.detach().double().cpu().numpy(), G.double().cpu().numpy())
    assert rel_err(x.grad.double().cpu().numpy(), ref["dX"]) <= TOL_F32
    assert rel_err(layer.w.grad.double().cpu().numpy(), ref["dw"]) <= TOL_F32
    assert rel_err(layer.bias.grad.double().cpu().numpy(), ref["dbias"]) <= TOL_F32


@pytest.mark.parametrize("name", sorted(kw.ks_workloads()))
def test_ks_full_size(name):
    """The bench's workload at full size through the same entry points the bench times."""
    wl = kw.ks_get(name)
    inp = kw.ks_inputs(wl)
    d = {k: v.to(DEV) for k, v in inp.items()}
    y = native.ks_forward(d["x"], d["w"], d["bias"])
    g = native.ks_backward(d["x"], d["w"], d["G"])
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    idx = np.unique(np.concatenate([[0, wl.N - 1], rng.integers(0, wl.N, 254)]))
    xs = inp["x"][idx].double().numpy()
    Gs = inp["G"][idx].double().numpy()
    wv = inp["w"].double().numpy()
    ry = oracle.ks_forward(xs, wv, inp["bias"].double().numpy())
    rdx = oracle.ks_backward(xs, wv, Gs)["dX"]
    e_y = rel_err(y[idx].double().cpu().numpy(), ry)
    e_dx = rel_err(g["dX"][idx].double().cpu().numpy(), rdx)
    # dbias: the exact column sums of dY; dw: <dw, w> = <dY, y - bias> (y - bias is linear in w)
    e_db = rel_err(g["dbias"].double().cpu().numpy(), inp["G"].double().sum(0).numpy())
    lhs = float((g["dw"].double() * d["w"].double()).sum())
    rhs = float((d["G"].double() * (y.double() - d["bias"].double())).sum())
    e_euler = abs(lhs - rhs) / max(1.0, abs(rhs))
    print(f"{name}: y {e_y:.2e} dX {e_dx:.2e} dbias {e_db:.2e} euler {e_euler:.2e}")
    assert e_y <= TOL_F32 and e_dx <= TOL_F32 and e_db <= TOL_F32 and e_euler <= TOL_F32
    # dw against the oracle on the first 2048 rows (the oracle's dw is dense in x^T dY)
    sub = {k: (v[:2048] if k in ("x", "G") else v) for k, v in inp.items()}
    got = _gpu(sub)
    _compare(got, _oracle(sub), ("dw", "dbias"))
