"""GPU parity of the tensor-core paths (TF32 and BF16), forward and full backward,
against the fp64 oracle on the same seeded inputs, on the tutorial layer's shape
(p = q = m1 = m2 = 32, r = 4) at ragged and full sizes."""
import dataclasses
import functools

import numpy as np
import pytest
import torch

import kron_workloads as kw
from parity import TOL, compare, gpu_run, oracle_run, rel_err, to_np

pytestmark = pytest.mark.gpu
TUT = kw.get("tutorial")


def _w(path, N=None, **kw_):
    w = TUT if N is None else TUT.with_rows(N)
    return dataclasses.replace(w, dtype="bf16" if path == "bf16" else "f32", **kw_)


@functools.lru_cache(maxsize=None)
def _inputs(w):
    return kw.inputs(w)


@functools.lru_cache(maxsize=None)
def _oracle(w):
    return oracle_run(_inputs(w))


@pytest.mark.parametrize("path", ["tf32", "bf16"])
@pytest.mark.parametrize("N", [1, 3, 4, 5, 37, 600, 1001])
def test_tc_forward_backward_ragged(path, N):
    w = _w(path, N)
    compare(gpu_run(_inputs(w), path), _oracle(w), path)


@pytest.mark.parametrize("path", ["tf32", "bf16"])
def test_tc_tutorial_full_size(path):
    """N = 20000: every element of y, dX, dS, dA, dB and dbias checked."""
    w = _w(path)
    errs = compare(gpu_run(_inputs(w), path), _oracle(w), path)
    print(path, errs)


@pytest.mark.parametrize("path", ["tf32", "bf16"])
def test_tc_no_bias_full_size(path):
    """N = 20000 with no bias: the forward without a bias vector, and the backward with
    neither dbias nor anything bias-related requested; every element of y, dX, dS, dA and
    dB against the oracle's bias-free layer."""
    import kronecker_factored_structured_b200 as kfs
    w = _w(path)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    y = kfs.forward(d["x"], d["S"], d["A"], d["B"], None, dtype=path)
    g = kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path, need_dbias=False)
    torch.cuda.synchronize()
    assert g["dbias"] is None
    got = {"y": to_np(y)}
    got.update({k: to_np(v) for k, v in g.items() if v is not None})
    ref = oracle_run(_inputs(w), with_bias=False)
    errs = compare(got, ref, path, keys=("y", "dX", "dS", "dA", "dB"))
    print(path, "no bias", errs)


@pytest.mark.parametrize("path", ["tf32", "bf16"])
def test_tc_s_all_ones_and_dense_zeroes(path):
    """S with no zeros, and S with 90% zeros (dS still exact where S = 0)."""
    for zeros in (0, 922):
        w = _w(path, 700, s_zero_entries=zeros, seed=77 + zeros)
        compare(gpu_run(_inputs(w), path), _oracle(w), path)


@pytest.mark.parametrize("path", ["tf32", "bf16"])
def test_tc_backward_deterministic(path):
    import kronecker_factored_structured_b200 as kfs
    w = _w(path, 5000)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    runs = [kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path) for _ in range(3)]
    torch.cuda.synchronize()
    for k in runs[0]:
        for r in runs[1:]:
            assert torch.equal(runs[0][k], r[k]), k


@pytest.mark.parametrize("path", ["tf32", "bf16"])
def test_tc_optional_outputs_and_empty(path):
    import kronecker_factored_structured_b200 as kfs
    w = _w(path, 64)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    g = kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path, need_dx=False,
                     need_dbias=False)
    torch.cuda.synchronize()
    ref = _oracle(w)
    for k in ("dS", "dA", "dB"):
        assert rel_err(to_np(g[k]), ref[k]) <= TOL[path], k
    w0 = _w(path, 0)
    d0 = {k: v.cuda() for k, v in _inputs(w0).items()}
    y0 = kfs.forward(d0["x"], d0["S"], d0["A"], d0["B"], d0["bias"], dtype=path)
    g0 = kfs.backward(d0["x"], d0["S"], d0["A"], d0["B"], d0["G"], dtype=path)
    torch.cuda.synchronize()
    assert y0.shape == (0, w0.d_out)
    for k in ("dS", "dA", "dB", "dbias"):
        assert torch.count_nonzero(g0[k]) == 0


@pytest.mark.parametrize("path", ["tf32", "bf16"])
def test_tc_autograd_module(path):
    import kronecker_factored_structured_b200 as kfs
    w = _w(path, 300)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    layer = kfs.KronLinear(w.d_in, w.d_out, w.m1, w.m2, rank=w.r, dtype=path, device="cuda")
    with torch.no_grad():
        for name in ("S", "A", "B", "bias"):
            getattr(layer, name).copy_(d[name])
    x = d["x"].clone().requires_grad_(True)
    y = layer(x)
    y.backward(d["G"])
    torch.cuda.synchronize()
    ref = _oracle(w)
    assert rel_err(to_np(y), ref["y"]) <= TOL[path]
    assert rel_err(to_np(x.grad), ref["dX"]) <= TOL[path]
    for name, key in (("S", "dS"), ("A", "dA"), ("B", "dB"), ("bias", "dbias")):
        assert rel_err(to_np(getattr(layer, name).grad), ref[key]) <= TOL[path], name


def test_tc_no_device_error():
    import kronecker_factored_structured_b200 as kfs
    torch.cuda.synchronize()
    kfs.native.device_error()
