"""GPU parity: the CUDA library against the fp64 oracle on the same seeded inputs,
output by output (y, dX, dS, dA, dB, dbias), within the path's tolerance."""
import functools

import numpy as np
import pytest
import torch

import kron_workloads as kw
from parity import TOL, compare, gpu_run, oracle_run, rel_err, to_np

pytestmark = pytest.mark.gpu

PATHS = ["f32"]


@functools.lru_cache(maxsize=None)
def _inputs(w):
    return kw.inputs(w)


@functools.lru_cache(maxsize=None)
def _oracle(w, with_bias=True):
    return oracle_run(_inputs(w), with_bias)


@pytest.mark.parametrize("path", PATHS)
def test_tiny_all_outputs(path):
    w = kw.get("tiny")
    compare(gpu_run(_inputs(w), path), _oracle(w), path)


@pytest.mark.parametrize("path", PATHS)
def test_tutorial_layer_full_size(path):
    """1024 x 1024, m = 32, r = 4, N = 20000: every output element checked."""
    w = kw.get("tutorial")
    errs = compare(gpu_run(_inputs(w), path), _oracle(w), path)
    print(path, errs)


FUZZ = [
    # N, p, q, m1, m2, r   (ragged N, rectangular factors, r = 1, several tiles)
    (1, 2, 3, 4, 8, 1),
    (37, 3, 5, 4, 8, 3),
    (129, 16, 8, 8, 4, 1),
    (77, 6, 12, 8, 16, 2),
    (250, 24, 48, 32, 64, 1),
    (251, 48, 24, 64, 32, 4),
    (64, 1, 1, 4, 4, 2),
    (33, 5, 7, 4, 4, 5),
    # the tutorial layer's shape, which has a compiled FP32 forward (8-row tiles): ragged N
    (1, 32, 32, 32, 32, 4),
    (37, 32, 32, 32, 32, 4),
    (300, 32, 32, 32, 32, 4),
]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("shape", FUZZ, ids=lambda s: "N{}_p{}q{}_m{}x{}_r{}".format(*s))
def test_shape_fuzz(path, shape):
    N, p, q, m1, m2, r = shape
    w = kw.custom(N, p, q, m1, m2, r, dtype="f32", seed=N + p, s_zero_entries=(p * q) // 3)
    compare(gpu_run(_inputs(w), path), _oracle(w), path)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("m", [8, 16, 64, 128])
@pytest.mark.parametrize("r", [1, 2, 8])
def test_sweep_shapes(path, m, r):
    """The block-size / rank sweep's shapes (1024^2) at 300 rows."""
    w = kw.get(f"sweep_m{m}_r{r}").with_rows(300)
    compare(gpu_run(_inputs(w), path), _oracle(w), path)


@pytest.mark.parametrize("path", PATHS)
def test_without_bias(path):
    w = kw.get("tiny")
    got = gpu_run(_inputs(w), path, with_bias=False)
    ref = _oracle(w, with_bias=False)
    assert rel_err(got["y"], ref["y"]) <= TOL[path]


@pytest.mark.parametrize("path", PATHS)
def test_backward_is_deterministic(path):
    import kronecker_factored_structured_b200 as kfs
    w = kw.get("tutorial").with_rows(5000)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    runs = [kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path) for _ in range(2)]
    torch.cuda.synchronize()
    for k in runs[0]:
        assert torch.equal(runs[0][k], runs[1][k]), k


@pytest.mark.parametrize("path", PATHS)
def test_skip_flag_matches_unflagged(path):
    w = kw.get("tiny")
    a = gpu_run(_inputs(w), path, flags=0)
    b = gpu_run(_inputs(w), path, flags=1)
    for k in a:
        assert rel_err(b[k], a[k]) <= TOL[path], k


@pytest.mark.parametrize("path", PATHS)
def test_empty_batch(path):
    import kronecker_factored_structured_b200 as kfs
    w = kw.get("tiny").with_rows(0)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    y = kfs.forward(d["x"], d["S"], d["A"], d["B"], d["bias"], dtype=path)
    g = kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path)
    torch.cuda.synchronize()
    assert y.shape == (0, w.d_out)
    for k in ("dS", "dA", "dB", "dbias"):
        assert torch.count_nonzero(g[k]) == 0, k


@pytest.mark.parametrize("path", PATHS)
def test_optional_outputs_skipped(path):
    import kronecker_factored_structured_b200 as kfs
    w = kw.get("tiny")
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    g = kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path, need_dx=False,
                     need_dbias=False)
    torch.cuda.synchronize()
    assert g["dX"] is None and g["dbias"] is None
    ref = _oracle(w)
    for k in ("dS", "dA", "dB"):
        assert rel_err(to_np(g[k]), ref[k]) <= TOL[path], k


@pytest.mark.parametrize("path", PATHS)
def test_autograd_module(path):
    import kronecker_factored_structured_b200 as kfs
    w = kw.get("tiny")
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
