"""GPU parity of the tensor-core forward (TF32 and BF16) against the fp64 oracle."""
import functools

import numpy as np
import pytest
import torch

import kron_workloads as kw
import oracle
from parity import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu


def _forward_case(w, path, with_bias=True):
    import kronecker_factored_structured_b200 as kfs
    d = kw.inputs(w)
    g = {k: v.cuda() for k, v in d.items()}
    y = kfs.forward(g["x"], g["S"], g["A"], g["B"], g["bias"] if with_bias else None, dtype=path)
    torch.cuda.synchronize()
    f = {k: to_np(v) for k, v in d.items()}
    ref = oracle.forward(f["x"], f["S"], f["A"], f["B"], f["bias"] if with_bias else None)
    return rel_err(to_np(y), ref)


TUT = kw.get("tutorial")


@pytest.mark.parametrize("path", ["tf32", "bf16"])
@pytest.mark.parametrize("N", [1, 3, 4, 37, 1000, 5001])
def test_tc_forward_ragged(path, N):
    import dataclasses
    w = dataclasses.replace(TUT.with_rows(N), dtype="bf16" if path == "bf16" else "f32")
    assert _forward_case(w, path) <= TOL[path]


@pytest.mark.parametrize("path", ["tf32", "bf16"])
def test_tc_forward_tutorial_full(path):
    import dataclasses
    w = dataclasses.replace(TUT, dtype="bf16" if path == "bf16" else "f32")
    err = _forward_case(w, path)
    print(path, err)
    assert err <= TOL[path]


def test_tc_forward_no_bias():
    assert _forward_case(TUT.with_rows(300), "tf32", with_bias=False) <= TOL["tf32"]


def test_tc_device_error_clear():
    import kronecker_factored_structured_b200 as kfs
    torch.cuda.synchronize()
    kfs.native.device_error()   # raises if any bounded wait has given up
