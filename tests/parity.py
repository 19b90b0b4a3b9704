"""Shared helpers of the GPU parity tests: run the CUDA library and the fp64
oracle on the same seeded inputs and compare them output by output."""
from __future__ import annotations

import numpy as np
import torch

import kron_workloads as kw
import oracle

# max |gpu - oracle| / max |oracle| per output tensor, by path (tolerances stated
# for the layer: 1e-5 exact FP32, 5e-3 TF32, 2e-2 BF16)
TOL = {"f32": 1e-5, "tf32": 5e-3, "bf16": 2e-2}
OUTPUTS = ("y", "dX", "dS", "dA", "dB", "dbias")


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / scale)


def to_np(t):
    return None if t is None else t.detach().float().cpu().numpy().astype(np.float64)


def gpu_run(inputs: dict, dtype: str, flags: int = 0, with_bias: bool = True):
    import kronecker_factored_structured_b200 as kfs
    dev = torch.device("cuda", 0)
    d = {k: v.to(dev) for k, v in inputs.items()}
    y = kfs.forward(d["x"], d["S"], d["A"], d["B"], d["bias"] if with_bias else None,
                    dtype=dtype, flags=flags)
    g = kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=dtype, flags=flags)
    torch.cuda.synchronize()
    out = {"y": to_np(y)}
    out.update({k: to_np(v) for k, v in g.items()})
    return out


def oracle_run(inputs: dict, with_bias: bool = True):
    f = {k: to_np(v) for k, v in inputs.items()}
    y = oracle.forward(f["x"], f["S"], f["A"], f["B"], f["bias"] if with_bias else None)
    g = oracle.backward(f["x"], f["S"], f["A"], f["B"], f["G"])
    g["y"] = y
    return g


def compare(got: dict, ref: dict, dtype: str, keys=OUTPUTS):
    errs = {k: rel_err(got[k], ref[k]) for k in keys}
    bad = {k: e for k, e in errs.items() if not e <= TOL[dtype]}
    assert not bad, f"{dtype}: relative errors above {TOL[dtype]}: {bad} (all: {errs})"
    return errs


def workload_inputs(w: kw.Workload) -> dict:
    return kw.inputs(w)
