"""kron_linear_backward_noalloc: the backward for callers that cannot allocate device
memory when they call it (its scratch is a fixed array inside the library).

Called through the C ABI twice in a row and compared with kron_linear_backward run
with a caller-owned workspace.  Both run the same kernels with the same fixed row-range
split and summation order, so the results must be equal bit for bit.  This file is
collected last on purpose."""
import ctypes
import dataclasses

import pytest
import torch

import kron_workloads as kw
from kronecker_factored_structured_b200 import native

pytestmark = pytest.mark.gpu


def _noalloc(d, w, path):
    """One call of kron_linear_backward_noalloc through ctypes; returns the gradients."""
    lib = native.load()
    dev = d["x"].device
    t = native.io_dtype(path)
    g = {"dX": torch.empty(w.N, w.d_in, dtype=t, device=dev),
         "dS": torch.empty(w.p, w.q, device=dev),
         "dA": torch.empty(w.r, w.p, w.q, device=dev),
         "dB": torch.empty(w.r, w.m1, w.m2, device=dev),
         "dbias": torch.empty(w.d_out, device=dev)}
    P = lambda x: ctypes.c_void_p(x.data_ptr())
    st = lib.kron_linear_backward_noalloc(
        P(d["x"]), P(d["S"]), P(d["A"]), P(d["B"]), P(d["G"]), P(g["dX"]), P(g["dS"]),
        P(g["dA"]), P(g["dB"]), P(g["dbias"]), w.N, w.p, w.q, w.m1, w.m2, w.r,
        native.DTYPES[path], 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, (native.STATUS.get(st), lib.kron_last_error().decode())
    return g


@pytest.mark.parametrize("path,workload", [("tf32", "tutorial"), ("bf16", "tutorial"),
                                           ("f32", "tiny")])
def test_noalloc_matches_workspace_entry_point(path, workload):
    w = kw.get(workload)
    if workload == "tutorial":
        w = w.with_rows(5000)
    w = dataclasses.replace(w, dtype="bf16" if path == "bf16" else "f32")
    need = native.workspace_size(w.N, w.p, w.q, w.m1, w.m2, w.r, path)
    assert 0 < need <= native.KRON_NOALLOC_SCRATCH_BYTES
    d = {k: v.cuda() for k, v in kw.inputs(w).items()}
    ref = native.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path)
    first = _noalloc(d, w, path)
    second = _noalloc(d, w, path)      # the shared scratch keeps the first call's contents
    torch.cuda.synchronize()
    for k in ref:
        assert torch.equal(first[k], ref[k]), k
        assert torch.equal(second[k], ref[k]), k


def test_noalloc_rejects_oversized_problem():
    # 20000 rows of the 8x8-block, rank-8 layer need ~78 MB of scratch: refused up front
    w = kw.get("sweep_m8_r8")
    lib = native.load()
    need = native.workspace_size(w.N, w.p, w.q, w.m1, w.m2, w.r, "f32")
    assert need > native.KRON_NOALLOC_SCRATCH_BYTES
    dev = torch.device("cuda", 0)
    x = torch.zeros(w.N, w.d_in, device=dev)
    G = torch.zeros(w.N, w.d_out, device=dev)
    S = torch.ones(w.p, w.q, device=dev)
    A = torch.zeros(w.r, w.p, w.q, device=dev)
    B = torch.zeros(w.r, w.m1, w.m2, device=dev)
    outs = [torch.empty_like(t) for t in (x, S, A, B)]
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.kron_linear_backward_noalloc(P(x), P(S), P(A), P(B), P(G), P(outs[0]), P(outs[1]),
                                          P(outs[2]), P(outs[3]), None, w.N, w.p, w.q, w.m1,
                                          w.m2, w.r, native.KRON_F32, 0, None)
    assert native.STATUS[st] == "KRON_ERR_WORKSPACE"
    assert "fixed scratch" in lib.kron_last_error().decode()
