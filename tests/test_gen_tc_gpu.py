"""GPU parity of the generic tensor-core kernels against the fp64 oracle: the GPT-2 small
FFN shapes (page "LLM Compression via Kronecker Product Decomposition", section "Factor
Dimensions for GPT-2") and the 4096^2 block-sparse stress layer on the BF16 path, and the
block-size sweep's 64 x 64 and 128 x 128 blocks on the TF32 forward.

At oracle-friendly sizes every output element is compared; the row counts are ragged and
span several tiles and (for the backward) several row ranges.  At the full sizes y and dX
are compared on sampled rows, dbias against an fp64 column sum of dY, and the parameter
gradients on the first 1024 rows."""
import functools

import numpy as np
import pytest
import torch

import kron_workloads as kw
import oracle
from parity import TOL, compare, gpu_run, oracle_run, rel_err, to_np

pytestmark = pytest.mark.gpu

GPT2 = ["gpt2_c_fc_r1", "gpt2_c_fc_r4", "gpt2_c_proj_r1", "gpt2_c_proj_r4"]


@functools.lru_cache(maxsize=None)
def _inputs(w):
    return kw.inputs(w)


@functools.lru_cache(maxsize=None)
def _oracle(w):
    return oracle_run(_inputs(w))


@pytest.mark.parametrize("N", [1, 37, 300])
@pytest.mark.parametrize("name", GPT2)
def test_gpt2_ffn_bf16_all_outputs(name, N):
    w = kw.get(name).with_rows(N)
    compare(gpu_run(_inputs(w), "bf16"), _oracle(w), "bf16")


@pytest.mark.parametrize("name", GPT2)
def test_gpt2_ffn_bf16_no_bias(name):
    w = kw.get(name).with_rows(129)
    got = gpu_run(_inputs(w), "bf16", with_bias=False)
    compare(got, oracle_run(_inputs(w), with_bias=False), "bf16")


def _full_size_checks(w, path, sample_rows, grad_rows=1024):
    """Forward + backward at the workload's full N through the public API; y and dX on
    sampled rows, dbias against an fp64 column sum, parameter gradients on the first
    grad_rows rows (both sides on exactly those rows)."""
    import kronecker_factored_structured_b200 as kfs
    dev = torch.device("cuda", 0)
    fac = {k: v.to(dev) for k, v in kw.factors(w).items()}
    x = kw.rows(w, "x")
    G = kw.rows(w, "G")
    xd, Gd = x.to(dev), G.to(dev)
    y = kfs.forward(xd, fac["S"], fac["A"], fac["B"], fac["bias"], dtype=path)
    g = kfs.backward(xd, fac["S"], fac["A"], fac["B"], Gd, dtype=path)
    torch.cuda.synchronize()
    idx = torch.as_tensor(sample_rows, dtype=torch.long)
    f = {k: to_np(v) for k, v in kw.factors(w).items()}
    xs = to_np(kw.rows_at(w, "x", idx))
    Gs = to_np(kw.rows_at(w, "G", idx))
    ref_y = oracle.forward(xs, f["S"], f["A"], f["B"], f["bias"])
    ref_dx = oracle.backward(xs, f["S"], f["A"], f["B"], Gs)["dX"]
    errs = {"y": rel_err(to_np(y[idx.to(dev)]), ref_y),
            "dX": rel_err(to_np(g["dX"][idx.to(dev)]), ref_dx),
            "dbias": rel_err(to_np(g["dbias"]), G.double().sum(dim=0).numpy())}
    del xd, Gd, y, g, x, G
    torch.cuda.empty_cache()
    wg = w.with_rows(grad_rows)
    got = gpu_run(_inputs(wg), path)
    ref = _oracle(wg)
    for k in ("dS", "dA", "dB", "dbias"):
        errs[k + f"@N{grad_rows}"] = rel_err(got[k], ref[k])
    bad = {k: e for k, e in errs.items() if not e <= TOL[path]}
    assert not bad, f"{w.name}: relative errors above {TOL[path]}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("name", GPT2)
def test_gpt2_ffn_bf16_full_size(name):
    w = kw.get(name)
    rng = np.random.default_rng(4)
    rows = sorted({0, w.N - 1, *rng.integers(0, w.N, 62).tolist()})
    print(name, _full_size_checks(w, "bf16", rows))


@pytest.mark.parametrize("flags", [0, 1])
def test_stress_bf16_all_outputs(flags):
    """4096^2, m = 64, r = 8, 58 of 64 8x8 patches of S zeroed: 40 rows (20 tiles, the
    rank groups' CTAs of every row range), every output, with and without the zero-block
    skip."""
    w = kw.get("stress").with_rows(40)
    compare(gpu_run(_inputs(w), "bf16", flags=flags), _oracle(w), "bf16")


def test_stress_skip_is_bitwise_the_dense_result():
    """The skip drops only MMAs whose C' block is all zero, in the same K order, so the
    flagged results equal the unflagged ones bit for bit (finite inputs)."""
    w = kw.get("stress").with_rows(300)
    a = gpu_run(_inputs(w), "bf16", flags=1)
    b = gpu_run(_inputs(w), "bf16", flags=0)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_stress_bf16_full_size_sampled():
    """The stress case at N = 262144 rows with the skip flag (the configuration it exists
    for): y and dX on 24 sampled rows, dbias in full, parameter gradients at N = 1024."""
    w = kw.get("stress")
    rng = np.random.default_rng(5)
    rows = sorted({0, w.N - 1, *rng.integers(0, w.N, 22).tolist()})
    print(_full_size_checks(w, "bf16", rows))


@pytest.mark.parametrize("name", GPT2 + ["stress"])
def test_generic_backward_deterministic(name):
    import kronecker_factored_structured_b200 as kfs
    w = kw.get(name).with_rows(2000 if name != "stress" else 500)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    runs = [kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype="bf16") for _ in range(3)]
    torch.cuda.synchronize()
    for k in runs[0]:
        for r in runs[1:]:
            assert torch.equal(runs[0][k], r[k]), k


SWEEP_TC = [(64, 1), (64, 2), (64, 8), (128, 1), (128, 2)]


@pytest.mark.parametrize("m,r", SWEEP_TC)
def test_sweep_tf32_forward(m, r):
    """TF32 forward of the sweep's 64 x 64 and 128 x 128 blocks against the oracle."""
    import kronecker_factored_structured_b200 as kfs
    w = kw.get(f"sweep_m{m}_r{r}").with_rows(301)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    y = kfs.forward(d["x"], d["S"], d["A"], d["B"], d["bias"], dtype="tf32")
    torch.cuda.synchronize()
    assert rel_err(to_np(y), _oracle(w)["y"]) <= TOL["tf32"]


@pytest.mark.parametrize("m,r", SWEEP_TC)
def test_sweep_tf32_backward_is_refused(m, r):
    """No TF32 parameter-gradient kernel exists for these blocks: the backward returns
    KRON_ERR_UNSUPPORTED rather than running another path."""
    import kronecker_factored_structured_b200 as kfs
    w = kw.get(f"sweep_m{m}_r{r}").with_rows(64)
    d = {k: v.cuda() for k, v in _inputs(w).items()}
    with pytest.raises(kfs.KronError, match="UNSUPPORTED"):
        kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype="tf32")
