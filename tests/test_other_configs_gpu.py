"""GPU parity on the configurations other than the tutorial layer: the block-size / rank
sweep, the GPT-2 small FFN shapes (page "LLM Compression via Kronecker Product
Decomposition", section "Factor Dimensions for GPT-2") and the 4096^2 block-sparse stress
case, on the exact-FP32 CUDA-core path (every tensor fp32; the BF16 workloads' inputs are
widened exactly from their bf16 values, which the oracle reads too).

At oracle-friendly sizes every output element is compared.  At the full sizes, y and dX are
compared on sampled rows (the oracle recomputes those rows from the same seeded
generators), dbias against an fp64 column sum of dY, and the parameter gradients on the
first 1024 rows."""
import functools

import numpy as np
import pytest
import torch

import kron_workloads as kw
import oracle
from parity import TOL, compare, gpu_run, oracle_run, rel_err, to_np

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def _inputs(w):
    return kw.inputs(w)


@functools.lru_cache(maxsize=None)
def _inputs_f32(w):
    """The workload's inputs as fp32 tensors (bf16 values widen exactly)."""
    return {k: v.float() for k, v in kw.inputs(w).items()}


@pytest.mark.parametrize("m", [8, 16, 64, 128])
@pytest.mark.parametrize("r", [1, 2, 8])
def test_sweep_shapes_f32(m, r):
    w = kw.get(f"sweep_m{m}_r{r}").with_rows(300)
    compare(gpu_run(_inputs(w), "f32"), oracle_run(_inputs(w)), "f32")


F32_FUZZ = [
    # N, p, q, m1, m2, r   (ragged N, rectangular factors)
    (1, 2, 3, 8, 16, 1),
    (37, 3, 5, 8, 8, 3),
    (129, 16, 8, 16, 8, 2),
    (77, 6, 12, 8, 16, 4),
]


@pytest.mark.parametrize("shape", F32_FUZZ, ids=lambda s: "N{}_p{}q{}_m{}x{}_r{}".format(*s))
def test_f32_shape_fuzz(shape):
    N, p, q, m1, m2, r = shape
    w = kw.custom(N, p, q, m1, m2, r, dtype="f32", seed=7 * N + p, s_zero_entries=(p * q) // 3)
    compare(gpu_run(_inputs(w), "f32"), oracle_run(_inputs(w)), "f32")


GPT2 = ["gpt2_c_fc_r1", "gpt2_c_fc_r4", "gpt2_c_proj_r1", "gpt2_c_proj_r4"]


@pytest.mark.parametrize("name", GPT2)
def test_gpt2_ffn_shapes_all_outputs_f32(name):
    w = kw.get(name).with_rows(300)
    compare(gpu_run(_inputs_f32(w), "f32"), oracle_run(_inputs(w)), "f32")


def _full_size_checks(w, path, sample_rows, grad_rows=1024):
    """Forward + backward at the workload's full N through the public API; y and dX on
    sampled rows, dbias against an fp64 column sum, parameter gradients on the first
    grad_rows rows (both sides on exactly those rows)."""
    import kronecker_factored_structured_b200 as kfs
    dev = torch.device("cuda", 0)
    fac = {k: v.to(dev) for k, v in kw.factors(w).items()}
    x = kw.rows(w, "x")
    G = kw.rows(w, "G")
    if path == "f32":
        fac = {k: v.float() for k, v in fac.items()}
        x, G = x.float(), G.float()
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
    got_y = to_np(y[idx.to(dev)])
    got_dx = to_np(g["dX"][idx.to(dev)])
    errs = {"y": rel_err(got_y, ref_y), "dX": rel_err(got_dx, ref_dx)}
    # dbias = sum over rows of dY, in fp64 on the host
    errs["dbias"] = rel_err(to_np(g["dbias"]), G.double().sum(dim=0).numpy())
    del xd, Gd, y, g
    torch.cuda.empty_cache()
    # parameter gradients on the first grad_rows rows, both sides
    wg = w.with_rows(grad_rows)
    got = gpu_run(_inputs_f32(wg) if path == "f32" else _inputs(wg), path)
    ref = oracle_run(_inputs(wg))
    for k in ("dS", "dA", "dB", "dbias"):
        errs[k + f"@N{grad_rows}"] = rel_err(got[k], ref[k])
    bad = {k: e for k, e in errs.items() if not e <= TOL[path]}
    assert not bad, f"{w.name}: relative errors above {TOL[path]}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("name", GPT2)
def test_gpt2_ffn_full_size_f32(name):
    w = kw.get(name)
    rng = np.random.default_rng(4)
    rows = sorted({0, w.N - 1, *rng.integers(0, w.N, 62).tolist()})
    print(name, _full_size_checks(w, "f32", rows))


def test_stress_small_all_outputs_f32():
    """4096^2, m = 64, r = 8, 58 of 64 8x8 patches of S zeroed, 40 rows, every output."""
    w = kw.get("stress").with_rows(40)
    compare(gpu_run(_inputs_f32(w), "f32"), oracle_run(_inputs(w)), "f32")


def test_skip_flag_on_block_sparse_s_f32():
    """KRON_FLAG_SKIP_ZERO_BLOCKS on the block-sparse stress pattern: the flagged CUDA-core
    path against the oracle, and bit for bit the unflagged results (only provably-zero
    work may be skipped, in the same accumulation order)."""
    w = kw.get("stress").with_rows(24)
    a = gpu_run(_inputs_f32(w), "f32", flags=1)
    compare(a, oracle_run(_inputs(w)), "f32")
    b = gpu_run(_inputs_f32(w), "f32", flags=0)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
