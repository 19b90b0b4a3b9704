"""The seeded input generator (no GPU): the readings it implements are checked here.

- "x% of S zeroed at random": exactly round(x * p * q) distinct entries; the stress case
  zeroes exactly 58 of its 64 8x8 patches and leaves the rest at 1.
- "N(0, v)": the second argument is the variance for the tutorial-like configurations
  (A ~ randn / sqrt(p), B ~ randn / sqrt(m) as the page "kronecker-layer-benchmark" initialises
  KronLinear) and a standard deviation of 0.02 for the GPT-2 shapes.
- Rows are drawn in chunks with their own generators, so any row range re-draws to the same
  values as the whole tensor.
"""
import math

import pytest
import torch

import kron_workloads as kw


@pytest.mark.parametrize("name,zeros", [("tiny", 16), ("tutorial", 512), ("sweep_m16_r2", 0),
                                        ("gpt2_c_fc_r4", 0), ("gpt2_c_proj_r1", 0)])
def test_exact_number_of_zero_entries_in_S(name, zeros):
    S = kw.factors(kw.get(name))["S"].float()
    assert int((S == 0).sum()) == zeros
    assert torch.all((S == 0) | (S == 1))


def test_stress_S_zeroes_exactly_58_patches():
    w = kw.get("stress")
    S = kw.factors(w)["S"].float()
    patches = S.view(8, 8, 8, 8).permute(0, 2, 1, 3).reshape(64, 64)   # one row per 8x8 patch
    zero = (patches == 0).all(dim=1)
    one = (patches == 1).all(dim=1)
    assert int(zero.sum()) == 58 and int(one.sum()) == 6
    assert float((S == 0).float().mean()) == pytest.approx(58 / 64)


def test_factor_scales():
    f = kw.factors(kw.get("tutorial"))                       # p = 32, m = 32
    assert float(f["A"].std()) == pytest.approx(1 / math.sqrt(32), rel=0.05)
    assert float(f["B"].std()) == pytest.approx(1 / math.sqrt(32), rel=0.05)
    assert float(f["bias"].std()) == pytest.approx(0.1, rel=0.1)
    g = kw.factors(kw.get("gpt2_c_fc_r4"))
    assert g["A"].dtype == torch.bfloat16
    assert float(g["A"].float().std()) == pytest.approx(0.02, rel=0.05)
    assert float(g["B"].float().std()) == pytest.approx(0.02, rel=0.05)
    t = kw.factors(kw.get("tiny"))                           # N(0, 1/8): variance 1/8
    assert float(t["A"].var()) == pytest.approx(1 / 8, rel=0.3)


def test_rows_redraw_any_range_identically():
    w = kw.get("tutorial").with_rows(9000)                   # three generator chunks
    x = kw.rows(w, "x")
    assert x.shape == (9000, 1024) and x.dtype == torch.float32
    a, b = kw.ROW_CHUNK - 5, 2 * kw.ROW_CHUNK + 7            # spans a whole chunk and two edges
    assert torch.equal(kw.rows(w, "x", a, b), x[a:b])
    idx = torch.tensor([8999, 0, kw.ROW_CHUNK, 17, kw.ROW_CHUNK - 1])
    assert torch.equal(kw.rows_at(w, "x", idx), x[idx])
    assert kw.rows(w, "G", 5, 5).shape == (0, 1024)
    assert float(x.std()) == pytest.approx(1.0, rel=0.01)


def test_same_seed_same_bytes_and_row_count_does_not_change_factors():
    w = kw.get("tiny")
    f1, f2 = kw.factors(w), kw.factors(w.with_rows(7))
    for k in f1:
        assert torch.equal(f1[k], f2[k]), k
    assert torch.equal(kw.rows(w, "G"), kw.rows(w, "G"))
    other = kw.custom(w.N, w.p, w.q, w.m1, w.m2, w.r, seed=w.seed + 1)
    assert not torch.equal(kw.factors(other)["A"], f1["A"])
    assert not torch.equal(kw.rows(w, "x"), kw.rows(w, "G")[:, : w.d_in])


def test_bf16_workloads_store_bf16():
    w = kw.get("gpt2_c_proj_r4").with_rows(3)
    d = kw.inputs(w)
    for k in ("x", "G", "S", "A", "B", "bias"):
        assert d[k].dtype == torch.bfloat16, k
    assert d["x"].shape == (3, 3072) and d["G"].shape == (3, 768)


def test_ks_workloads_shapes_and_draws():
    """KS workloads: widths from the pattern, values ~ randn/sqrt(b) in the [a][d][b][c] layout,
    seeded (the same bytes on every draw), and rows re-drawable chunk by chunk."""
    import math

    import kron_workloads as kw
    wl = kw.ks_get("ks_monarch_tr")
    a, b, c, d = wl.pattern
    assert (wl.d_in, wl.d_out) == (a * b * d, a * c * d) == (1024, 1024)
    f1, f2 = kw.ks_factors(wl), kw.ks_factors(wl)
    assert f1["w"].shape == (a, d, b, c) and f1["bias"].shape == (a * c * d,)
    assert torch.equal(f1["w"], f2["w"]) and torch.equal(f1["bias"], f2["bias"])
    assert abs(f1["w"].std().item() - 1 / math.sqrt(b)) < 0.02 / math.sqrt(b) * 10
    assert abs(f1["bias"].std().item() - wl.bias_std) < 0.02
    small = wl.with_rows(5000)
    full = kw.rows(small, "x")
    assert full.shape == (5000, 1024) and full.dtype == torch.float32
    idx = torch.tensor([4999, 0, 4096, 17])
    assert torch.equal(kw.rows_at(small, "x", idx), full[idx])
    assert torch.equal(kw.rows(small, "G", 4000, 4200), kw.rows(small, "G")[4000:4200])
    # every bench pattern is a valid factor
    for name, w in kw.ks_workloads().items():
        assert min(w.pattern) >= 1 and w.N > 0, name
