"""Work accounting pinned to figures the pages print (tests/golden/page_figures.txt)."""
import os

from kronecker_factored_structured_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.txt")


def _figures():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val, _src = [s.strip() for s in line.split("|", 2)]
        out[key] = val
    return out


def _range(s):
    lo, hi = s.split("..")
    return int(lo), int(hi)


def test_param_counts_match_page():
    f = _figures()
    lo, hi = _range(f["params_r1_m8_1024_approx"])
    assert lo <= acc.param_count(128, 128, 8, 8, 1) <= hi
    lo, hi = _range(f["params_dense_1024_approx"])
    assert lo <= acc.dense_param_count(1024, 1024) <= hi
    exceeds = acc.param_count(512, 512, 2, 2, 4) > acc.dense_param_count(1024, 1024)
    assert str(exceeds).lower() == f["params_r4_m2_exceeds_dense"]


def test_gpt2_factor_counts_match_page():
    f = _figures()
    # rank-1 Kronecker factors without S and bias, W = A kron B with A 48x12, B 64x64
    assert 48 * 64 * 12 * 64 == int(f["gpt2_c_fc_params_before"])
    assert acc.param_count(48, 12, 64, 64, 1, bias=False, with_s=False) == int(f["gpt2_c_fc_params_after"])


def test_mac_ratio_matches_page():
    f = _figures()
    ratio = acc.mac_ratio_vs_dense(128, 128, 8, 8, 1)
    assert round(100 * ratio) == int(f["mac_ratio_r1_m8_percent"])
    # "about r/m of a dense layer's multiply-adds" for square blocks
    for m, r in ((8, 1), (32, 4), (16, 2)):
        p = 1024 // m
        assert abs(acc.mac_ratio_vs_dense(p, p, m, m, r) - r / m) <= r / p + 1e-12


def test_tutorial_layer_work():
    # 1024^2, m = 32, r = 4: 1,572,864 flop and 20,480 bytes per row (fp32), fwd + bwd
    assert acc.flops_per_row(32, 32, 32, 32, 4) == 1572864
    assert acc.bytes_per_row(1024, 1024, 4) == 20480
    assert acc.flops_per_row(32, 32, 32, 32, 4, backward=False) * 3 == 1572864


def test_gpt2_ffn_work_takes_the_cheaper_order():
    # c_fc 768 -> 3072 (C 24 x 48, B 32 x 64): X.B first is cheaper, 49,152 + 73,728 MACs per
    # rank; c_proj 3072 -> 768 (C 48 x 24, B 64 x 32): C first, 73,728 + 49,152
    assert acc.macs_per_row_forward(24, 48, 32, 64, 1) == 122880
    assert acc.macs_per_row_forward(48, 24, 64, 32, 1) == 122880
    for r in (1, 4):
        assert acc.flops_per_row(24, 48, 32, 64, r) == 737280 * r
        assert acc.flops_per_row(48, 24, 64, 32, r, backward=False) == 245760 * r
    assert acc.bytes_per_row(768, 3072, 2) == 16896
    assert acc.bytes_per_row(3072, 768, 2) == 21504
    assert acc.bytes_per_row(768, 3072, 2, backward=False) == 7680


def test_stress_work_with_and_without_the_skip_credit():
    # 4096^2, m = 64, r = 8: 25,165,824 flop per row with S dense; with 6 of 64 patches
    # non-zero the two contractions with C (y and U) shrink to 6/64, dC does not
    assert acc.flops_per_row(64, 64, 64, 64, 8) == 25165824
    assert acc.flops_per_row(64, 64, 64, 64, 8, skip_fraction=1.0) == 25165824
    assert acc.flops_per_row(64, 64, 64, 64, 8, skip_fraction=6 / 64) == 17563648
    assert acc.bytes_per_row(4096, 4096, 2) == 40960


def test_sweep_work():
    # square blocks on the 1024^2 layer: 6144 * r * (m + p) flop per row, p = 1024 / m
    for m in (8, 16, 64, 128):
        for r in (1, 2, 8):
            p = 1024 // m
            assert acc.flops_per_row(p, p, m, m, r) == 6144 * r * (m + p)
    assert 20000 * acc.flops_per_row(128, 128, 8, 8, 1) == 16711680000


def test_ks_work_counts_the_support():
    """A KS factor's values, flops and density against the oracle's dense K (its non-zeros)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(5)
    for a, b, c, d in ((2, 3, 4, 5), (16, 2, 2, 32), (1, 8, 16, 4)):
        w = rng.uniform(0.5, 1.5, (a, d, b, c))
        nnz = int(np.count_nonzero(oracle.ks_dense(w)))
        assert acc.ks_param_count(a, b, c, d, bias=False) == nnz
        assert acc.ks_param_count(a, b, c, d) == nnz + a * c * d
        assert acc.ks_flops_per_row(a, b, c, d, backward=False) == 2 * nnz
        assert acc.ks_flops_per_row(a, b, c, d) == 6 * nnz
        # density 1 / (a d) of the dense (a b d) x (a c d) matrix
        assert nnz * a * d == (a * b * d) * (a * c * d)
