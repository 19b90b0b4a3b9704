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
