"""Plant plausible mistakes in a copy of the oracle's C source and check that the
pins catch every one of them (a dropped term, a wrong sign or index, a missing
factor).  The copies are compiled and run on the CPU only."""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "kron_oracle.c")

# (name, exact text in kron_oracle.c, replacement, occurrence index)
MUTATIONS = [
    ("weight_drops_S",
     "const double Cac = S[(long)a * q + c] * A[((long)i * p + a) * q + c];",
     "const double Cac = A[((long)i * p + a) * q + c];", 0),
    ("weight_row_interleave_swapped",
     "W[((long)a * m1 + j) * out + (long)c * m2 + k] +=",
     "W[((long)j * p + a) * out + (long)c * m2 + k] +=", 0),
    ("weight_col_interleave_swapped",
     "W[((long)a * m1 + j) * out + (long)c * m2 + k] +=",
     "W[((long)a * m1 + j) * out + (long)k * q + c] +=", 0),
    ("bias_dropped", "yn[o] = bias ? bias[o] : 0.0;", "yn[o] = 0.0;", 0),
    ("dx_wrong_sign", "s += Gn[o] * Wu[o];", "s -= Gn[o] * Wu[o];", 0),
    ("dw_reads_wrong_column", "const double xv = x[n * in + u];",
     "const double xv = x[n * in + (in - 1 - u)];", 0),
    ("dB_drops_S",
     "S[(long)a * q + c] * A[((long)i * p + a) * q + c];\n                        dB",
     "A[((long)i * p + a) * q + c];\n                        dB", 0),
    ("dA_forgets_S", "dA[(long)i * p * q + ac] = dC[(long)i * p * q + ac] * S[ac];",
     "dA[(long)i * p * q + ac] = dC[(long)i * p * q + ac];", 0),
    ("dS_uses_S_not_A", "s += dC[(long)i * p * q + ac] * A[(long)i * p * q + ac];",
     "s += dC[(long)i * p * q + ac] * S[ac];", 0),
    ("dbias_skips_first_row", "for (long n = 0; n < N; ++n) s += G[n * out + o];",
     "for (long n = 1; n < N; ++n) s += G[n * out + o];", 0),
    ("dC_uses_only_first_rank_of_B",
     "B[((long)i * m1 + j) * m2 + k];\n                    dC",
     "B[((long)0 * m1 + j) * m2 + k];\n                    dC", 0),
    ("l1_grad_wrong_sign", "out[ac] = v > 0.0 ? lam : (v < 0.0 ? -lam : 0.0);",
     "out[ac] = v > 0.0 ? -lam : (v < 0.0 ? lam : 0.0);", 0),
    ("l1_grad_nonzero_at_kink", "out[ac] = v > 0.0 ? lam : (v < 0.0 ? -lam : 0.0);",
     "out[ac] = v >= 0.0 ? lam : -lam;", 0),
    ("l1_grad_drops_weight", "out[ac] = v > 0.0 ? lam : (v < 0.0 ? -lam : 0.0);",
     "out[ac] = v > 0.0 ? 1.0 : (v < 0.0 ? -1.0 : 0.0);", 0),
    ("vanloan_rows_transposed",
     "Wt[((size_t)a * q + c) * ((size_t)m1 * m2) + (size_t)j * m2 + k] =",
     "Wt[((size_t)c * p + a) * ((size_t)m1 * m2) + (size_t)j * m2 + k] =", 0),
    ("vanloan_block_read_transposed",
     "W[((size_t)a * m1 + j) * ((size_t)q * m2) + (size_t)c * m2 + k];",
     "W[((size_t)a * m1 + j) * ((size_t)q * m2) + (size_t)k * q + c];", 0),
    ("vanloan_inner_index_swapped",
     "Wt[((size_t)a * q + c) * ((size_t)m1 * m2) + (size_t)j * m2 + k] =",
     "Wt[((size_t)a * q + c) * ((size_t)m1 * m2) + (size_t)k * m1 + j] =", 0),
    ("kron3_weight_swaps_inner_factors",
     "W[(((long)a * m1 + j) * s1 + u) * out + ((long)c * m2 + k) * s2 + v] +=\n                                    av * bv",
     "W[(((long)a * m1 + j) * s1 + u) * out + ((long)c * m2 + k) * s2 + v] +=\n                                    av * av", 0),
    ("kron3_dA_drops_C",
     "B[((long)i * m1 + j) * m2 + k] * C[((long)i * s1 + u) * s2 + v];\n                dA",
     "B[((long)i * m1 + j) * m2 + k];\n                dA", 0),
    ("kron3_dC_uses_B_twice",
     "A[((long)i * p + a) * q + c] * B[((long)i * m1 + j) * m2 + k];\n                dC",
     "B[((long)i * m1 + j) * m2 + k] * B[((long)i * m1 + j) * m2 + k];\n                dC", 0),
    ("ks_rows_in_wrong_interleave",
     "K[(((long)al * b + be) * d + de) * out + ((long)al * c + ga) * d + de] =",
     "K[(((long)al * d + de) * b + be) * out + ((long)al * c + ga) * d + de] =", 0),
    ("ks_cols_in_wrong_interleave",
     "K[(((long)al * b + be) * d + de) * out + ((long)al * c + ga) * d + de] =",
     "K[(((long)al * b + be) * d + de) * out + ((long)al * d + de) * c + ga] =", 0),
    ("ks_block_read_transposed",
     "w[(((long)al * d + de) * b + be) * c + ga];",
     "w[(((long)al * d + de) * c + ga) * b + be];", 0),
    ("ks_blocks_in_wrong_order",
     "w[(((long)al * d + de) * b + be) * c + ga];",
     "w[(((long)de * a + al) * b + be) * c + ga];", 0),
    ("ks_forward_drops_bias", "oracle_matmul_bias(x, K, bias, N, in, out, y);",
     "oracle_matmul_bias(x, K, NULL, N, in, out, y);", 0),
    ("ks_dx_wrong_sign", "s += G[n * out + o] * K[u * out + o];",
     "s -= G[n * out + o] * K[u * out + o];", 0),
    ("ks_dw_reads_mirrored_delta",
     "dK[(((long)al * b + be) * d + de) * out + ((long)al * c + ga) * d + de];",
     "dK[(((long)al * b + be) * d + de) * out + ((long)al * c + ga) * d + (d - 1 - de)];", 0),
    ("ks_dbias_skips_first_row", "for (long n = 0; n < N; ++n) s += G[n * out + o];",
     "for (long n = 1; n < N; ++n) s += G[n * out + o];", 2),
]


def _mutate(text, old, new, occ):
    pos = -1
    for _ in range(occ + 1):
        pos = text.index(old, pos + 1)
    return text[:pos] + new + text[pos + len(old):]


@pytest.mark.parametrize("name,old,new,occ", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(tmp_path, name, old, new, occ):
    text = open(SRC).read()
    assert old in text, f"mutation anchor for {name} not found in the oracle source"
    src = tmp_path / f"mut_{name}.c"
    src.write_text(_mutate(text, old, new, occ))
    so = oracle.build(force=True, src=str(src), out=str(tmp_path / f"mut_{name}.so"))
    orc = oracle.Oracle(so)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
