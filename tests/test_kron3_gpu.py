"""GPU parity of the triple Kronecker layer (kron3_linear_forward / _backward through the C
ABI) against the fp64 oracle's triple layer (page "LLM Compression via Kronecker Product
Decomposition", section "Triple Kronecker -- AxBxC (Extreme Compression)"): the exact-FP32
path on several shapes, and the tensor-core paths on shapes whose block kron(B_i, C_i) has a
tensor-core kernel (the tutorial layer's 32 x 32 blocks in TF32, the GPT-2 c_fc blocks of
32 x 64 in BF16)."""
import numpy as np
import pytest
import torch

import oracle
from kronecker_factored_structured_b200 import native
from parity import TOL, rel_err

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _case(seed, N, p, q, m1, m2, s1, s2, r, path):
    g = torch.Generator().manual_seed(seed)
    t = native.io_dtype(path)
    d = {"A": torch.randn(r, p, q, generator=g) / np.sqrt(p),
         "B": torch.randn(r, m1, m2, generator=g) / np.sqrt(m1),
         "C": torch.randn(r, s1, s2, generator=g) / np.sqrt(s1),
         "bias": 0.1 * torch.randn(q * m2 * s2, generator=g),
         "x": torch.randn(N, p * m1 * s1, generator=g),
         "G": torch.randn(N, q * m2 * s2, generator=g)}
    return {k: v.to(t) for k, v in d.items()}


def _check(d, path):
    dd = {k: v.to(DEV) for k, v in d.items()}
    y = native.forward3(dd["x"], dd["A"], dd["B"], dd["C"], dd["bias"], dtype=path)
    g = native.backward3(dd["x"], dd["A"], dd["B"], dd["C"], dd["G"], dtype=path)
    torch.cuda.synchronize()
    f = {k: v.double().numpy() for k, v in d.items()}
    ref = oracle.backward3(f["x"], f["A"], f["B"], f["C"], f["G"])
    ref["y"] = oracle.forward3(f["x"], f["A"], f["B"], f["C"], f["bias"])
    got = {"y": y, **g}
    errs = {k: rel_err(got[k].double().cpu().numpy(), ref[k]) for k in ref}
    bad = {k: e for k, e in errs.items() if not e <= TOL[path]}
    assert not bad, f"{path}: {bad} (all {errs})"
    return errs


@pytest.mark.parametrize("shape", [(37, 2, 3, 4, 4, 2, 2, 1), (64, 4, 4, 2, 3, 4, 4, 2),
                                   (129, 3, 5, 4, 8, 2, 1, 3)],
                         ids=lambda s: "N{}_A{}x{}_B{}x{}_C{}x{}_r{}".format(*s))
def test_kron3_f32(shape):
    _check(_case(sum(shape), *shape, "f32"), "f32")


def test_kron3_tf32_tutorial_blocks():
    """A 32 x 32, B 4 x 4, C 8 x 8, r = 4: blocks of 32 x 32, the tuned TF32 kernels."""
    _check(_case(3, 600, 32, 32, 4, 4, 8, 8, 4, "tf32"), "tf32")


def test_kron3_bf16_gpt2_blocks():
    """A 24 x 48, B 4 x 8, C 8 x 8, r = 4: the GPT-2 c_fc blocks (32 x 64), generic BF16."""
    _check(_case(4, 300, 24, 48, 4, 8, 8, 8, 4, "bf16"), "bf16")


def test_kron3_unsupported_block_is_refused():
    """A block shape without a tensor-core kernel is refused on the BF16 path."""
    d = {k: v.to(DEV) for k, v in _case(5, 16, 3, 5, 2, 2, 4, 4, 1, "bf16").items()}
    with pytest.raises(native.KronError, match="UNSUPPORTED"):
        native.forward3(d["x"], d["A"], d["B"], d["C"], d["bias"], dtype="bf16")
