"""Seeded synthetic workloads for the Kronecker layer (shared by tests, bench, smoke).

This module holds shapes, distributions and random draws only -- none of the
layer's arithmetic -- so that both the fp64 oracle and the CUDA library can be
fed the very same bytes without depending on each other.

Shapes and distributions follow the page "kronecker-layer-benchmark"
(section "Setup": rows = images x tokens, 1024 x 1024 hidden layers, block size
m and rank r; section "1. Build W, then multiply": S = ones, A_i ~ randn/sqrt(p),
B_i ~ randn/sqrt(m), bias zeros) and the GPT-2 small FFN shapes of the page
"LLM Compression via Kronecker Product Decomposition" (section "Factor
Dimensions for GPT-2", c_fc 768->3072 and c_proj 3072->768).

The Kronecker-sparse factors (page "Fast Inference with Kronecker-Sparse
Matrices": supports kron(I_a, kron(1_{b x c}, I_d)), the factors of Monarch and
butterfly matrices; the page reports FP32 runs and end-to-end ViT-S/16 and GPT-2
medium models) get ``KSWorkload`` entries: the two factors of a 1024 x 1024
Monarch matrix and one radix-2 butterfly factor on the tutorial's 20000 rows, a
1024 -> 4096 factor at GPT-2 medium's width on 8 x 1024 tokens, and a factor of
large 128 x 128 blocks.  Values ~ randn/sqrt(b) (each output sums b inputs).

Large row tensors are drawn in fixed chunks of rows, each chunk from its own
generator seeded by (seed, tensor tag, chunk index), so any subset of rows can
be re-drawn on the CPU without materialising the whole tensor.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

ROW_CHUNK = 4096  # rows drawn per generator chunk

_TAGS = {"x": 11, "G": 13}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    p: int
    q: int
    m1: int
    m2: int
    r: int
    dtype: str            # "f32" (exact FP32 and TF32 paths) or "bf16"
    seed: int
    x_std: float = 1.0
    g_std: float = 1.0
    a_std: Optional[float] = None   # default 1/sqrt(p)
    b_std: Optional[float] = None   # default 1/sqrt(m1)
    bias_std: float = 0.1
    s_zero_entries: int = 0         # exactly this many distinct zero entries of S
    s_zero_patch: int = 0           # patch edge for patch-wise zeroing (0: element-wise)
    s_zero_patches: int = 0         # exactly this many zero patches

    @property
    def d_in(self) -> int:
        return self.p * self.m1

    @property
    def d_out(self) -> int:
        return self.q * self.m2

    def with_rows(self, N: int) -> "Workload":
        return dataclasses.replace(self, N=N, name=f"{self.name}@N{N}")


def _tutorial_like(name, N, m, r, seed, s_zero_frac):
    p = 1024 // m
    return Workload(name=name, N=N, p=p, q=p, m1=m, m2=m, r=r, dtype="f32", seed=seed,
                    a_std=math.sqrt(1.0 / p), b_std=math.sqrt(1.0 / m),
                    bias_std=0.1, s_zero_entries=int(round(s_zero_frac * p * p)))


def all_workloads() -> dict:
    w = {}
    # tiny oracle-scale case: in=out=64, 8x8 blocks, rank 2, 25% of S zeroed
    w["tiny"] = Workload(name="tiny", N=64, p=8, q=8, m1=8, m2=8, r=2, dtype="f32", seed=1,
                         a_std=math.sqrt(1 / 8), b_std=math.sqrt(1 / 8), bias_std=0.1,
                         s_zero_entries=16)
    # the tutorial layer: 20000 rows (~100 images x 197 tokens), 1024^2, m=32, r=4, 50% of S zeroed
    w["tutorial"] = _tutorial_like("tutorial", 20000, 32, 4, 2, 0.5)
    # block-size / rank sweep on 1024^2, S all ones
    for m in (8, 16, 64, 128):
        for r in (1, 2, 8):
            w[f"sweep_m{m}_r{r}"] = _tutorial_like(f"sweep_m{m}_r{r}", 20000, m, r, 3, 0.0)
    # GPT-2 small FFN shapes, bf16, factors ~ N(0, 0.02) read as std 0.02
    for r in (1, 4):
        w[f"gpt2_c_fc_r{r}"] = Workload(name=f"gpt2_c_fc_r{r}", N=8192, p=24, q=48, m1=32, m2=64,
                                        r=r, dtype="bf16", seed=4, x_std=0.02, a_std=0.02,
                                        b_std=0.02, bias_std=0.02)
        w[f"gpt2_c_proj_r{r}"] = Workload(name=f"gpt2_c_proj_r{r}", N=8192, p=48, q=24, m1=64,
                                          m2=32, r=r, dtype="bf16", seed=4, x_std=0.02,
                                          a_std=0.02, b_std=0.02, bias_std=0.02)
    # large stress case: 4096^2, m=64, r=8, bf16, 58 of 64 8x8 patches of S zeroed
    w["stress"] = Workload(name="stress", N=262144, p=64, q=64, m1=64, m2=64, r=8, dtype="bf16",
                           seed=5, a_std=1 / 8, b_std=1 / 8, bias_std=0.1,
                           s_zero_patch=8, s_zero_patches=58)
    return w


def get(name: str) -> Workload:
    return all_workloads()[name]


@dataclasses.dataclass(frozen=True)
class KSWorkload:
    """One Kronecker-sparse factor of pattern (a, b, c, d): x [N][a*b*d] -> y [N][a*c*d]."""
    name: str
    N: int
    a: int
    b: int
    c: int
    d: int
    seed: int
    dtype: str = "f32"
    x_std: float = 1.0
    g_std: float = 1.0
    bias_std: float = 0.1

    @property
    def pattern(self):
        return (self.a, self.b, self.c, self.d)

    @property
    def d_in(self) -> int:
        return self.a * self.b * self.d

    @property
    def d_out(self) -> int:
        return self.a * self.c * self.d

    def with_rows(self, N: int) -> "KSWorkload":
        return dataclasses.replace(self, N=N, name=f"{self.name}@N{N}")


def ks_workloads() -> dict:
    w = {}
    for name, N, pat in (("ks_monarch_bd", 20000, (32, 32, 32, 1)),
                         ("ks_monarch_tr", 20000, (1, 32, 32, 32)),
                         ("ks_butterfly", 20000, (16, 2, 2, 32)),
                         ("ks_gpt2m_up", 8192, (1, 32, 128, 32)),
                         ("ks_block128", 20000, (8, 128, 128, 1))):
        w[name] = KSWorkload(name=name, N=N, a=pat[0], b=pat[1], c=pat[2], d=pat[3], seed=6)
    return w


def ks_get(name: str) -> KSWorkload:
    return ks_workloads()[name]


def ks_custom(N, a, b, c, d, seed=0) -> KSWorkload:
    return KSWorkload(name=f"ks_N{N}_{a}x{b}x{c}x{d}", N=N, a=a, b=b, c=c, d=d, seed=seed)


def ks_factors(w: KSWorkload) -> dict:
    """Values w [a][d][b][c] ~ randn/sqrt(b) and bias ~ N(0, bias_std^2) (CPU float32)."""
    g = _gen(w.seed, 2, w.a, w.b, w.c, w.d)
    vals = torch.randn(w.a, w.d, w.b, w.c, generator=g) / math.sqrt(w.b)
    bias = torch.randn(w.d_out, generator=g) * w.bias_std
    return {"w": vals, "bias": bias}


def ks_inputs(w: KSWorkload) -> dict:
    d = ks_factors(w)
    d["x"] = rows(w, "x")
    d["G"] = rows(w, "G")
    return d


def custom(N, p, q, m1, m2, r, dtype="f32", seed=0, s_zero_entries=0, **kw) -> Workload:
    """An ad-hoc workload (shape fuzzing); default init as in the tutorial layer."""
    return Workload(name=f"custom_N{N}_p{p}q{q}_m{m1}x{m2}_r{r}_{dtype}", N=N, p=p, q=q, m1=m1,
                    m2=m2, r=r, dtype=dtype, seed=seed, s_zero_entries=s_zero_entries, **kw)


def _gen(*key) -> torch.Generator:
    g = torch.Generator(device="cpu")
    s = 0
    for k in key:
        s = (s * 1000003 + int(k)) % (2 ** 62)
    g.manual_seed(s)
    return g


def _storage_dtype(w: Workload) -> torch.dtype:
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def factors(w: Workload) -> dict:
    """S, A, B and bias (CPU tensors in the workload's storage dtype)."""
    g = _gen(w.seed, 1)
    S = torch.ones(w.p, w.q)
    if w.s_zero_entries:
        idx = torch.randperm(w.p * w.q, generator=g)[: w.s_zero_entries]
        S.view(-1)[idx] = 0.0
    if w.s_zero_patches:
        P = w.s_zero_patch
        npr, npc = w.p // P, w.q // P
        idx = torch.randperm(npr * npc, generator=g)[: w.s_zero_patches]
        for t in idx.tolist():
            br, bc = divmod(t, npc)
            S[br * P:(br + 1) * P, bc * P:(bc + 1) * P] = 0.0
    a_std = w.a_std if w.a_std is not None else 1.0 / math.sqrt(w.p)
    b_std = w.b_std if w.b_std is not None else 1.0 / math.sqrt(w.m1)
    A = torch.randn(w.r, w.p, w.q, generator=g) * a_std
    B = torch.randn(w.r, w.m1, w.m2, generator=g) * b_std
    bias = torch.randn(w.q * w.m2, generator=g) * w.bias_std
    dt = _storage_dtype(w)
    return {"S": S.to(dt), "A": A.to(dt), "B": B.to(dt), "bias": bias.to(dt)}


def rows(w: Workload, tag: str, n0: int = 0, n1: Optional[int] = None) -> torch.Tensor:
    """Rows [n0, n1) of the input x (tag "x") or the upstream gradient G (tag "G")."""
    n1 = w.N if n1 is None else n1
    width = w.d_in if tag == "x" else w.d_out
    std = w.x_std if tag == "x" else w.g_std
    dt = _storage_dtype(w)
    out = torch.empty(max(n1 - n0, 0), width, dtype=dt)
    c0, c1 = n0 // ROW_CHUNK, (n1 - 1) // ROW_CHUNK if n1 > n0 else -1
    for c in range(c0, c1 + 1):
        lo, hi = c * ROW_CHUNK, min((c + 1) * ROW_CHUNK, w.N)
        chunk = torch.randn(hi - lo, width, generator=_gen(w.seed, _TAGS[tag], c)) * std
        a, b = max(lo, n0), min(hi, n1)
        out[a - n0:b - n0] = chunk[a - lo:b - lo].to(dt)
    return out


def rows_at(w: Workload, tag: str, index: torch.Tensor) -> torch.Tensor:
    """The rows listed in ``index`` (any order) of x or G, drawn chunk by chunk."""
    index = torch.as_tensor(index, dtype=torch.long)
    width = w.d_in if tag == "x" else w.d_out
    out = torch.empty(index.numel(), width, dtype=_storage_dtype(w))
    chunks = torch.unique(index // ROW_CHUNK).tolist()
    for c in chunks:
        lo, hi = c * ROW_CHUNK, min((c + 1) * ROW_CHUNK, w.N)
        block = rows(w, tag, lo, hi)
        sel = (index // ROW_CHUNK) == c
        out[sel] = block[index[sel] - lo]
    return out


def inputs(w: Workload) -> dict:
    """All inputs of one forward+backward: x, G and the factors (CPU tensors)."""
    d = factors(w)
    d["x"] = rows(w, "x")
    d["G"] = rows(w, "G")
    return d
