"""Data-parallel plumbing for the Kronecker layer (and the Kronecker-sparse factor): row sharding
and the one gradient exchange.

Rows are independent (page "kronecker-layer-benchmark", section "Setup": a batch is just rows
fed to the layer), so N rows split into contiguous per-rank ranges and the forward needs no
communication.  The backward's only exchange is the sum over ranks of the parameter gradients
dS, dA, dB and dbias; they live as views of one flat fp32 buffer so that a single all-reduce
moves them all (dX stays sharded like x).
"""
from __future__ import annotations

from typing import Dict, Tuple

import torch


def shard_rows(n_rows: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous row range (start, count) of `rank`: the first n_rows % world ranks take one
    extra row; every row belongs to exactly one rank."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if n_rows < 0:
        raise ValueError("n_rows must be non-negative")
    base, extra = divmod(n_rows, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def param_grad_sizes(p: int, q: int, m1: int, m2: int, r: int) -> Dict[str, tuple]:
    """Shapes of the parameter gradients, in the order they sit in the flat buffer."""
    return {"dS": (p, q), "dA": (r, p, q), "dB": (r, m1, m2), "dbias": (q * m2,)}


def ks_param_grad_sizes(a: int, b: int, c: int, d: int) -> Dict[str, tuple]:
    """Shapes of a Kronecker-sparse factor's parameter gradients (pattern (a, b, c, d))."""
    return {"dw": (a, d, b, c), "dbias": (a * c * d,)}


def flat_grad_buffer(p: int, q: int, m1: int, m2: int, r: int,
                     device="cpu") -> Tuple[torch.Tensor, Dict[str, torch.Tensor]]:
    """One fp32 buffer holding dS, dA, dB, dbias back to back, and a view of it per gradient
    (the layout the backward call writes into through `grads=`)."""
    return flat_buffer(param_grad_sizes(p, q, m1, m2, r), device)


def ks_flat_grad_buffer(a: int, b: int, c: int, d: int,
                        device="cpu") -> Tuple[torch.Tensor, Dict[str, torch.Tensor]]:
    """The same for a Kronecker-sparse factor: dw and dbias as views of one buffer, so its
    data-parallel backward also exchanges one all-reduce per step."""
    return flat_buffer(ks_param_grad_sizes(a, b, c, d), device)


def flat_buffer(shapes: Dict[str, tuple],
                device="cpu") -> Tuple[torch.Tensor, Dict[str, torch.Tensor]]:
    """One zeroed fp32 buffer and a view of it per named shape, back to back in dict order."""
    total = sum(int(torch.Size(s).numel()) for s in shapes.values())
    flat = torch.zeros(total, dtype=torch.float32, device=device)
    views, o = {}, 0
    for k, s in shapes.items():
        n = int(torch.Size(s).numel())
        views[k] = flat[o:o + n].view(*s)
        o += n
    return flat, views


def allreduce_grads(flat: torch.Tensor, group=None, deterministic: bool = False,
                    gathered: torch.Tensor = None) -> torch.Tensor:
    """Sum the flat parameter-gradient buffer over the ranks of `group` (in place).

    Default: one NCCL (or gloo) all-reduce.  Its summation order is the library's choice
    (ring or tree, and on NVSwitch possibly in the switch), so the sum over ranks is not
    bitwise reproducible across world sizes or runs.

    deterministic=True: every rank all-gathers the ranks' buffers and adds them in rank
    order, rank 0 first, so every rank gets bitwise the same sum in every run with the same
    world size (the per-rank gradients are themselves bitwise reproducible).  It moves
    world-1 buffers to each rank instead of about two: for the tutorial layer's 40 KB of
    gradients that is latency, not bandwidth.  `gathered` may hold a preallocated buffer of
    world * numel elements."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return flat
    world = dist.get_world_size(group)
    if world <= 1:
        return flat
    if not deterministic:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
        return flat
    n = flat.numel()
    if gathered is None:
        gathered = torch.empty(world * n, dtype=flat.dtype, device=flat.device)
    dist.all_gather_into_tensor(gathered, flat.contiguous(), group=group)
    flat.copy_(gathered[:n])
    for r in range(1, world):
        flat.add_(gathered[r * n:(r + 1) * n])
    return flat
