"""Training-step benchmark of the page "kronecker-layer-benchmark" (section "Setup") on one GPU.

The network is the page's 3-layer MLP 1024 -> 1024 -> 1024 -> 10 with ReLU. Its two hidden
layers are `KronLinear` layers, run by the library's kernels. The 10-way head is a dense
`nn.Linear`.

One step is:
- forward;
- cross-entropy plus the penalty lambda * sum|S| over both Kronecker layers;
- backward;
- an Adam update.

The penalty's gradient takes one of two routes: autograd through |S| (the page's form), or,
for the model `kron_fused_l1`, the library's backward, which adds lambda * sign(S) where it
writes dS (the penalty then enters the loss as a value only).

Inputs and labels are random, seeded, and resident on the device.

For context, the same step is timed for the page's dense baselines: three `nn.Linear`, with
and without the group-LASSO penalty over m x m blocks. Those run torch/cuBLAS and are not
part of the library.

    python -m kronecker_factored_structured_b200.train_step [--path tf32|f32|bf16]
        [--batches 256,20000] [--block 32] [--rank 4] [--warmup 10] [--steps 100] [--graph]

Each configuration prints one JSON line with:
- `ms_per_step`: CUDA events around the timed steps, on the launching stream;
- `wall_ms_per_step`: host clock after a synchronize, as the page measures;
- `peak_mem_mb`: `torch.cuda.max_memory_allocated` during the timed steps.
"""
from __future__ import annotations

import argparse
import json
import time

import torch
from torch import nn

import kronecker_factored_structured_b200 as kfs


class KronMLP(nn.Module):
    """``fused_l1=lam``: the layers' backward adds lam * sign(S) to dS, and penalty()
    returns sum|S| without a gradient; the caller scales it by the same lam for the loss
    value it reports."""

    def __init__(self, d=1024, classes=10, block=32, rank=4, path="tf32", device="cuda",
                 fused_l1=None):
        super().__init__()
        lam = 0.0 if fused_l1 is None else float(fused_l1)
        self.fused_l1 = fused_l1
        self.l1 = kfs.KronLinear(d, d, block, rank=rank, dtype=path, device=device, l1=lam)
        self.l2 = kfs.KronLinear(d, d, block, rank=rank, dtype=path, device=device, l1=lam)
        self.head = nn.Linear(d, classes, device=device, dtype=kfs.native.io_dtype(path))

    def forward(self, x):
        return self.head(torch.relu(self.l2(torch.relu(self.l1(x)))))

    def penalty(self):
        pen = self.l1.S.float().abs().sum() + self.l2.S.float().abs().sum()
        return pen.detach() if self.fused_l1 is not None else pen


class DenseMLP(nn.Module):
    def __init__(self, d=1024, classes=10, block=32, group_lasso=False, dtype=torch.float32,
                 device="cuda"):
        super().__init__()
        self.l1 = nn.Linear(d, d, device=device, dtype=dtype)
        self.l2 = nn.Linear(d, d, device=device, dtype=dtype)
        self.head = nn.Linear(d, classes, device=device, dtype=dtype)
        self.block, self.group_lasso = block, group_lasso

    def forward(self, x):
        return self.head(torch.relu(self.l2(torch.relu(self.l1(x)))))

    def _blocks_norm(self, w):
        # sum over the m x m blocks of their Frobenius norms
        o, i = w.shape
        m = self.block
        blocks = w.float().view(o // m, m, i // m, m)
        return (blocks.square().sum(dim=(1, 3)) + 1e-12).sqrt().sum()

    def penalty(self):
        if not self.group_lasso:
            return None
        return self._blocks_norm(self.l1.weight) + self._blocks_norm(self.l2.weight)


_SIDE = None


def _side_stream():
    """The one side stream that every graph warm-up uses.  A new stream per model would
    give each its own cuBLAS workspace, kept for the life of the process, and every later
    model's peak memory would include the earlier ones'."""
    global _SIDE
    if _SIDE is None:
        _SIDE = torch.cuda.Stream()
    return _SIDE


def time_model(model, batch, d, classes, lam, warmup, steps, dtype, seed=0, graph=False,
               capturable=None):
    """Times `steps` training steps after `warmup` untimed ones.  With graph=True the whole
    step (forward, loss, backward, Adam) is captured once in a CUDA graph and replayed, so
    the host issues one launch per step instead of one per kernel.  Adam keeps its step
    count on the device (capturable) when graphed, or when asked to."""
    fused = getattr(model, "fused_l1", None)
    if fused is not None and fused != lam:
        raise ValueError(f"the model fuses the penalty weight {fused}, the step uses {lam}")
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(batch, d, device="cuda", generator=g).to(dtype)
    labels = torch.randint(0, classes, (batch,), device="cuda", generator=g)
    opt = torch.optim.Adam(model.parameters(), lr=1e-3,
                           capturable=graph if capturable is None else capturable)
    loss_fn = nn.CrossEntropyLoss()

    def step():
        opt.zero_grad(set_to_none=True)
        loss = loss_fn(model(x).float(), labels)
        pen = model.penalty()
        if pen is not None:
            loss = loss + lam * pen
        loss.backward()
        opt.step()
        return loss

    if graph:
        # warm-up on a side stream (as torch's whole-network capture requires), then capture
        side = _side_stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(max(3, warmup)):
                step()
        torch.cuda.current_stream().wait_stream(side)
        cg = torch.cuda.CUDAGraph()
        opt.zero_grad(set_to_none=True)
        with torch.cuda.graph(cg):
            static_loss = step()

        def step():   # noqa: F811 -- the replayed step
            cg.replay()
            return static_loss
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record(stream)
    for _ in range(steps):
        loss = step()
    b.record(stream)
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) * 1e3 / steps
    return {"ms_per_step": a.elapsed_time(b) / steps, "wall_ms_per_step": wall,
            "peak_mem_mb": torch.cuda.max_memory_allocated() / 2**20,
            "final_loss": float(loss.item())}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--path", default="tf32", choices=["tf32", "f32", "bf16"])
    ap.add_argument("--batches", default="256,20000")
    ap.add_argument("--block", type=int, default=32)
    ap.add_argument("--rank", type=int, default=4)
    ap.add_argument("--lam", type=float, default=1e-4, help="weight of the sparsity penalty")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--no-dense", action="store_true", help="skip the dense baselines")
    ap.add_argument("--models", default=None,
                    help="comma-separated models to time, in this order (default: kron, "
                         "kron_fused_l1, dense, dense_group_lasso; a name may repeat)")
    ap.add_argument("--graph", action="store_true",
                    help="capture each model's whole step in a CUDA graph and replay it")
    args = ap.parse_args(argv)
    kfs.native.load()
    d, classes = 1024, 10
    dtype = kfs.native.io_dtype(args.path)
    old_tf32 = torch.backends.cuda.matmul.allow_tf32
    # the dense baselines and the head use the same arithmetic as the Kronecker path
    torch.backends.cuda.matmul.allow_tf32 = args.path == "tf32"
    try:
        for batch in [int(v) for v in args.batches.split(",")]:
            # each model is built just before it is timed and released after, so neither
            # its time nor its peak memory includes another model's state
            make = {
                "kron": lambda: KronMLP(d, classes, args.block, args.rank, args.path),
                "kron_fused_l1": lambda: KronMLP(d, classes, args.block, args.rank, args.path,
                                                 fused_l1=args.lam),
                "dense": lambda: DenseMLP(d, classes, args.block, False, dtype),
                "dense_group_lasso": lambda: DenseMLP(d, classes, args.block, True, dtype),
            }
            names = (args.models.split(",") if args.models else
                     ["kron", "kron_fused_l1"] + ([] if args.no_dense else
                                                  ["dense", "dense_group_lasso"]))
            unknown = sorted(set(names) - set(make))
            if unknown:
                raise SystemExit(f"unknown model(s) {unknown}; choose from {sorted(make)}")
            for name in names:
                torch.manual_seed(0)
                model = make[name]()
                r = time_model(model, batch, d, classes, args.lam, args.warmup, args.steps, dtype,
                               graph=args.graph)
                line = {"benchmark": "mlp_train_step", "model": name, "batch": batch,
                        "path": args.path, "block": args.block, "rank": args.rank,
                        "cuda_graph": args.graph,
                        "warmup": args.warmup, "steps": args.steps, **r}
                print(json.dumps(line), flush=True)
                del model
                torch.cuda.empty_cache()
    finally:
        torch.backends.cuda.matmul.allow_tf32 = old_tf32
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
