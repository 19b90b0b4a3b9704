"""Run one seeded workload's forward + backward through the library a few times, then
print one timed step (CUDA events).  A small driver for profilers (one kernel per capture):

    python -m kronecker_factored_structured_b200.run_workload WORKLOAD N PATH FLAGS ITERS [fwd]

WORKLOAD is a name from kron_workloads (tutorial, gpt2_c_fc_r4, stress, sweep_m64_r2, ...),
N the number of rows, PATH f32 | tf32 | bf16, FLAGS the flag bits (1 = skip zero blocks),
ITERS the untimed steps before the timed one; `fwd` runs the forward only.  A
Kronecker-sparse workload (ks_monarch_tr, ks_gpt2m_up, ...) runs the KS factor's calls
(PATH f32, FLAGS 0)."""
from __future__ import annotations

import dataclasses
import os
import sys


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import torch

    import kron_workloads as kw
    import kronecker_factored_structured_b200 as kfs
    name, N, path, flags, iters = argv[0], int(argv[1]), argv[2], int(argv[3]), int(argv[4])
    fwd_only = len(argv) > 5 and argv[5] == "fwd"
    if name.startswith("ks_"):
        return _run_ks(kw, kfs, torch, name, N, iters, fwd_only)
    w = kw.get(name).with_rows(N)
    if path == "bf16":
        w = dataclasses.replace(w, dtype="bf16")
    t = kfs.native.io_dtype(path)
    d = {k: v.to(t).cuda() for k, v in kw.inputs(w).items()}
    def backward():
        if not fwd_only:
            kfs.backward(d["x"], d["S"], d["A"], d["B"], d["G"], dtype=path, flags=flags)
    for _ in range(iters):
        kfs.forward(d["x"], d["S"], d["A"], d["B"], d["bias"], dtype=path, flags=flags)
        backward()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    kfs.forward(d["x"], d["S"], d["A"], d["B"], d["bias"], dtype=path, flags=flags)
    ev[1].record()
    backward()
    ev[2].record()
    torch.cuda.synchronize()
    print(f"{name} N={N} {path} flags={flags}: forward {ev[0].elapsed_time(ev[1]) * 1e3:.1f} us, "
          f"backward {ev[1].elapsed_time(ev[2]) * 1e3:.1f} us")
    return 0


def _run_ks(kw, kfs, torch, name, N, iters, fwd_only):
    w = kw.ks_get(name).with_rows(N)
    d = {k: v.cuda() for k, v in kw.ks_inputs(w).items()}
    nat = kfs.native
    def backward():
        if not fwd_only:
            nat.ks_backward(d["x"], d["w"], d["G"])
    for _ in range(iters):
        nat.ks_forward(d["x"], d["w"], d["bias"])
        backward()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    nat.ks_forward(d["x"], d["w"], d["bias"])
    ev[1].record()
    backward()
    ev[2].record()
    torch.cuda.synchronize()
    print(f"{name} N={N} pattern={w.pattern} f32: forward {ev[0].elapsed_time(ev[1]) * 1e3:.1f} us, "
          f"backward {ev[1].elapsed_time(ev[2]) * 1e3:.1f} us")
    return 0


if __name__ == "__main__":
    sys.exit(main())
