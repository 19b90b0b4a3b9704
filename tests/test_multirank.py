"""Host side of the data-parallel path on CPU ranks (gloo, world size 2).

The layer's only exchange is the sum over ranks of the parameter gradients (rows are
independent, page "kronecker-layer-benchmark", section "Setup").  Each rank takes its row
shard, computes the gradients of its rows with the fp64 oracle, writes them into the flat
buffer the backward call fills, and all-reduces; the result must equal the full-batch
gradients, and the row shards must tile the batch exactly.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_q, deterministic=False):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import kron_workloads as kw
    import oracle
    from kronecker_factored_structured_b200 import dp

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = kw.get("tiny")
        d = {k: v.double().numpy() for k, v in kw.inputs(w).items()}
        start, count = dp.shard_rows(w.N, world, rank)
        sl = slice(start, start + count)
        g = oracle.backward(d["x"][sl], d["S"], d["A"], d["B"], d["G"][sl])
        flat, views = dp.flat_grad_buffer(w.p, w.q, w.m1, w.m2, w.r)
        for k in ("dS", "dA", "dB", "dbias"):
            views[k].copy_(torch.from_numpy(g[k]).float())
        dp.allreduce_grads(flat, deterministic=deterministic)
        result_q.put((rank, start, count, {k: v.double().numpy().copy() for k, v in views.items()},
                      g["dX"]))
    finally:
        dist.destroy_process_group()


def test_shard_rows_tiles_the_batch():
    from kronecker_factored_structured_b200 import dp
    for n in (0, 1, 7, 64, 20000, 20001):
        for world in (1, 2, 3, 8):
            got = [dp.shard_rows(n, world, r) for r in range(world)]
            assert sum(c for _, c in got) == n
            pos = 0
            for s, c in got:
                assert s == pos and c >= 0
                pos += c
            assert max(c for _, c in got) - min(c for _, c in got) <= 1
    with pytest.raises(ValueError):
        dp.shard_rows(10, 2, 2)


def test_flat_buffer_views_cover_it_once():
    from kronecker_factored_structured_b200 import dp
    flat, views = dp.flat_grad_buffer(8, 6, 4, 5, 3)
    assert flat.numel() == 8 * 6 + 3 * 8 * 6 + 3 * 4 * 5 + 6 * 5
    for i, v in enumerate(views.values()):
        v.fill_(i + 1)
    assert torch.all(flat > 0)  # every element belongs to one view
    assert sorted(set(flat.tolist())) == [1.0, 2.0, 3.0, 4.0]


def _run_ranks(world, deterministic):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, deterministic))
             for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort(key=lambda t: t[0])
    return out


@pytest.mark.parametrize("world", [2, 3])
def test_deterministic_exchange_is_the_rank_ordered_sum(world):
    """deterministic=True: every rank holds bitwise the same sum, equal to adding the ranks'
    fp32 buffers in rank order on the host, and close to the full-batch gradients."""
    import kron_workloads as kw
    import oracle
    from kronecker_factored_structured_b200 import dp
    out = _run_ranks(world, True)
    w = kw.get("tiny")
    d = {k: v.double().numpy() for k, v in kw.inputs(w).items()}
    parts = []
    for rank in range(world):
        start, count = dp.shard_rows(w.N, world, rank)
        sl = slice(start, start + count)
        parts.append(oracle.backward(d["x"][sl], d["S"], d["A"], d["B"], d["G"][sl]))
    full = oracle.backward(d["x"], d["S"], d["A"], d["B"], d["G"])
    for k in ("dS", "dA", "dB", "dbias"):
        want = parts[0][k].astype(np.float32)
        for r in range(1, world):
            want = want + parts[r][k].astype(np.float32)
        for rank, _, _, grads, _ in out:
            assert np.array_equal(grads[k].astype(np.float32), want), (rank, k)
        assert np.abs(out[0][3][k] - full[k]).max() <= 1e-6 * np.abs(full[k]).max(), k


def test_two_gloo_ranks_sum_to_full_batch_gradients():
    import kron_workloads as kw
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = kw.get("tiny")
    d = {k: v.double().numpy() for k, v in kw.inputs(w).items()}
    full = oracle.backward(d["x"], d["S"], d["A"], d["B"], d["G"])
    out.sort(key=lambda t: t[0])
    dx = np.concatenate([o[4] for o in out])
    np.testing.assert_allclose(dx, full["dX"], rtol=0, atol=1e-12)
    for rank, start, count, grads, _ in out:
        for k in ("dS", "dA", "dB", "dbias"):
            scale = np.abs(full[k]).max()
            assert np.abs(grads[k] - full[k]).max() <= 1e-6 * scale, (rank, k)


def test_reference_arm_prints_once_under_two_ranks():
    """`bench.py --impl reference` under torchrun: rank 0 prints one JSON line, rank 1 exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--ref-rows", "8", "--workload", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    import json
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2


def _ks_rank_main(rank, world, port, result_q, deterministic):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import kron_workloads as kw
    import oracle
    from kronecker_factored_structured_b200 import dp

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = kw.ks_custom(53, 2, 3, 4, 5, seed=8)
        d = {k: v.double().numpy() for k, v in kw.ks_inputs(w).items()}
        start, count = dp.shard_rows(w.N, world, rank)
        sl = slice(start, start + count)
        g = oracle.ks_backward(d["x"][sl], d["w"], d["G"][sl])
        flat, views = dp.ks_flat_grad_buffer(*w.pattern)
        for k in ("dw", "dbias"):
            views[k].copy_(torch.from_numpy(g[k]).float())
        dp.allreduce_grads(flat, deterministic=deterministic)
        result_q.put((rank, {k: v.double().numpy().copy() for k, v in views.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("deterministic", [False, True])
def test_ks_factor_ranks_sum_to_full_batch_gradients(deterministic):
    """The Kronecker-sparse factor's data-parallel backward: row shards on two gloo ranks, dw
    and dbias in one flat buffer, one exchange; equal to the full batch's gradients."""
    import kron_workloads as kw
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ks_rank_main, args=(r, 2, port, q, deterministic))
             for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = kw.ks_custom(53, 2, 3, 4, 5, seed=8)
    d = {k: v.double().numpy() for k, v in kw.ks_inputs(w).items()}
    full = oracle.ks_backward(d["x"], d["w"], d["G"])
    for rank, grads in out:
        for k in ("dw", "dbias"):
            assert grads[k].shape == full[k].shape
            assert np.abs(grads[k] - full[k]).max() <= 1e-6 * np.abs(full[k]).max(), (rank, k)
    if deterministic:
        for k in ("dw", "dbias"):
            assert np.array_equal(out[0][1][k], out[1][1][k])
