"""The N > 1 host logic of bench.py on CPU: two ranks over gloo (127.0.0.1).

Each rank runs its own replica of the workload, so the only cross-rank steps are the barriers
around the timed region and the max-reduce of the device time; rank 0 alone reports. These tests
run exactly those functions with rank-dependent times and check what the job would report.
"""
import importlib.util
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    bench = _bench()
    import torch.distributed as dist
    w, r, local = bench.dist_setup("gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    mx = bench.max_over_ranks(10.0 * (rank + 1), w)
    # rank r timed 100 + 50 r ms over 10 steps, each on a replica of 1000 tokens
    value, ms_step = bench.throughput(100.0 + 50.0 * rank, 10, 1000, w)

    class Args:
        workload, steps, warmup = "tiny-2k-fp32", 1, 0

    ref = bench.run_reference(Args, w, r) if r != 0 else "rank0-skipped"
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((rank, mx, value, ms_step, ref))


@pytest.mark.timeout(300)
def test_two_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = [out.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    by_rank = {g[0]: g[1:] for g in got}
    slowest_ms_step = (100.0 + 50.0 * (world - 1)) / 10
    for r in range(world):
        mx, value, ms_step, ref = by_rank[r]
        assert mx == 10.0 * world                      # the max, on every rank
        assert ms_step == pytest.approx(slowest_ms_step)  # the slowest rank sets the time
        assert value == pytest.approx(1000 * world / (slowest_ms_step / 1e3))  # weak scaling
        if r != 0:
            assert ref is None                         # only rank 0 runs the reference arm


def test_single_rank_needs_no_process_group():
    bench = _bench()
    assert bench.max_over_ranks(3.5, 1) == 3.5
    value, ms = bench.throughput(20.0, 4, 500, 1)
    assert ms == 5.0 and value == pytest.approx(500 / 5e-3)
