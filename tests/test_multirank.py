"""Multi-rank host logic of bench.py on CPU: two gloo ranks, as torchrun would
start them (RANK / WORLD_SIZE / MASTER_ADDR from the environment).

What runs on N GPUs is N independent decode problems (one per rank, weak
scaling) with no collective on the data path; the only cross-rank steps are
the barriers around the timed region and the max-reduction of the device
time.  Those, the whole-job throughput formula and the reference arm's
rank-0-only rule are checked here."""

import os
import socket
import sys
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank_ms, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        total = bench.max_over_ranks(per_rank_ms[rank], world, torch.device("cpu"))
        dist.barrier()
        value = bench.whole_job_gbs(world, 100, 412_076_336, total)
        ref = bench.run_reference(types.SimpleNamespace(workload="tiny_2k", seed=0, steps=1,
                                                        warmup=0), rank, world) if rank else None
        out_q.put((rank, total, value, ref))
    finally:
        dist.destroy_process_group()


def run_ranks(world, per_rank_ms):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, per_rank_ms, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_two_ranks_take_the_slowest_device_time():
    res = run_ranks(2, [10.0, 12.5])
    for rank, total, value, ref in res:
        assert total == 12.5
        # 2 ranks x 100 steps x 412 MB in 12.5 ms
        assert value == pytest.approx(2 * 100 * 412_076_336 / 12.5e-3 / 1e9)
    # the reference arm does its work on rank 0 only; other ranks return at once
    assert res[1][3] is None


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.25, 1, torch.device("cpu")) == 7.25
    assert bench.whole_job_gbs(1, 10, 1000, 1.0) == pytest.approx(10 * 1000 / 1e-3 / 1e9)


def test_reference_arm_sample_stays_inside_the_window():
    """With a 512-key window the oracle sample holds at most the visible keys
    (the bytes it reports are the bytes it read)."""
    import re
    ref = bench.run_reference(types.SimpleNamespace(workload="v1_sliding_100k", seed=0, steps=1,
                                                    warmup=0), 0, 1)
    n = int(re.search(r"the last (\d+) visible keys", ref["cpu_baseline"]["sample"]).group(1))
    assert 0 < n <= 512
    assert ref["value"] == ref["cpu_baseline"]["value"] > 0
