"""The multi-GPU path of bench.py runs one independent replica per rank (the denoiser
does not shard below a sample): barrier + synchronize around exactly K timed
steps, max over ranks, whole-job value = ranks x units / slowest time.  Exercised
here with two gloo ranks on the CPU, ranks made deliberately unequal."""
import os
import socket
import time

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


class WallTimer:
    """CPU stand-in for the CUDA-event timer (the GPU path times on the device)."""

    def start(self):
        self.t0 = time.perf_counter()

    def stop(self):
        self.t1 = time.perf_counter()

    def elapsed_ms(self):
        return (self.t1 - self.t0) * 1e3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        calls = []
        step = lambda: (calls.append(1), time.sleep(0.01 * (rank + 1)))
        ms = bench.timed_region(step, 5, dist.barrier, lambda: None, WallTimer())
        mx = bench.max_over_ranks([ms, 2.0 * ms], dist, "cpu")
        q.put((rank, len(calls), ms, mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, n0, ms0, mx0), (r1, n1, ms1, mx1) = res
    assert n0 == n1 == 5                          # exactly K steps on every rank
    assert ms1 > ms0 >= 5 * 10.0                  # rank 1 sleeps twice as long
    assert mx0 == mx1 == pytest.approx([ms1, 2 * ms1])   # every rank sees the max
    # whole-job value: both ranks' units over the slowest rank's time per step
    v = bench.job_value(4096 * 4, world, mx0[0] / 5)
    assert v == pytest.approx(2 * 4096 * 4 / (ms1 / 5 / 1e3))


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks([1.5, 2.5], None, "cpu") == [1.5, 2.5]
    assert bench.job_value(100, 1, 10.0) == pytest.approx(10_000.0)
