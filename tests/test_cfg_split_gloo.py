"""CFG split over rank pairs, on the CPU with gloo: four ranks form two pairs, each
pair samples its own seed; within a pair rank 0 evaluates the conditional half and
rank 1 the unconditional half, and they exchange the halves every step.  The library
steps are stood in for by the CPU oracle on a tiny model, so this checks the exchange
schedule: which half each rank computes, the gather order, and that both ranks of a
pair apply the same update and end bit-identical, equal to one batched sampler."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from flow_matching_mmdit_b200 import cfg_split
from lens_inputs import TINY, make_weights, text_features
from oracle import lens_oracle as o

B, GH, GW, NT, STEPS, G = 1, 2, 3, 3, 3, 4.0
SEEDS = (21, 22)                       # one per pair


class OracleSteps:
    """The CPU oracle standing in for the library's step-wise sampler on one rank."""

    def __init__(self, W, E, seed, mu, phi):
        C, p = TINY.latent_channels, TINY.patch
        self.W, self.E, self.mu, self.phi = W, E, mu, phi
        self.x = o.noise(seed, B * C * p * GH * p * GW).reshape(B, C, p * GH, p * GW)
        self.grid = o.time_grid(STEPS, mu)
        self.v_all = torch.zeros((2, B, GH * GW, TINY.in_channels), dtype=torch.float64)
        self.v_local = torch.zeros((B, GH * GW, TINY.in_channels), dtype=torch.float64)

    def velocity(self, k, out):
        v = o.forward(self.W, TINY, o.patchify(self.x, TINY.patch), GH, GW, self.E, [self.grid[k]] * B)
        out.copy_(torch.from_numpy(v))

    def update(self, k, vc, vu):
        vc, vu = vc.numpy(), vu.numpy()
        vel = o.cfg_combine(vc, vu, G) if self.phi == 0.0 else o.cfg_rescaled(vc, vu, G, self.phi)
        dt = 1.0 / STEPS if self.mu is None else self.grid[k] - self.grid[k + 1]
        self.x = o.euler(self.x, o.unpatchify(vel, GH, GW, TINY.latent_channels, TINY.patch), dt)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mu, phi, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        groups = cfg_split.pair_groups(world, dist.new_group)
        pair, half = cfg_split.pair_of(rank)
        W = o.Weights(make_weights(TINY, seed=11, std=0.2, bias_std=0.05, gain_std=0.2))
        Ec = text_features(B, NT, 30 + pair, TINY)
        E = Ec if half == 0 else np.zeros_like(Ec)
        ops = OracleSteps(W, E, SEEDS[pair], mu, phi)
        cfg_split.cfg_split_steps(ops, STEPS, half, cfg_split.make_gather(groups[pair], dist.all_gather))
        q.put((rank, ops.x))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mu,phi", [(None, 0.0), (0.9, 1.0)])
def test_cfg_split_pairs_match_the_batched_sampler(mu, phi):
    world, port = 4, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mu, phi, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W = o.Weights(make_weights(TINY, seed=11, std=0.2, bias_std=0.05, gain_std=0.2))
    for pair in range(2):
        a, b = res[2 * pair], res[2 * pair + 1]
        assert np.array_equal(a, b)                       # both halves hold the same state
        Ec = text_features(B, NT, 30 + pair, TINY)
        ref = o.sample(W, TINY, Ec, None, B, GH, GW, STEPS, G, SEEDS[pair], mu=mu, phi=phi)
        assert np.allclose(a, ref, rtol=0, atol=1e-10)
    assert not np.allclose(res[0], res[2])                # the pairs are different samples


def test_pairing_rules():
    assert [cfg_split.pair_of(r) for r in range(4)] == [(0, 0), (0, 1), (1, 0), (1, 1)]
    made = []
    cfg_split.pair_groups(6, lambda ranks: made.append(list(ranks)) or len(made))
    assert made == [[0, 1], [2, 3], [4, 5]]
    for bad in (1, 3):
        with pytest.raises(ValueError):
            cfg_split.pair_groups(bad, lambda r: None)


# ------------------------------------------------------------------ bench.py --cfg-split plumbing
def test_bench_cfg_split_plan_and_refusals():
    import bench
    from lens_inputs import WORKLOADS
    wl = WORKLOADS["cfg_1024"]
    plans = [bench.cfg_split_plan(wl, r, 4) for r in range(4)]
    assert [(p["pair"], p["half"], p["conditional"]) for p in plans] == \
        [(0, 0, True), (0, 1, False), (1, 0, True), (1, 1, False)]
    assert plans[0]["seed"] == plans[1]["seed"] != plans[2]["seed"] == plans[3]["seed"]
    # whole-job units: each pair's sample counted once
    total = sum(p["units_per_rank"] for p in plans)
    assert total == 2 * wl.batch * wl.n_img * wl.steps
    assert bench.job_value(plans[0]["units_per_rank"], 4, 1000.0) == pytest.approx(total)
    assert bench.cfg_split_error(wl, 2, 2) is None
    assert bench.cfg_split_error(wl, 1, 1) and bench.cfg_split_error(wl, 3, 3) and bench.cfg_split_error(wl, 4, 2)
    assert bench.cfg_split_error(WORKLOADS["turbo_1024"], 2, 2)


class _WallTimer:
    def start(self):
        import time
        self.t0 = time.perf_counter()

    def stop(self):
        import time
        self.t1 = time.perf_counter()

    def elapsed_ms(self):
        return (self.t1 - self.t0) * 1e3


def _bench_worker(rank, world, port, q):
    import bench
    from lens_inputs import WORKLOADS
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = bench.cfg_split_plan(WORKLOADS["cfg_1024"], rank, world)
        groups = cfg_split.pair_groups(world, dist.new_group)
        W = o.Weights(make_weights(TINY, seed=11, std=0.2, bias_std=0.05, gain_std=0.2))
        Ec = text_features(B, NT, plan["text_seed"], TINY)
        E = Ec if plan["conditional"] else np.zeros_like(Ec)
        runs = []

        def step():
            ops = OracleSteps(W, E, plan["seed"], None, 0.0)
            cfg_split.cfg_split_steps(ops, STEPS, plan["half"], cfg_split.make_gather(groups[plan["pair"]],
                                                                                     dist.all_gather))
            runs.append(ops.x)

        ms = bench.timed_region(step, 2, dist.barrier, lambda: None, _WallTimer())
        mx = bench.max_over_ranks([ms], dist, "cpu")
        q.put((rank, runs, mx, plan["seed"], plan["text_seed"]))
    finally:
        dist.destroy_process_group()


def test_bench_cfg_split_timed_steps_on_two_ranks():
    """The two ranks of one pair, timed the way bench.py --cfg-split times them: exactly
    K steps each, both halves end on the same latent, equal to the batched sampler."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bench_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r[0], r[1:]) for r in (q.get(timeout=300) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (runs0, mx0, seed, tseed), (runs1, mx1, _, _) = res[0], res[1]
    assert len(runs0) == len(runs1) == 2 and mx0 == mx1
    W = o.Weights(make_weights(TINY, seed=11, std=0.2, bias_std=0.05, gain_std=0.2))
    ref = o.sample(W, TINY, text_features(B, NT, tseed, TINY), None, B, GH, GW, STEPS, G, seed)
    for a, b in zip(runs0, runs1):
        assert np.array_equal(a, b)
        assert np.allclose(a, ref, rtol=0, atol=1e-10)
