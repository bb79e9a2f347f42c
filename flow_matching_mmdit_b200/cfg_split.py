"""Classifier-free guidance split across GPUs: the conditional and the unconditional
half of every step on two ranks, one velocity exchange per step.

Ranks form pairs (2p, 2p + 1).  Rank 2p evaluates the conditional text, rank 2p + 1
the unconditional text, of the same sample(s) with the same noise seed.  Each step
both ranks compute their half's velocity with the library's step-wise sampler, the
pair all-gathers the two halves (NCCL over NVLink / NVSwitch on GPUs), and both apply
the same Euler/CFG update to the same state, so the two copies stay bit-identical and
equal to the one-GPU sampler, whose batch rows do not depend on each other.  Pairs
are independent replicas of one another (different samples, no exchange).

Where the method needs it: summary page "Lens: 重新思考基础文生图模型的训练效率",
section "方法步骤详情" (20 steps at CFG 5.0) and the blog "Lens", section "Exploring
Image Editing" (uncond + s (cond - uncond)): each step needs both halves once.  The
exchange is 4 * B * N_img * 128 bytes per rank per step (2 MB at 1024^2), against a
forward of several milliseconds, so a plain all-gather is the whole collective.
"""
from __future__ import annotations

from typing import Callable, List, Sequence

from . import binding as L


def pair_of(rank: int) -> tuple:
    """(pair index, half): half 0 = conditional, 1 = unconditional."""
    return rank // 2, rank % 2


def pair_groups(world: int, new_group: Callable[[Sequence[int]], object]) -> List[object]:
    """One process group per pair.  Every rank must call this with the same world so
    that all ranks create the groups in the same order."""
    if world < 2 or world % 2:
        raise ValueError(f"CFG split needs an even number of ranks, got {world}")
    return [new_group([2 * p, 2 * p + 1]) for p in range(world // 2)]


def make_gather(group, all_gather: Callable) -> Callable:
    """gather(v_all, v_local): v_all[0] <- the conditional half (pair rank 0), v_all[1]
    <- the unconditional half (pair rank 1); all_gather is torch.distributed's."""
    def gather(v_all, v_local):
        all_gather(list(v_all.unbind(0)), v_local, group=group)
    return gather


def cfg_split_steps(ops, steps: int, half: int, gather: Callable) -> None:
    """The exchange schedule.  ops.velocity(k, out) writes this rank's half at step k,
    ops.update(k, v_cond, v_uncond) applies step k; ops.v_all holds both halves
    ([2, ...]) and ops.v_local this rank's."""
    if half not in (0, 1):
        raise ValueError("half must be 0 (conditional) or 1 (unconditional)")
    for k in range(steps):
        ops.velocity(k, ops.v_local)
        gather(ops.v_all, ops.v_local)
        ops.update(k, ops.v_all[0], ops.v_all[1])


class LibrarySteps:
    """The library's step-wise sampler on one handle (this rank's half)."""

    def __init__(self, h, v_all, v_local, stream=None):
        self.h, self.v_all, self.v_local, self.stream = h, v_all, v_local, stream

    def velocity(self, k, out):
        L.lens_sampler_velocity(self.h, k, out, self.stream)

    def update(self, k, v_cond, v_uncond):
        L.lens_sampler_update(self.h, k, v_cond, v_uncond, self.stream)


def sample_cfg_split(h, txt, txt_len, B: int, n_txt: int, height_px: int, width_px: int, steps: int,
                     opt, seed: int, latent_out, group, half: int) -> None:
    """One CFG sample split over the pair `group` (this rank is `half`).

    txt is this rank's text: the conditional features on half 0, the unconditional
    ones on half 1 (None = zeros, the plain sampler's unconditional text).  Work runs
    on torch's current stream, which the collective orders against.  latent_out
    (dev fp32 [B, 32, height/8, width/8]) receives the same latent on both ranks."""
    import torch
    import torch.distributed as dist

    if opt.guidance == 1.0:
        raise ValueError("guidance 1 has no unconditional half to split")
    ni = (height_px // 16) * (width_px // 16)
    stream = torch.cuda.current_stream()
    L.lens_sampler_prepare(h, txt, txt_len, B, n_txt, height_px, width_px, steps, opt, seed, stream)
    v_all = torch.empty((2, B, ni, 128), dtype=torch.float32, device="cuda")
    v_local = torch.empty((B, ni, 128), dtype=torch.float32, device="cuda")
    ops = LibrarySteps(h, v_all, v_local, stream)
    cfg_split_steps(ops, steps, half, make_gather(group, dist.all_gather))
    L.lens_sampler_finish(h, latent_out, stream)
