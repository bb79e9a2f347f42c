#!/usr/bin/env python
"""Throughput of the Lens MMDiT denoiser + flow-matching Euler sampler on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload turbo_1024] [--impl lens|reference]
                    [--cfg-rescale PHI] [--shift-mu MU] [--weight-bits 16|4] [--txt-valid T]

One step = one `lens_sample_euler_ex` call on seeded synthetic inputs: noise, text
input head, timestep/AdaLN modulation for every step, S denoiser forwards of 48
blocks, Euler (+CFG) updates and unpatchify.  Default workload: Turbo-style
4-step sampling at 1024^2 (4096 image + 256 text tokens, batch 1, guidance 1).
The metric counts image tokens through the 48-block denoiser per second (S forwards
per step), and the line also gives ms per sample and the fraction of bf16 peak.

Timing: W untimed steps, then K steps between a barrier + device synchronize,
CUDA events on the launching stream, max over ranks.  The 8.2 GB of weights are
streamed by every forward, so the working set is far larger than L2 (126 MB).
Multi-GPU (torchrun): independent replicas, one sample stream per GPU, no data
exchange (weak scaling).  --impl reference times the CPU oracle instead.
--cfg-rescale / --shift-mu time the sampler variants (norm-rescaled CFG, shifted
time grid); without them the call is the plain sampler.  --weight-bits 4 runs the
int4 weight-only model (block Linears 4-bit, group 64).  --txt-valid T marks all but the
first T text tokens of every sample as padding (masked keys in attention).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from lens_inputs import LENS, WORKLOADS, image_tokens, make_weights, text_features  # noqa: E402

METRIC = "DiT img-tokens/s per 1024² forward; ms per 4-step 1024² sample; % bf16 peak"
SPEC_BF16_TFLOPS = 2250.0
KERNEL_FAMILIES = ["attention", "gemm_qkv", "gemm_out", "gemm_w13", "gemm_w2", "rmsnorm_mod", "gemm_mod"]
KERNEL_SOURCES = {
    "attention": ["attention.cu", "ptx.cuh", "exp2_poly.h"],
    "gemm_qkv": ["gemm_tc.cuh", "gemm.cu", "ptx.cuh"], "gemm_out": ["gemm_tc.cuh", "gemm.cu", "ptx.cuh"],
    "gemm_w13": ["gemm_tc.cuh", "gemm.cu", "ptx.cuh"], "gemm_w2": ["gemm_tc.cuh", "gemm.cu", "ptx.cuh"],
    "gemm_mod": ["gemm_tc.cuh", "gemm.cu", "ptx.cuh"], "rmsnorm_mod": ["elementwise.cu"],
}


# ---------------------------------------------------------------- arithmetic of the workload
def forward_flops(n_img: int, n_txt: int, blocks: int = 48) -> float:
    """Algorithmic FLOPs of one denoiser forward for one batch row: block GEMMs
    (QKV, out, w1|w3, w2 on every token), joint attention (QK^T and PV), txt_in,
    img_in and proj_out."""
    N = n_img + n_txt
    D, F = 1536, 4096
    per_block = 2 * N * D * (3 * D + D + 2 * F + F) + 4 * N * N * D
    return blocks * per_block + 2 * n_txt * 4 * 2880 * D + 2 * n_img * 128 * D * 2


def kernel_work(kernel: str, B: int, n_img: int, n_txt: int):
    """(unit, algorithmic amount per launch) for one launch of a kernel family."""
    N, D, F = n_img + n_txt, 1536, 4096
    M = B * N
    if kernel == "attention":
        return "flop", 4.0 * B * N * N * D
    if kernel == "gemm_qkv":
        return "flop", 2.0 * M * D * 3 * D
    if kernel == "gemm_out":
        return "flop", 2.0 * M * D * D
    if kernel == "gemm_w13":
        return "flop", 2.0 * M * D * 2 * F
    if kernel == "gemm_w2":
        return "flop", 2.0 * M * F * D
    if kernel == "rmsnorm_mod":   # both streams in one launch: fp32 row in, bf16 row out
        return "byte", B * (n_img + n_txt) * D * (4.0 + 2.0)
    if kernel == "gemm_mod":
        return "byte", (48 * 2 * 9216 + 3072) * D * 2.0
    raise ValueError(kernel)


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "flow_matching_mmdit_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def dram_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on the
    current source of that kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    for rec in json.load(open(p)).get("records", []):
        if rec.get("kernel") == kernel and rec.get("workload") == workload and \
                rec.get("source_hash") == source_hash(kernel):
            return rec.get("dram_bytes_per_launch")
    return None


# ---------------------------------------------------------------- replica plumbing
class EventTimer:
    """Device timing with CUDA events on the launching stream."""

    def __init__(self, stream):
        import torch
        self.stream = stream
        self.ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    def start(self):
        self.ev[0].record(self.stream)

    def stop(self):
        self.ev[1].record(self.stream)

    def elapsed_ms(self) -> float:
        return self.ev[0].elapsed_time(self.ev[1])


def timed_region(step, steps: int, barrier, sync, timer) -> float:
    """Barrier + synchronize, time exactly `steps` calls of step(), synchronize +
    barrier; returns this rank's elapsed milliseconds."""
    barrier()
    sync()
    timer.start()
    for _ in range(steps):
        step()
    timer.stop()
    sync()
    barrier()
    return timer.elapsed_ms()


def max_over_ranks(values, dist, device) -> list:
    """Element-wise max of per-rank values (identity without a process group)."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_value(units_per_step_per_rank: float, n_ranks: int, ms_per_step: float) -> float:
    """Whole-job throughput: the units every rank processed per step / the slowest
    rank's time per step (weak scaling: each rank runs its own replica)."""
    return n_ranks * units_per_step_per_rank / (ms_per_step / 1e3)


# ---------------------------------------------------------------- CFG split over rank pairs
def cfg_split_error(wl, gpus: int, world: int):
    """Why --cfg-split cannot run with these settings (None when it can)."""
    if wl.guidance == 1.0:
        return "--cfg-split needs a CFG workload (guidance != 1)"
    if gpus < 2 or gpus % 2 or world != gpus:
        return "--cfg-split needs an even --gpus >= 2, launched as that many torchrun ranks"
    return None


def cfg_split_plan(wl, rank: int, world: int) -> dict:
    """This rank's part of a CFG-split job: pair p = rank // 2 samples seed wl.seed +
    1000 p; half 0 runs the conditional text (features drawn from that seed), half 1 the
    unconditional (zeros).  units_per_rank: image tokens through the denoiser per step
    and rank, so that job_value over all ranks counts each pair's sample once."""
    pair, half = rank // 2, rank % 2
    seed = wl.seed + 1000 * pair
    return {"pair": pair, "half": half, "pairs": world // 2, "seed": seed, "text_seed": seed,
            "conditional": half == 0, "units_per_rank": wl.batch * wl.n_img * wl.steps / 2.0}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.first = 0

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # the query tool takes a while to start: begin the region once it samples, and
            # keep only the samples from the region on
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0:
                time.sleep(0.005)
            self.first = len(self.lines)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            # a region shorter than the sampling interval takes the first sample after it
            t0 = time.time()
            while len(self.lines) <= self.first and time.time() - t0 < 1.0:
                time.sleep(0.005)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        for l in self.lines[self.first:]:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9 or (self.uuid and self.uuid not in f[0]):
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clocks not sampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower().startswith("active")})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle leg
def oracle_block_seconds(wl, max_seconds: float = 20.0):
    """Time the oracle (as it stands, fp64 numpy) on one denoiser block at the
    workload's shape, repeated while under max_seconds.  Returns (s per block,
    blocks timed, threads)."""
    from oracle import lens_oracle as o
    d = LENS.with_blocks(1)
    W = o.Weights(make_weights(d, seed=0))
    rng = np.random.default_rng(0)
    B = wl.batch * (2 if wl.guidance != 1.0 else 1)
    hi = rng.standard_normal((B, wl.n_img, 1536))
    ht = rng.standard_normal((B, wl.n_txt, 1536))
    temb = o.timestep_embedding(W, np.full(B, 0.5), 256)
    ang = o.rope_angles(o.position_ids(wl.grid_h, wl.grid_w, wl.n_txt), d.rope_axes, d.rope_theta)
    times = []
    t_all = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        o.block(W, 0, hi, ht, temb, ang, d.heads, d.eps)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all + times[-1] > max_seconds or len(times) >= 20:
            break
    return float(np.median(times)), len(times), os.cpu_count()


def oracle_value(wl, s_per_block: float) -> float:
    """img-tokens/s of the oracle on the workload: S forwards of 48 blocks per
    sample (the non-block work is < 1% of the FLOPs and not counted)."""
    B = wl.batch * (2 if wl.guidance != 1.0 else 1)
    steps = max(wl.steps, 1)
    t_sample = steps * 48 * s_per_block
    return wl.batch * wl.n_img * steps / t_sample, B


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=None, choices=[k for k, v in WORKLOADS.items() if v.num_blocks == 48],
                    help="default: turbo_1024 (cfg_1024 with --cfg-split); fwd_512 times single forwards")
    ap.add_argument("--impl", default="lens", choices=["lens", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cfg-rescale", type=float, default=0.0,
                    help="norm-rescaled CFG weight phi in [0, 1] (0: plain CFG)")
    ap.add_argument("--shift-mu", type=float, default=None,
                    help="shifted time grid with this mu (default: uniform grid)")
    ap.add_argument("--txt-valid", type=int, default=None,
                    help="valid text tokens per sample (the rest are padding, masked in attention)")
    ap.add_argument("--weight-bits", type=int, default=16, choices=[16, 4],
                    help="4: int4 weight-only block Linears (group 64), quantized at create")
    ap.add_argument("--cfg-split", action="store_true",
                    help="CFG halves on rank pairs (even --gpus >= 2 under torchrun): the conditional and the "
                         "unconditional forward of each sample on two GPUs, one velocity all-gather per step")
    args = ap.parse_args()
    if args.workload is None:
        args.workload = "cfg_1024" if args.cfg_split else "turbo_1024"
    wl = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.cfg_split:
        err = cfg_split_error(wl, args.gpus, world)
        if err:
            print(json.dumps({"metric": METRIC, "error": err}), flush=True)
            return 2
    config = {"workload": f"{args.workload}: {wl.name}", "batch": wl.batch, "img_tokens": wl.n_img,
              "txt_tokens": wl.n_txt, "sampling_steps": wl.steps, "guidance": wl.guidance, "blocks": 48,
              "forward_rows": wl.batch * (2 if wl.guidance != 1.0 else 1),
              "l2": "inputs larger than L2: 8.2 GB of weights streamed by every forward",
              "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU"}
    if args.cfg_split:
        config["forward_rows"] = wl.batch            # each rank runs one half of the CFG batch
        config["parallelism"] = f"CFG split: {world // 2} rank pair(s), one velocity all-gather per step"
    if args.txt_valid is not None:
        config["txt_valid"] = args.txt_valid
    if args.weight_bits != 16:
        config["weight_bits"] = args.weight_bits
        config["l2"] = "inputs larger than L2: 2.35 GB of 4-bit block weights streamed by every forward"
    if args.cfg_rescale != 0.0 or args.shift_mu is not None:
        config["sampler_variant"] = {"cfg_rescale": args.cfg_rescale, "shift_mu": args.shift_mu}

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, wl, config)

    import torch
    import flow_matching_mmdit_b200 as L

    torch.cuda.set_device(local)
    # a created stream: the library captures each sampler call as a CUDA graph there
    work_stream = torch.cuda.Stream()
    with torch.cuda.stream(work_stream):
        return _run_lens(args, wl, config, world, rank, local, torch, L)


def _run_lens(args, wl, config, world, rank, local, torch, L):
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))

    weights = make_weights(LENS, seed=0)
    cfg = L.lens_dit_default_config()
    rows = config["forward_rows"]
    cfg.max_batch, cfg.max_img_tokens, cfg.max_txt_tokens = rows, wl.n_img, wl.n_txt
    cfg.weight_bits = args.weight_bits
    h = L.lens_dit_create(cfg, weights)
    del weights
    plan = cfg_split_plan(wl, rank, world) if args.cfg_split else None
    seed = plan["seed"] if plan else wl.seed + 1000 * rank
    txt_host = text_features(wl.batch, wl.n_txt, seed)
    txt = torch.from_numpy(txt_host.view(np.int16)).cuda()
    out = torch.empty((wl.batch, 32, 2 * wl.grid_h, 2 * wl.grid_w), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    opt = L.lens_sampler_default_options()
    opt.guidance, opt.cfg_rescale = wl.guidance, args.cfg_rescale
    if args.shift_mu is not None:
        opt.time_shift, opt.shift_mu = 1, args.shift_mu

    lens = None if args.txt_valid is None else [args.txt_valid] * wl.batch

    if plan:
        from flow_matching_mmdit_b200 import cfg_split
        groups = cfg_split.pair_groups(world, dist.new_group)

        def sample(text):                            # noqa: F811
            cfg_split.sample_cfg_split(h, text if plan["conditional"] else None, lens, wl.batch, wl.n_txt,
                                       wl.height_px, wl.width_px, wl.steps, opt, seed, out, groups[plan["pair"]],
                                       plan["half"])
    elif wl.steps == 0:
        # a single-forward workload: one step = one 48-block forward of seeded N(0, 1) tokens at wl.t
        tok_host = image_tokens(wl.batch, wl.n_img, seed)
        tok = torch.from_numpy(tok_host).cuda()
        out = torch.empty((wl.batch, wl.n_img, 128), dtype=torch.float32, device="cuda")

        def sample(text):                            # noqa: F811
            L.lens_dit_forward_masked(h, tok, wl.batch, wl.grid_h, wl.grid_w, text, wl.n_txt, lens,
                                      [wl.t] * wl.batch, out)
    else:
        def sample(text):                            # noqa: F811
            L.lens_sample_euler_ex(h, text, lens, None, lens, wl.batch, wl.n_txt, wl.height_px, wl.width_px,
                                   wl.steps, opt, seed, out)

    def step():
        sample(txt)

    for _ in range(args.warmup):
        step()
    L.lens_dit_sync(h)

    # which kernel family dominates the step (one profiled sample per family, untimed)
    fam_ms, fam_n = {}, {}
    for k in KERNEL_FAMILIES:
        L.lens_dit_profile_kernel(h, k, 4096)
        step()
        n, ms = L.lens_dit_profile_read(h)
        fam_ms[k], fam_n[k] = ms, n
    dominant = max(fam_ms, key=fam_ms.get)
    L.lens_dit_profile_kernel(h, "none", 0)
    step()                                     # re-capture the uninstrumented graph, untimed
    L.lens_dit_sync(h)

    # ------------------------------------------------ timed region (device-resident inputs, no instrumentation)
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    launches0 = L.lens_dit_launch_count(h)
    barrier = dist.barrier if dist else (lambda: None)
    with ClockSampler(uuid) as clk:
        ms_total = timed_region(step, args.steps, barrier, torch.cuda.synchronize, EventTimer(stream))
    L.lens_dit_sync(h)
    gpu_launches = L.lens_dit_launch_count(h) - launches0

    # ------------------------------------------------ end to end through host buffers (right after the timed
    # region, so that both see the same clocks)
    txt_pinned = torch.from_numpy(txt_host.view(np.int16)).pin_memory()
    out_pinned = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    txt_dev = torch.empty_like(txt)
    for _ in range(2):
        txt_dev.copy_(txt_pinned, non_blocking=True)
        sample(txt_dev)
        out_pinned.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    tok_pinned = torch.from_numpy(tok_host).pin_memory() if wl.steps == 0 else None

    def e2e_step():
        txt_dev.copy_(txt_pinned, non_blocking=True)
        if tok_pinned is not None:
            tok.copy_(tok_pinned, non_blocking=True)
        sample(txt_dev)
        out_pinned.copy_(out, non_blocking=True)

    e2e_ms = timed_region(e2e_step, args.steps, barrier, torch.cuda.synchronize, EventTimer(stream))
    L.lens_dit_sync(h)
    assert np.all(np.isfinite(out_pinned.numpy()))

    # ------------------------------------------------ profiled pass (untimed): the dominant family's launches
    # bracketed by CUDA-event pairs that the library records on the launching stream; the same steps as the
    # timed region, run after the timed and the end-to-end regions
    prof_steps = max(1, min(args.steps, 5))
    L.lens_dit_profile_kernel(h, dominant, 4096 * prof_steps)
    with ClockSampler(uuid) as clk_prof:
        for _ in range(prof_steps):
            step()
        L.lens_dit_sync(h)
    k_launches, k_ms = L.lens_dit_profile_read(h)
    L.lens_dit_profile_kernel(h, "none", 0)
    step()
    L.lens_dit_sync(h)

    ms_total, e2e_ms = max_over_ranks([ms_total, e2e_ms], dist, "cuda")

    ms_step = ms_total / args.steps
    forwards = max(wl.steps, 1)
    tokens_per_step = plan["units_per_rank"] if plan else wl.batch * wl.n_img * forwards
    value = job_value(tokens_per_step, args.gpus, ms_step)
    e2e_value = job_value(tokens_per_step, args.gpus, e2e_ms / args.steps)
    flops_step = forwards * config["forward_rows"] * forward_flops(wl.n_img, wl.n_txt)
    peaks = measured_peaks()
    tflops = flops_step / (ms_step / 1e3) / 1e12

    unit, work = kernel_work(dominant, config["forward_rows"], wl.n_img, wl.n_txt)
    # On the created stream each sampler call replays one captured graph whose event
    # nodes are re-recorded by every replay: the events hold the profiled pass's last step.
    avg_launch_s = (k_ms / max(k_launches, 1)) / 1e3
    if unit == "flop":
        achieved = work / avg_launch_s / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "unit": "TFLOP/s", "peak_kind": f"bf16 sustained ({peaks['source']})"}
    else:
        achieved = work / avg_launch_s / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "unit": "GB/s", "peak_kind": f"HBM copy ({peaks['source']})"}
    roof.update({"kernel": dominant, "achieved": round(achieved, 2), "peak": peak, "frac": round(achieved / peak, 4),
                 "traffic": dram_traffic(dominant, args.workload), "launches_timed": k_launches,
                 "avg_launch_us": round(avg_launch_s * 1e6, 2), "algorithmic_per_launch": work,
                 "share_of_step": round(avg_launch_s * 1e3 * fam_n[dominant] / ms_step, 4),
                 "events": "CUDA-event pairs around each launch of the kernel, recorded by the library on the "
                           f"launching stream in an untimed pass of {prof_steps} steps run right after the timed "
                           "region (graph replay: the events hold the pass's last step)",
                 "profiled_pass_clocks": clk_prof.summary(),
                 "family_ms_one_step": {k: round(v, 3) for k, v in fam_ms.items()}})

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "img-tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) text features "
        "and noise; random-init N(0,0.02) bf16 weights of the 48-block Lens DiT)", "config": config,
        "ms_per_sample": round(ms_step, 3),
        "pct_bf16_peak": {"tflops": round(tflops, 1), "of_spec_2250": round(tflops / SPEC_BF16_TFLOPS, 4),
                          f"of_{peaks['source']}_burst": round(tflops * 1e0 / peaks["bf16_tflops"], 4),
                          f"of_{peaks['source']}_sustained": round(tflops / peaks["bf16_tflops_sustained"], 4)},
        "e2e": {"value": round(e2e_value, 1), "unit": "img-tokens/s",
                "h2d_bytes_per_step": int(txt_host.nbytes) + (int(tok_host.nbytes) if wl.steps == 0 else 0),
                "d2h_bytes_per_step": int(out.numel() * 4),
                "ms_per_step": round(e2e_ms / args.steps, 3)},
        "roofline": roof, "gpu_launches": int(gpu_launches), "clocks": clk.summary(),
        "context": {"pages_h100_turbo_4step_1024_s": 0.84, "pages_h100_20step_cfg5_1024_s": 3.15,
                    "note": "pages' latencies are end-to-end on H100 (encoder/VAE inclusion unstated)"},
    }
    if rank == 0 and args.gpus == 1 and not args.no_cpu_baseline:
        s_blk, n_blk, cores = oracle_block_seconds(wl, 20.0)
        v_cpu, rows_cpu = oracle_value(wl, s_blk)
        line["cpu_baseline"] = {"value": round(v_cpu, 3), "unit": "img-tokens/s", "cores": cores, "kind": "oracle",
                                "extrapolated": True,
                                "measured": {"what": f"one block of the 48-block model at the workload shape "
                                                     f"({rows_cpu} rows x {wl.n_img + wl.n_txt} tokens, fp64 numpy)",
                                             "s_per_block_median": round(s_blk, 3), "runs": n_blk},
                                "sample": f"{n_blk} timed runs of one block; value = that median scaled by "
                                          f"48 blocks x {wl.steps} forwards (extrapolated, not a timed sample)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    h.destroy()
    if dist:
        dist.destroy_process_group()
    return 0


def run_reference(args, wl, config):
    """The CPU oracle as it stands, on this host's cores: each step is a bounded
    sample (one denoiser block at the workload's shape), scaled to the metric."""
    from oracle import lens_oracle as o
    d = LENS.with_blocks(1)
    W = o.Weights(make_weights(d, seed=0))
    rng = np.random.default_rng(0)
    B = config["forward_rows"]
    hi = rng.standard_normal((B, wl.n_img, 1536))
    ht = rng.standard_normal((B, wl.n_txt, 1536))
    temb = o.timestep_embedding(W, np.full(B, 0.5), 256)
    ang = o.rope_angles(o.position_ids(wl.grid_h, wl.grid_w, wl.n_txt), d.rope_axes, d.rope_theta)
    for _ in range(args.warmup):
        o.block(W, 0, hi, ht, temb, ang, d.heads, d.eps)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.block(W, 0, hi, ht, temb, ang, d.heads, d.eps)
    s_blk = (time.perf_counter() - t0) / args.steps
    v, _ = oracle_value(wl, s_blk)
    sample = (f"each step: one block of the 48-block model at the workload shape ({B} rows x "
              f"{wl.n_img + wl.n_txt} tokens, fp64 numpy), timed; value = img-tokens/s of a whole sample "
              f"extrapolated from the per-block time by 48 blocks x {wl.steps} forwards")
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "img-tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * s_blk, 1),
            "step": "one denoiser block at the workload shape (the bounded sample that was timed)",
            "extrapolated": True,
            "extrapolated_ms_per_sample": round(1e3 * max(wl.steps, 1) * 48 * s_blk, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": round(v, 3), "unit": "img-tokens/s", "kind": "oracle", "cores": os.cpu_count(),
                             "extrapolated": True, "sample": sample},
            "e2e": {"value": round(v, 3), "unit": "img-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
