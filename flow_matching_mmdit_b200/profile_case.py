"""Run one kernel family of the denoiser on seeded inputs at a workload's shape, for
profiling (ncu) and quick timing:

    python -m flow_matching_mmdit_b200.profile_case --case attention --workload turbo_1024 --iters 3
    python -m flow_matching_mmdit_b200.profile_case --case blocks --workload turbo_1024 --blocks 2 --iters 2

`attention` runs the joint-attention op on random q, k, v of the workload's
sequence; `blocks` runs `blocks` denoiser blocks (every GEMM epilogue, attention and
RMSNorm) through the debug hook of a model with that many blocks; `gemm` runs the
plain tcgen05 GEMM op at M = rows x tokens, N = 8192, K = 1536; `rmsnorm` runs
RMSNorm + modulate over all rows x tokens fp32 rows (one sample's shift and scale
per batch row).  Prints the CUDA-event time per iteration.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main() -> int:
    import torch

    import flow_matching_mmdit_b200 as L
    from lens_inputs import LENS, WORKLOADS, f32_to_bf16_bits, make_weights

    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=["attention", "blocks", "gemm", "rmsnorm"], required=True)
    ap.add_argument("--workload", default="turbo_1024")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--blocks", type=int, default=2)
    a = ap.parse_args()
    wl = WORKLOADS[a.workload]
    rows = wl.batch * (2 if wl.guidance != 1.0 else 1)
    N = wl.n_img + wl.n_txt
    rng = np.random.default_rng(0)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    unit = "TFLOP/s"

    if a.case == "attention":
        q, k, v = (torch.from_numpy(f32_to_bf16_bits(rng.standard_normal((rows, 24, N, 64)).astype(np.float32))
                                    .view(np.int16)).cuda() for _ in range(3))
        ot = torch.empty((rows, wl.n_txt, 1536), dtype=torch.int16, device="cuda")
        oi = torch.empty((rows, wl.n_img, 1536), dtype=torch.int16, device="cuda")
        run = lambda: L.lens_op_attention(q, k, v, rows, wl.n_txt, wl.n_img, ot, oi)
        flops = 4.0 * rows * N * N * 1536
    elif a.case == "gemm":
        M = rows * N
        A = torch.from_numpy(f32_to_bf16_bits(rng.standard_normal((M, 1536)).astype(np.float32)).view(np.int16)).cuda()
        B = torch.from_numpy(f32_to_bf16_bits(rng.standard_normal((8192, 1536)).astype(np.float32) * 0.02)
                             .view(np.int16)).cuda()
        C = torch.empty((M, 8192), dtype=torch.float32, device="cuda")
        run = lambda: L.lens_op_gemm_bf16(A, B, None, C, M, 8192, 1536)
        flops = 2.0 * M * 8192 * 1536
    elif a.case == "rmsnorm":
        M = rows * N
        x = torch.from_numpy(rng.standard_normal((M, 1536)).astype(np.float32) * 3).cuda()
        mod = torch.from_numpy(rng.standard_normal((rows, 6 * 1536)).astype(np.float32) * 0.2).cuda()
        y = torch.empty((M, 1536), dtype=torch.int16, device="cuda")
        run = lambda: L.lens_op_rmsnorm_modulate(x, M, N, mod[:, 1536:], mod[:, 3072:], 6 * 1536, 1e-6, y)
        flops, unit = M * 1536 * 6.0, "TB/s"   # bytes: fp32 in, bf16 out
    else:
        d = LENS.with_blocks(a.blocks)
        cfg = L.lens_dit_default_config()
        cfg.num_blocks = a.blocks
        cfg.max_batch, cfg.max_img_tokens, cfg.max_txt_tokens = rows, wl.n_img, wl.n_txt
        h = L.lens_dit_create(cfg, make_weights(d, seed=0))
        hi = torch.from_numpy(rng.standard_normal((rows, wl.n_img, 1536)).astype(np.float32) * 0.3).cuda()
        ht = torch.from_numpy(rng.standard_normal((rows, wl.n_txt, 1536)).astype(np.float32) * 2).cuda()
        run = lambda: L.lens_dit_debug_blocks(h, 0, a.blocks, hi, ht, rows, wl.grid_h, wl.grid_w, wl.n_txt,
                                              [0.5] * rows)
        flops = a.blocks * rows * (2 * N * 1536 * (4608 + 1536 + 8192 + 4096) + 4 * N * N * 1536)

    run()
    torch.cuda.synchronize()
    for i in range(a.iters):
        ev0.record()
        run()
        ev1.record()
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1)
        print(f"{a.case} {a.workload} iter {i}: {ms:.3f} ms, {flops / ms / 1e9:.2f} {unit}", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
