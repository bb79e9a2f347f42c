"""Write the oracle's references for the full-size workloads into tests/golden/full/.

Run once, offline, on the CPU (it imports only `oracle` and `lens_inputs`; nothing here
touches the CUDA library):

    OPENBLAS_NUM_THREADS=4 python tests/golden/make_full_refs.py turbo_1024 cfg_1024
    OPENBLAS_NUM_THREADS=4 python tests/golden/make_full_refs.py cfg_1440 cfg_1024x2048

The fp64 oracle takes about 9 CPU-minutes (8 cores) per 48-block forward of one batch
row at 4096 + 256 tokens and about 25 at 8100 + 256, so the runs are sized to the
forwards each comparison needs:

  turbo_1024    one forward at t = 0.5 on N(0, 1) image tokens (seed 3), and the whole
                4-step sample at guidance 1 (the workload itself): 5 forwards.
  cfg_1024      the first forward of the CFG sample (t = 1 on the seeded noise, the
                conditional and the zero-text row), a complete 2-step sample at CFG 5
                (grid 1, 1/2), and the state after the first step of the 20-step grid:
                4 forwards (the 20-step state reuses the first two).
  cfg_1440,     the first forward (t = 1, both rows), a complete 1-step sample at CFG 5
  cfg_1024x2048 and the state after the first step of the 50-step grid: 2 forwards.

Each file holds float16 copies (relative rounding 2^-11, far below the cosine bars the
tests apply) of the velocities and of the displacements latent - noise(seed), the part
of the latent the denoiser decides; the tests rebuild the noise with oracle.noise.
The oracle source's SHA-256 at generation time is stored beside them.
"""
from __future__ import annotations

import hashlib
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from lens_inputs import LENS, WORKLOADS, image_tokens, make_weights, text_features  # noqa: E402
from oracle import lens_oracle as o  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "full")


def oracle_sha() -> str:
    with open(os.path.join(ROOT, "oracle", "lens_oracle.py"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def _noise_latent(wl) -> np.ndarray:
    C = LENS.latent_channels
    n = C * 2 * wl.grid_h * 2 * wl.grid_w
    return o.noise(wl.seed, n).astype(np.float64).reshape(1, C, 2 * wl.grid_h, 2 * wl.grid_w)


def _f16(x) -> np.ndarray:
    return np.asarray(x, np.float64).astype(np.float16)


def make(name: str, W) -> dict:
    wl = WORKLOADS[name]
    E = text_features(1, wl.n_txt, wl.seed)
    z = _noise_latent(wl)
    rec = {"workload": np.array(name), "oracle_sha256": np.array(oracle_sha()), "seed": np.array(wl.seed)}
    if name == "turbo_1024":
        X = image_tokens(1, wl.n_img, wl.seed)
        rec["fwd_t"] = np.array([0.5])
        rec["fwd_input"] = np.array("image_tokens")
        rec["fwd_v"] = _f16(o.forward(W, LENS, X, wl.grid_h, wl.grid_w, E, [0.5]))
        x = o.sample(W, LENS, E, None, 1, wl.grid_h, wl.grid_w, wl.steps, wl.guidance, wl.seed)
        rec["sample_steps"] = np.array(wl.steps)
        rec["sample_disp"] = _f16(x - z)
        return rec
    # CFG workloads: the first forward of the sample is the forward reference
    S_full = 2 if name == "cfg_1024" else 1
    trace: list = []
    x = o.sample(W, LENS, E, None, 1, wl.grid_h, wl.grid_w, S_full, wl.guidance, wl.seed, trace=trace)
    (t0, c0, X0, vc), (t1, c1, X1, vu) = trace[0], trace[1]
    assert t0 == t1 == 1.0 and c0 and not c1 and np.array_equal(X0, X1)
    rec["fwd_t"] = np.array([1.0, 1.0])
    rec["fwd_input"] = np.array("noise")
    rec["fwd_v"] = _f16(np.concatenate([vc, vu]))           # rows: conditional, zero text
    rec["sample_steps"] = np.array(S_full)
    rec["sample_disp"] = _f16(x - z)
    # the first step of the workload's own grid: the oracle's step loop over the two
    # velocities above (both grids start at t = 1 on the same noise)
    C = LENS.latent_channels
    first = {True: o.unpatchify(vc, wl.grid_h, wl.grid_w, C), False: o.unpatchify(vu, wl.grid_h, wl.grid_w, C)}

    def cached(xx, t, cond):
        assert t == 1.0 and np.array_equal(xx, z)
        return first[cond]

    xs = o.sample_euler(cached, z, wl.steps, wl.guidance, stop_after=1)
    rec["grid_steps"] = np.array(wl.steps)
    rec["grid_disp_after_1"] = _f16(xs - z)
    return rec


def main(names) -> None:
    os.makedirs(OUT, exist_ok=True)
    t0 = time.time()
    W = o.Weights(make_weights(LENS, seed=0))
    print(f"weights ready in {time.time() - t0:.0f} s", flush=True)
    for name in names:
        t1 = time.time()
        rec = make(name, W)
        np.savez_compressed(os.path.join(OUT, name + ".npz"), **rec)
        print(f"{name}: {time.time() - t1:.0f} s", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:] or ["turbo_1024", "cfg_1024", "cfg_1440", "cfg_1024x2048"])
