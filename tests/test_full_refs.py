"""The stored oracle references for the full-size workloads (tests/golden/full, written
by tests/golden/make_full_refs.py) are checked for shape and internal consistency on the
CPU: for a one-step CFG sample the latent moves by -unpatchify(u + s (c - u)), where c
and u are the two stored forward rows (conditional first), and the first step of the
S-step grid moves by 1/S of that.  A swapped row order, a wrong guidance or a
mislabelled file fails here."""
import os

import numpy as np
import pytest

from lens_inputs import WORKLOADS
from oracle import lens_oracle as o

FULL = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "full")
NAMES = ["turbo_1024", "cfg_1024", "cfg_1440", "cfg_1024x2048"]


def _load(name):
    p = os.path.join(FULL, name + ".npz")
    if not os.path.exists(p):
        pytest.skip(f"{name} reference not written")
    return np.load(p)


@pytest.mark.parametrize("name", NAMES)
def test_reference_shapes_and_values(name):
    r, wl = _load(name), WORKLOADS[name]
    assert str(r["workload"]) == name and int(r["seed"]) == wl.seed
    rows = 1 if wl.guidance == 1.0 else 2
    assert r["fwd_v"].shape == (rows, wl.n_img, 128)
    assert r["sample_disp"].shape == (1, 32, 2 * wl.grid_h, 2 * wl.grid_w)
    for k in ("fwd_v", "sample_disp"):
        v = r[k].astype(np.float64)
        assert np.all(np.isfinite(v)) and 0.1 < np.sqrt(np.mean(v * v)) < 100.0
    if rows == 2:
        assert int(r["grid_steps"]) == wl.steps and r["grid_disp_after_1"].shape == r["sample_disp"].shape


@pytest.mark.parametrize("name", ["cfg_1440", "cfg_1024x2048"])
def test_one_step_cfg_references_agree_with_their_forward(name):
    r, wl = _load(name), WORKLOADS[name]
    assert int(r["sample_steps"]) == 1
    c, u = (r["fwd_v"][i].astype(np.float64)[None] for i in (0, 1))
    step = -o.unpatchify(u + wl.guidance * (c - u), wl.grid_h, wl.grid_w, 32)
    disp = r["sample_disp"].astype(np.float64)
    # float16 storage: about 2^-11 relative per stored value
    assert np.linalg.norm(disp - step) / np.linalg.norm(step) < 5e-3
    grid = r["grid_disp_after_1"].astype(np.float64)
    assert np.linalg.norm(grid * wl.steps - step) / np.linalg.norm(step) < 5e-3
