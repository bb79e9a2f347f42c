"""The full 48-block denoiser on the GPU against the fp64 oracle: the 512^2 forward
computed on the spot, and the 1024^2, 1440^2 and 1024x2048 workloads against oracle
references written offline by tests/golden/make_full_refs.py (a 48-block oracle
forward there takes minutes).  Each of those workloads is checked on one forward
(velocity cosine >= 0.995 per batch row), on a complete sample with the library's
fused sampler (final latent cosine >= 0.99, and the same bar on the displacement
latent - noise, which the denoiser decides), and, for the CFG workloads, on the first
step of their own 20- or 50-step grid run as a CFG split over two handles.  The
sample references use reduced step counts (4 at 1024^2 Turbo, 2 at 1024^2 CFG, 1 at
1440^2 and 1024x2048): the oracle cannot run 20 or 50 steps of 48 blocks.  The
composed-Euler checks below stay as plumbing checks of the sampler."""
import os

import numpy as np
import pytest

from lens_inputs import LENS, WORKLOADS, image_tokens, make_weights, text_features
from oracle import lens_oracle as o
from tests.helpers import cos_sim, dev, host, rel_l2

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import flow_matching_mmdit_b200 as L  # noqa: E402


@pytest.fixture(scope="module")
def full():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = make_weights(LENS, seed=0)
    cfg = L.lens_dit_default_config()
    cfg.max_batch, cfg.max_img_tokens, cfg.max_txt_tokens = 2, 8192, 256
    h = L.lens_dit_create(cfg, w)
    yield w, h
    h.destroy()


def test_forward_48_blocks_512(full):
    """48 blocks at 512^2: 32x32 image tokens + 128 text tokens, t = 0.5."""
    w, h = full
    wl = WORKLOADS["fwd_512"]
    X = image_tokens(1, wl.n_img, wl.seed)
    E = text_features(1, wl.n_txt, wl.seed)
    v = torch.empty((1, wl.n_img, 128), dtype=torch.float32, device="cuda")
    L.lens_dit_forward(h, dev(X), 1, wl.grid_h, wl.grid_w, dev(E), wl.n_txt, [wl.t], v)
    L.lens_dit_sync(h)
    ref = o.forward(o.Weights(w), LENS, X, wl.grid_h, wl.grid_w, E, [wl.t])
    got = host(v)
    c, r = cos_sim(got, ref), rel_l2(got, ref)
    print(f"48-block 512^2 velocity: cosine {c:.7f}, rel L2 {r:.3e}")
    assert c >= 0.995


FULL_REFS = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "full")
FULL_NAMES = ["turbo_1024", "cfg_1024", "cfg_1440", "cfg_1024x2048"]


def _full_ref(name):
    p = os.path.join(FULL_REFS, name + ".npz")
    if not os.path.exists(p):
        pytest.skip(f"no oracle reference for {name} (tests/golden/make_full_refs.py writes it)")
    return np.load(p)


def _oracle_noise(wl):
    """The oracle's seeded noise latent [1, 32, 2h, 2w] (fp32, as the sampler starts)."""
    n = 32 * 2 * wl.grid_h * 2 * wl.grid_w
    return o.noise(wl.seed, n).reshape(1, 32, 2 * wl.grid_h, 2 * wl.grid_w)


@pytest.mark.parametrize("name", FULL_NAMES)
def test_forward_48_blocks_vs_oracle_reference(full, name):
    """One 48-block forward at the workload's size against the oracle's: the 1024^2
    Turbo reference is a forward at t = 1/2 on N(0, 1) tokens; the CFG references are
    the first forward of the CFG sample (t = 1 on the oracle's noise, rows: the
    conditional text and the zero text)."""
    w, h = full
    wl = WORKLOADS[name]
    r = _full_ref(name)
    E = text_features(1, wl.n_txt, wl.seed)
    if str(r["fwd_input"]) == "image_tokens":
        X, Eb = image_tokens(1, wl.n_img, wl.seed), E
    else:
        X0 = o.patchify(_oracle_noise(wl))
        X, Eb = np.concatenate([X0, X0]), np.concatenate([E, np.zeros_like(E)])
    t = [float(x) for x in r["fwd_t"]]
    rows = X.shape[0]
    v = torch.empty((rows, wl.n_img, 128), dtype=torch.float32, device="cuda")
    L.lens_dit_forward(h, dev(np.ascontiguousarray(X, np.float32)), rows, wl.grid_h, wl.grid_w, dev(Eb), wl.n_txt,
                       t, v)
    L.lens_dit_sync(h)
    got, ref = host(v), r["fwd_v"].astype(np.float64)
    for b in range(rows):
        c, e = cos_sim(got[b], ref[b]), rel_l2(got[b], ref[b])
        print(f"{name} forward row {b}: cosine {c:.7f}, rel L2 {e:.3e}")
        assert c >= 0.995


@pytest.mark.parametrize("name", FULL_NAMES)
def test_sampler_vs_oracle_reference(full, name):
    """The library's fused sampler (lens_sample_euler) over the reference's step count,
    at the workload's guidance, against the oracle's latent."""
    w, h = full
    wl = WORKLOADS[name]
    r = _full_ref(name)
    S = int(r["sample_steps"])
    Ec = dev(text_features(1, wl.n_txt, wl.seed))
    out = torch.empty((1, 32, 2 * wl.grid_h, 2 * wl.grid_w), dtype=torch.float32, device="cuda")
    L.lens_sample_euler(h, Ec, None, 1, wl.n_txt, wl.height_px, wl.width_px, S, wl.guidance, wl.seed, out)
    L.lens_dit_sync(h)
    z = _oracle_noise(wl).astype(np.float64)
    got, disp = host(out).astype(np.float64), r["sample_disp"].astype(np.float64)
    c_lat, c_disp = cos_sim(got, z + disp), cos_sim(got - z, disp)
    print(f"{name} sampler, {S} step(s): latent cosine {c_lat:.7f}, displacement cosine {c_disp:.7f}, "
          f"rel L2 {rel_l2(got - z, disp):.3e}")
    assert c_lat >= 0.99 and c_disp >= 0.99


@pytest.mark.parametrize("name", ["cfg_1024", "cfg_1440", "cfg_1024x2048"])
def test_cfg_split_first_step_vs_oracle_reference(full, name):
    """The CFG split (two handles standing in for the two ranks of a pair, the exchange
    a shared buffer) over the first step of the workload's own 20- or 50-step grid,
    against the oracle; both halves hold the same latent."""
    w, h = full
    wl = WORKLOADS[name]
    r = _full_ref(name)
    cfg = L.lens_dit_default_config()
    cfg.max_batch, cfg.max_img_tokens, cfg.max_txt_tokens = 1, wl.n_img, wl.n_txt
    h2 = L.lens_dit_create(cfg, w)
    try:
        opt = L.lens_sampler_default_options()
        opt.guidance = wl.guidance
        Ec = dev(text_features(1, wl.n_txt, wl.seed))
        S = int(r["grid_steps"])
        L.lens_sampler_prepare(h, Ec, None, 1, wl.n_txt, wl.height_px, wl.width_px, S, opt, wl.seed)
        L.lens_sampler_prepare(h2, None, None, 1, wl.n_txt, wl.height_px, wl.width_px, S, opt, wl.seed)
        v_all = torch.empty((2, 1, wl.n_img, 128), dtype=torch.float32, device="cuda")
        L.lens_sampler_velocity(h, 0, v_all[0])
        L.lens_sampler_velocity(h2, 0, v_all[1])
        L.lens_sampler_update(h, 0, v_all[0], v_all[1])
        L.lens_sampler_update(h2, 0, v_all[0], v_all[1])
        outs = [torch.empty((1, 32, 2 * wl.grid_h, 2 * wl.grid_w), dtype=torch.float32, device="cuda")
                for _ in range(2)]
        L.lens_sampler_finish(h, outs[0])
        L.lens_sampler_finish(h2, outs[1])
        L.lens_dit_sync(h)
        L.lens_dit_sync(h2)
        a, b = host(outs[0]), host(outs[1])
        assert np.array_equal(a, b)
        z = _oracle_noise(wl).astype(np.float64)
        disp = r["grid_disp_after_1"].astype(np.float64)
        c_lat, c_disp = cos_sim(a, z + disp), cos_sim(a - z, disp)
        print(f"{name} CFG split, step 1 of {S}: latent cosine {c_lat:.9f}, displacement cosine {c_disp:.7f}")
        assert c_lat >= 0.99 and c_disp >= 0.99
    finally:
        h2.destroy()


def _composed(h, Ec, B, gh, gw, nt, steps, guidance, seed, gpu_euler=False, mu=None, phi=0.0):
    """Oracle Euler/CFG loop whose velocity field is the library's forward.  With
    gpu_euler the update runs through the library's fp32 Euler/CFG op instead of
    the oracle's fp64 one, so the two sides round identically.  mu / phi select the
    shifted grid and the norm-rescaled CFG."""
    Ni = gh * gw
    x = torch.empty((B, Ni, 128), dtype=torch.float32, device="cuda")
    L.lens_op_noise_tokens(seed, B, gh, gw, x)
    xk = host(x).astype(np.float64)
    cfg = guidance != 1.0
    E = torch.cat([Ec, torch.zeros_like(Ec)]) if cfg else Ec
    rows = 2 * B if cfg else B
    v = torch.empty((rows, Ni, 128), dtype=torch.float32, device="cuda")
    grid = o.time_grid(steps, mu)
    for k in range(steps):
        t = grid[k]
        dt = 1.0 / steps if mu is None else float(np.float32(grid[k] - grid[k + 1]))
        xin = np.concatenate([xk, xk]) if cfg else xk
        L.lens_dit_forward(h, dev(xin.astype(np.float32)), rows, gh, gw, E, nt, [float(np.float32(t))] * rows, v)
        if gpu_euler:
            xd = dev(xk.astype(np.float32))
            if cfg and phi != 0.0:
                L.lens_dit_op_euler_cfg_rescaled(h, xd, v[:B], v[B:], B, Ni * 128, dt, guidance, phi)
            else:
                L.lens_op_euler_cfg(xd, v[:B], v[B:] if cfg else None, xd.numel(), dt, guidance)
            xk = host(xd).astype(np.float64)
            continue
        vv = host(v).astype(np.float64)
        vel = vv if not cfg else (o.cfg_combine(vv[:B], vv[B:], guidance) if phi == 0.0 else
                                  o.cfg_rescaled(vv[:B], vv[B:], guidance, phi))
        xk = o.euler(xk, vel, dt)
        xk = xk.astype(np.float32).astype(np.float64)      # the sampler keeps its state in fp32
    return o.unpatchify(xk, gh, gw, 32)


@pytest.mark.parametrize("name,steps", [("turbo_1024", 4), ("cfg_1024", 2), ("cfg_1440", 2), ("cfg_1024x2048", 1)])
def test_sampler_is_euler_over_forward(full, name, steps):
    w, h = full
    wl = WORKLOADS[name]
    B = 1
    Ec = dev(text_features(B, wl.n_txt, wl.seed))
    out = torch.empty((B, 32, 2 * wl.grid_h, 2 * wl.grid_w), dtype=torch.float32, device="cuda")
    L.lens_sample_euler(h, Ec, None, B, wl.n_txt, wl.height_px, wl.width_px, steps, wl.guidance, wl.seed, out)
    L.lens_dit_sync(h)
    got = host(out)
    assert np.all(np.isfinite(got))
    # (a) plumbing: the same fp32 update through the library's own Euler/CFG op
    same = _composed(h, Ec, B, wl.grid_h, wl.grid_w, wl.n_txt, steps, wl.guidance, wl.seed, gpu_euler=True)
    assert rel_l2(got, same) < 1e-6, rel_l2(got, same)
    # (b) the oracle's fp64 Euler/CFG over the same forwards.  Under CFG the fp32
    # combine rounds differently from fp64; those ulp-level input changes are
    # amplified through the bf16 operands of the next forward and by the guidance
    # scale, so the bar is the sampler bar (cosine >= 0.99), not bit-exactness.
    ref = _composed(h, Ec, B, wl.grid_h, wl.grid_w, wl.n_txt, steps, wl.guidance, wl.seed)
    c, r = cos_sim(got, ref), rel_l2(got, ref)
    print(f"{name}: sampler vs composed forwards: cosine {c:.9f}, rel L2 {r:.3e}")
    assert c >= 0.99 and r < 5e-2


@pytest.mark.parametrize("name,steps,phi,shift", [("turbo_1024", 4, 0.0, True), ("cfg_1024", 2, 1.0, True),
                                                  ("cfg_1440", 2, 1.0, False)])
def test_sampler_variants_are_euler_over_forward(full, name, steps, phi, shift):
    """Shifted grid (mu from the pages' 512^2 anchor and a 1.15 anchor at 4096
    tokens) and norm-rescaled CFG at full sizes, checked as for the plain sampler."""
    w, h = full
    wl = WORKLOADS[name]
    B = 1
    mu = L.lens_shift_mu(wl.grid_h * wl.grid_w, 1024, 1.06, 4096, 1.15) if shift else None
    opt = L.lens_sampler_default_options()
    opt.guidance, opt.cfg_rescale = wl.guidance, phi
    if shift:
        opt.time_shift, opt.shift_mu = 1, mu
    mu32 = None if mu is None else float(np.float32(mu))
    Ec = dev(text_features(B, wl.n_txt, wl.seed))
    out = torch.empty((B, 32, 2 * wl.grid_h, 2 * wl.grid_w), dtype=torch.float32, device="cuda")
    L.lens_sample_euler_ex(h, Ec, None, None, None, B, wl.n_txt, wl.height_px, wl.width_px, steps, opt, wl.seed, out)
    L.lens_dit_sync(h)
    got = host(out)
    assert np.all(np.isfinite(got))
    same = _composed(h, Ec, B, wl.grid_h, wl.grid_w, wl.n_txt, steps, wl.guidance, wl.seed, gpu_euler=True,
                     mu=mu32, phi=phi)
    assert rel_l2(got, same) < 1e-6, rel_l2(got, same)
    ref = _composed(h, Ec, B, wl.grid_h, wl.grid_w, wl.n_txt, steps, wl.guidance, wl.seed, mu=mu32, phi=phi)
    c, r = cos_sim(got, ref), rel_l2(got, ref)
    print(f"{name} variant (phi {phi}, shift {shift}): cosine {c:.9f}, rel L2 {r:.3e}")
    assert c >= 0.99 and r < 5e-2


def test_w4_model_footprint_and_single_pass_fidelity(full):
    """The 48-block model with weight_bits = 4: device bytes taken by create (the page
    gives about 2.35 GB of weights) and the single-forward cosine against the bf16
    model at 512^2 (the page reports 0.9976 for trained weights against PyTorch; these
    are random weights, so the figure is a measurement, not a bar)."""
    w_bf, h_bf = full
    wl = WORKLOADS["fwd_512"]
    free0 = torch.cuda.mem_get_info()[0]
    cfg = L.lens_dit_default_config()
    cfg.weight_bits = 4
    cfg.max_batch, cfg.max_img_tokens, cfg.max_txt_tokens = 2, 4096, 256
    h4 = L.lens_dit_create(cfg, w_bf)
    try:
        used = free0 - torch.cuda.mem_get_info()[0]
        B = 1
        X = dev(image_tokens(B, wl.n_img, wl.seed))
        E = dev(text_features(B, wl.n_txt, wl.seed))
        v4 = torch.empty((B, wl.n_img, 128), dtype=torch.float32, device="cuda")
        vb = torch.empty_like(v4)
        L.lens_dit_forward(h4, X, B, wl.grid_h, wl.grid_w, E, wl.n_txt, [wl.t], v4)
        L.lens_dit_forward(h_bf, X, B, wl.grid_h, wl.grid_w, E, wl.n_txt, [wl.t], vb)
        L.lens_dit_sync(h4)
        c = cos_sim(host(v4), host(vb))
        print(f"int4 model: create took {used / 1e9:.2f} GB of device memory; single pass cosine vs bf16 {c:.5f}")
        assert used < 4.0e9 and np.all(np.isfinite(host(v4))) and c > 0.9
    finally:
        h4.destroy()
