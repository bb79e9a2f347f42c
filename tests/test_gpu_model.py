"""GPU parity of the denoiser through the C ABI (handle API) against the CPU oracle.

Bars (floating point; the oracle runs in fp64 on the same bf16 weights):
  one block         cosine >= 0.9995 and relative L2 <= 1e-2 on the block output and
                    on its update (h_out - h_in), which carries all the rounding
  48-block forward  velocity cosine >= 0.995
  sampler           final latent cosine >= 0.99
Large sequences are checked on sampled query rows the oracle computes one by one
(keys and values always cover every token)."""
import numpy as np
import pytest

from lens_inputs import LENS, WORKLOADS, image_tokens, make_weights, text_features
from oracle import lens_oracle as o
from tests.helpers import bf16_to_f64, cos_sim, dev, host, rel_l2

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import flow_matching_mmdit_b200 as L  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L.load_library()


def _handle(weights, blocks, max_batch, max_img, max_txt, max_t=64):
    cfg = L.lens_dit_default_config()
    cfg.num_blocks = blocks
    cfg.max_batch, cfg.max_img_tokens, cfg.max_txt_tokens, cfg.max_timesteps = max_batch, max_img, max_txt, max_t
    return L.lens_dit_create(cfg, weights)


@pytest.fixture(scope="module")
def small():
    """Two-block model with random biases and gains (so every term is exercised)."""
    d = LENS.with_blocks(2)
    w = make_weights(d, seed=0, bias_std=0.02, gain_std=0.1)
    h = _handle(w, 2, max_batch=4, max_img=8192, max_txt=256)
    yield d, w, h
    h.destroy()


def _sync(h):
    L.lens_dit_sync(h)


# ------------------------------------------------------------------ step-invariant heads
def test_timestep_embedding_and_modulation(small):
    d, w, h = small
    W = o.Weights(w)
    t = [0.7, 0.0, 1.0, 0.333]
    T = len(t)
    modw = d.num_blocks * 2 * 9216 + 3072
    temb = torch.empty((T, 1536), dtype=torch.float32, device="cuda")
    mod = torch.empty((T, modw), dtype=torch.float32, device="cuda")
    L.lens_dit_op_timestep(h, t, temb, mod)
    _sync(h)
    ref_t = o.timestep_embedding(W, np.array(t), 256)
    assert rel_l2(host(temb), ref_t) < 1e-5
    got = host(mod)
    for i in range(d.num_blocks):
        for s, name in enumerate(("img_mod", "txt_mod")):
            ref = np.concatenate(o.modulation(W, f"transformer_blocks.{i}.{name}", ref_t, 6), axis=-1)
            part = got[:, i * 18432 + s * 9216:i * 18432 + (s + 1) * 9216]
            # the GEMM operand SiLU(temb) is rounded to bf16 once
            assert cos_sim(part, ref) > 0.99999 and rel_l2(part, ref) < 5e-3
    ref_no = np.concatenate(o.modulation(W, "norm_out.linear", ref_t, 2), axis=-1)
    assert rel_l2(got[:, d.num_blocks * 18432:], ref_no) < 5e-3


@pytest.mark.parametrize("B,nt", [(1, 16), (2, 256), (3, 1)])
def test_text_input(small, B, nt):
    d, w, h = small
    E = text_features(B, nt, seed=nt)
    c = torch.empty((B, nt, 1536), dtype=torch.float32, device="cuda")
    L.lens_dit_op_text_input(h, dev(E), B, nt, c)
    _sync(h)
    ref = o.text_input(o.Weights(w), bf16_to_f64(E), d.eps)
    # normalised features are rounded to bf16 once before the 11520-deep GEMM
    assert cos_sim(host(c), ref) > 0.99999 and rel_l2(host(c), ref) < 3e-3


# ------------------------------------------------------------------ one block
def _block_case(w, d, B, gh, gw, nt, seed):
    W = o.Weights(w)
    X = image_tokens(B, gh * gw, seed)
    E = text_features(B, nt, seed)
    h_img = o.linear(W, "img_in", X.astype(np.float64))
    h_txt = o.text_input(W, bf16_to_f64(E), d.eps)
    return W, h_img.astype(np.float32), h_txt.astype(np.float32)


def _check_block(got_i, got_t, ref_i, ref_t, in_i, in_t):
    for got, ref, x in ((got_i, ref_i, in_i), (got_t, ref_t, in_t)):
        assert cos_sim(got, ref) >= 0.9995 and rel_l2(got, ref) <= 1e-2
        assert cos_sim(got - x, ref - x) >= 0.9995 and rel_l2(got - x, ref - x) <= 1e-2, \
            (cos_sim(got - x, ref - x), rel_l2(got - x, ref - x))


def test_block_parity_8x8(small):
    """One block, 8x8 image tokens + 16 text tokens, t = 0.7, batch 1."""
    d, w, h = small
    wl = WORKLOADS["block_8x8"]
    W, hi, ht = _block_case(w, d, 1, wl.grid_h, wl.grid_w, wl.n_txt, wl.seed)
    hi_d, ht_d = dev(hi), dev(ht)
    L.lens_dit_debug_blocks(h, 0, 1, hi_d, ht_d, 1, wl.grid_h, wl.grid_w, wl.n_txt, [wl.t])
    _sync(h)
    temb = o.timestep_embedding(W, np.array([wl.t]), 256)
    ang = o.rope_angles(o.position_ids(wl.grid_h, wl.grid_w, wl.n_txt), d.rope_axes, d.rope_theta)
    ri, rt = o.block(W, 0, hi.astype(np.float64), ht.astype(np.float64), temb, ang, d.heads, d.eps)
    _check_block(host(hi_d), host(ht_d), ri, rt, hi, ht)


@pytest.mark.parametrize("B,gh,gw,nt", [(2, 64, 64, 256), (2, 90, 90, 256), (2, 64, 128, 256), (1, 5, 7, 3)])
def test_block_parity_sampled_rows(small, B, gh, gw, nt):
    """Full-size sequences (1024^2, 1440^2, 1024x2048 with CFG batch 2) and a
    ragged tiny one: block 1 on sampled query rows."""
    d, w, h = small
    W, hi, ht = _block_case(w, d, B, gh, gw, nt, seed=gh + gw)
    hi_d, ht_d = dev(hi), dev(ht)
    t = [0.5, 0.25][:B]
    L.lens_dit_debug_blocks(h, 1, 2, hi_d, ht_d, B, gh, gw, nt, t)
    _sync(h)
    rng = np.random.default_rng(1)
    ni = gh * gw
    ir = np.unique(np.r_[0, ni - 1, rng.choice(ni, size=min(ni, 96), replace=False)])
    tr = np.unique(np.r_[0, nt - 1, rng.choice(nt, size=min(nt, 16), replace=False)])
    temb = o.timestep_embedding(W, np.array(t), 256)
    ang = o.rope_angles(o.position_ids(gh, gw, nt), d.rope_axes, d.rope_theta)
    ri, rt = o.block(W, 1, hi.astype(np.float64), ht.astype(np.float64), temb, ang, d.heads, d.eps,
                     img_rows=ir, txt_rows=tr)
    _check_block(host(hi_d)[:, ir], host(ht_d)[:, tr], ri, rt, hi[:, ir], ht[:, tr])


def test_block_without_text(small):
    """n_txt = 0: the joint attention reduces to image self-attention."""
    d, w, h = small
    W, hi, _ = _block_case(w, d, 1, 6, 6, 0, seed=4)
    hi_d = dev(hi)
    L.lens_dit_debug_blocks(h, 0, 1, hi_d, None, 1, 6, 6, 0, [0.9])
    _sync(h)
    temb = o.timestep_embedding(W, np.array([0.9]), 256)
    ang = o.rope_angles(o.position_ids(6, 6, 0), d.rope_axes, d.rope_theta)
    ri, rt = o.block(W, 0, hi.astype(np.float64), np.zeros((1, 0, 1536)), temb, ang, d.heads, d.eps)
    got = host(hi_d)
    assert cos_sim(got - hi, ri - hi) >= 0.9995 and rel_l2(got - hi, ri - hi) <= 1e-2


# ------------------------------------------------------------------ forward and sampler, small model
def test_forward_two_blocks(small):
    d, w, h = small
    B, gh, gw, nt = 2, 8, 8, 16
    X = image_tokens(B, gh * gw, 11)
    E = text_features(B, nt, 11)
    t = [0.7, 0.2]
    v = torch.empty((B, gh * gw, 128), dtype=torch.float32, device="cuda")
    L.lens_dit_forward(h, dev(X), B, gh, gw, dev(E), nt, t, v)
    _sync(h)
    ref = o.forward(o.Weights(w), d, X, gh, gw, E, t)
    assert cos_sim(host(v), ref) >= 0.999 and rel_l2(host(v), ref) <= 2e-2


@pytest.mark.parametrize("guidance,steps", [(1.0, 4), (5.0, 3)])
def test_sampler_two_blocks(small, guidance, steps):
    d, w, h = small
    B, gh, gw, nt, seed = 2, 8, 6, 16, 1234
    Ec = text_features(B, nt, 21)
    out = torch.empty((B, 32, 2 * gh, 2 * gw), dtype=torch.float32, device="cuda")
    L.lens_sample_euler(h, dev(Ec), None, B, nt, 16 * gh, 16 * gw, steps, guidance, seed, out)
    _sync(h)
    ref = o.sample(o.Weights(w), d, Ec, None, B, gh, gw, steps, guidance, seed)
    got = host(out)
    assert cos_sim(got, ref) >= 0.99 and rel_l2(got, ref) <= 5e-2, (cos_sim(got, ref), rel_l2(got, ref))
    # with a single step from pure noise the output is noise - v(noise, 1)
    assert np.all(np.isfinite(got))


def test_argument_validation(small):
    d, w, h = small
    x = torch.zeros((1, 64, 128), device="cuda")
    e = torch.zeros((1, 16, 4, 2880), dtype=torch.int16, device="cuda")
    with pytest.raises(L.LensError) as ei:
        L.lens_dit_forward(h, x, 1, 100, 100, e, 16, [0.5], x)            # grid beyond capacity
    assert ei.value.status == 2
    with pytest.raises(L.LensError) as ei:
        L.lens_sample_euler(h, e, None, 1, 16, 100, 128, 2, 1.0, 0, x)   # height not a multiple of 16
    assert ei.value.status == 2
    with pytest.raises(L.LensError) as ei:
        L.lens_sample_euler(h, e, None, 1, 16, 128, 128, 0, 1.0, 0, x)   # steps < 1
    assert ei.value.status == 1
    with pytest.raises(L.LensError) as ei:
        L.lens_sample_euler(h, e, None, 3, 16, 128, 128, 2, 5.0, 0, x)   # 2 x 3 CFG rows > max_batch 4
    assert ei.value.status == 2
    with pytest.raises(L.LensError) as ei:
        L.lens_dit_debug_blocks(h, 1, 3, x, None, 1, 8, 8, 0, [0.5])     # block range beyond num_blocks
    assert ei.value.status == 2


def test_create_rejects_bad_weights():
    d = LENS.with_blocks(1)
    w = make_weights(d, seed=3)
    bad = dict(w)
    bad["transformer_blocks.0.attn.img_qkv.weight"] = np.zeros((4608, 1535), np.uint16)
    with pytest.raises(L.LensError) as ei:
        _handle(bad, 1, 1, 64, 16)
    assert ei.value.status == 2
    bad = dict(w)
    del bad["proj_out.weight"]
    with pytest.raises(L.LensError) as ei:
        _handle(bad, 1, 1, 64, 16)
    assert ei.value.status == 1
    bad = dict(w)
    bad["not_a_tensor.weight"] = np.zeros(3, np.uint16)
    with pytest.raises(L.LensError) as ei:
        _handle(bad, 1, 1, 64, 16)
    assert ei.value.status == 1
    cfg = L.lens_dit_default_config()
    cfg.hidden = 1024
    with pytest.raises(L.LensError) as ei:
        L.lens_dit_create(cfg, w)
    assert ei.value.status == 6


def test_sampler_graph_capture_replays_exactly(small):
    """On a created stream the sampler call is captured as a CUDA graph and replayed;
    the result must match the direct launches on the default stream bit for bit,
    and a changed argument must re-capture."""
    d, w, h = small
    B, gh, gw, nt = 1, 8, 8, 16
    E = dev(text_features(B, nt, 31))
    ref = torch.empty((B, 32, 2 * gh, 2 * gw), dtype=torch.float32, device="cuda")
    L.lens_sample_euler(h, E, None, B, nt, 16 * gh, 16 * gw, 3, 5.0, 77, ref)     # default stream: direct
    _sync(h)
    s = torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(s):
        o = torch.empty_like(ref)                                 # the same output pointer each call
        counts = []
        for seed in (77, 77, 78, 77):
            n0 = L.lens_dit_launch_count(h)
            L.lens_sample_euler(h, E, None, B, nt, 16 * gh, 16 * gw, 3, 5.0, seed, o)
            L.lens_dit_sync(h, s)
            counts.append(L.lens_dit_launch_count(h) - n0)
            outs.append(host(o).copy())
    assert counts[0] > 50 and len(set(counts)) == 1               # replays count their kernels too
    assert np.array_equal(outs[0], host(ref)) and np.array_equal(outs[1], host(ref))
    assert not np.array_equal(outs[2], host(ref))                 # new seed: re-captured
    assert np.array_equal(outs[3], host(ref))


def test_forward_text_padding(small):
    """Padded text tokens are never attended: the velocity matches the masked oracle,
    and changing the padding's features changes nothing (bit for bit)."""
    d, w, h = small
    B, gh, gw, nt = 2, 8, 8, 16
    X = image_tokens(B, gh * gw, 41)
    E = text_features(B, nt, 41)
    lens, t = [6, 16], [0.6, 0.3]
    v = torch.empty((B, gh * gw, 128), dtype=torch.float32, device="cuda")
    L.lens_dit_forward_masked(h, dev(X), B, gh, gw, dev(E), nt, lens, t, v)
    _sync(h)
    ref = o.forward(o.Weights(w), d, X, gh, gw, E, t, txt_len=lens)
    assert cos_sim(host(v), ref) >= 0.999 and rel_l2(host(v), ref) <= 2e-2
    E2 = E.copy()
    E2[0, 6:] = text_features(1, nt - 6, 99)[0]
    v2 = torch.empty_like(v)
    L.lens_dit_forward_masked(h, dev(X), B, gh, gw, dev(E2), nt, lens, t, v2)
    _sync(h)
    assert np.array_equal(host(v2), host(v))


def test_sampler_text_padding(small):
    d, w, h = small
    B, gh, gw, nt, seed = 1, 8, 8, 16, 5
    Ec = text_features(B, nt, 51)
    out = torch.empty((B, 32, 2 * gh, 2 * gw), dtype=torch.float32, device="cuda")
    L.lens_sample_euler_masked(h, dev(Ec), [9], None, [0], B, nt, 16 * gh, 16 * gw, 3, 5.0, seed, out)
    _sync(h)
    ref = o.sample(o.Weights(w), d, Ec, None, B, gh, gw, 3, 5.0, seed, len_cond=[9], len_uncond=[0])
    got = host(out)
    assert cos_sim(got, ref) >= 0.99 and rel_l2(got, ref) <= 5e-2, (cos_sim(got, ref), rel_l2(got, ref))


# ------------------------------------------------------------------ sampler variants
@pytest.mark.parametrize("B,per,phi", [(3, 128 * 37, 0.0), (3, 128 * 37, 0.5), (3, 128 * 37, 1.0),
                                       (2, 4096 * 128, 1.0), (1, 128, 0.25)])
def test_euler_cfg_rescaled_op(small, B, per, phi):
    """Norm-rescaled CFG + Euler against the oracle: per-sample norms over every
    value of the sample, so samples with different scales must not mix."""
    d, w, h = small
    rng = np.random.default_rng(31 + B)
    x, c, u = (rng.standard_normal((B, per)).astype(np.float32) for _ in range(3))
    u[-1] *= 3.0
    c[0] *= 0.2
    xd = dev(x)
    L.lens_dit_op_euler_cfg_rescaled(h, xd, dev(c), dev(u), B, per, 0.0625, 5.0, phi)
    _sync(h)
    ref = o.euler(x.astype(np.float64), o.cfg_rescaled(c.astype(np.float64), u.astype(np.float64), 5.0, phi), 0.0625)
    err = np.max(np.abs(host(xd) - ref))
    assert err <= 2e-5 * np.max(np.abs(ref)), err


def test_euler_cfg_rescaled_edge_cases(small):
    d, w, h = small
    B, per = 2, 256
    x = np.arange(B * per, dtype=np.float32).reshape(B, per) / 7.0
    z = np.zeros((B, per), np.float32)
    xd = dev(x)
    L.lens_dit_op_euler_cfg_rescaled(h, xd, dev(z), dev(z), B, per, 0.5, 5.0, 1.0)   # zero velocity: no move
    _sync(h)
    assert np.array_equal(host(xd), x)
    with pytest.raises(L.LensError) as e:
        L.lens_dit_op_euler_cfg_rescaled(h, xd, dev(z), dev(z), B, per, 0.5, 5.0, 1.5)
    assert e.value.status == 1
    with pytest.raises(L.LensError) as e:
        L.lens_dit_op_euler_cfg_rescaled(h, xd, dev(z), dev(z), 5, per, 0.5, 5.0, 1.0)  # > max_batch 4
    assert e.value.status == 2


def _options(guidance, phi, mu):
    opt = L.lens_sampler_default_options()
    opt.guidance, opt.cfg_rescale = guidance, phi
    if mu is not None:
        opt.time_shift, opt.shift_mu = 1, mu
    return opt


@pytest.mark.parametrize("guidance,phi,mu", [(5.0, 1.0, 1.2), (5.0, 0.5, None), (1.0, 0.0, 0.5), (4.0, 1.0, -0.3)])
def test_sampler_variants_two_blocks(small, guidance, phi, mu):
    d, w, h = small
    B, gh, gw, nt, seed, steps = 2, 8, 6, 16, 99, 3
    Ec = text_features(B, nt, 23)
    out = torch.empty((B, 32, 2 * gh, 2 * gw), dtype=torch.float32, device="cuda")
    L.lens_sample_euler_ex(h, dev(Ec), None, None, None, B, nt, 16 * gh, 16 * gw, steps, _options(guidance, phi, mu),
                           seed, out)
    _sync(h)
    mu64 = None if mu is None else float(np.float32(mu))
    ref = o.sample(o.Weights(w), d, Ec, None, B, gh, gw, steps, guidance, seed, mu=mu64, phi=phi)
    got = host(out)
    assert cos_sim(got, ref) >= 0.99 and rel_l2(got, ref) <= 5e-2, (cos_sim(got, ref), rel_l2(got, ref))


def test_sampler_options_are_part_of_the_replay_key(small):
    """Changing only the variant options on a created stream re-captures the graph."""
    d, w, h = small
    B, gh, gw, nt = 1, 8, 8, 16
    E = dev(text_features(B, nt, 41))
    shape = (B, 32, 2 * gh, 2 * gw)
    plain, resc = _options(5.0, 0.0, None), _options(5.0, 1.0, 0.8)
    refs = []
    for opt in (plain, resc):
        r = torch.empty(shape, dtype=torch.float32, device="cuda")
        L.lens_sample_euler_ex(h, E, None, None, None, B, nt, 16 * gh, 16 * gw, 3, opt, 5, r)   # direct
        _sync(h)
        refs.append(host(r).copy())
    assert not np.array_equal(refs[0], refs[1])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = torch.empty(shape, dtype=torch.float32, device="cuda")
        for opt, want in ((plain, 0), (resc, 1), (plain, 0), (plain, 0)):
            L.lens_sample_euler_ex(h, E, None, None, None, B, nt, 16 * gh, 16 * gw, 3, opt, 5, out)
            L.lens_dit_sync(h, s)
            assert np.array_equal(host(out), refs[want])


# ------------------------------------------------------------------ step-wise sampler / CFG split
@pytest.mark.parametrize("gh,gw,nt,steps,phi,mu", [(8, 6, 16, 3, 0.0, None), (64, 64, 256, 2, 1.0, 0.8)])
def test_cfg_split_halves_reproduce_the_fused_sampler(small, gh, gw, nt, steps, phi, mu):
    """Two handles stand in for the two ranks of a CFG pair (one GPU: run in turn,
    the exchange is a shared buffer).  Both end on the fused sampler's latent, bit
    for bit: a batch row's velocity does not depend on the other rows."""
    d, w, h = small
    h2 = _handle(w, 2, max_batch=4, max_img=8192, max_txt=256)
    try:
        B, seed = 1, 7
        Ec = dev(text_features(B, nt, 61))
        opt = _options(5.0, phi, mu)
        shape = (B, 32, 2 * gh, 2 * gw)
        ref = torch.empty(shape, dtype=torch.float32, device="cuda")
        L.lens_sample_euler_ex(h, Ec, None, None, None, B, nt, 16 * gh, 16 * gw, steps, opt, seed, ref)
        _sync(h)
        L.lens_sampler_prepare(h, Ec, None, B, nt, 16 * gh, 16 * gw, steps, opt, seed)
        L.lens_sampler_prepare(h2, None, None, B, nt, 16 * gh, 16 * gw, steps, opt, seed)
        v_all = torch.empty((2, B, gh * gw, 128), dtype=torch.float32, device="cuda")
        for k in range(steps):
            L.lens_sampler_velocity(h, k, v_all[0])
            L.lens_sampler_velocity(h2, k, v_all[1])
            L.lens_sampler_update(h, k, v_all[0], v_all[1])
            L.lens_sampler_update(h2, k, v_all[0], v_all[1])
        outs = [torch.empty(shape, dtype=torch.float32, device="cuda") for _ in range(2)]
        L.lens_sampler_finish(h, outs[0])
        L.lens_sampler_finish(h2, outs[1])
        _sync(h)
        assert np.array_equal(host(outs[0]), host(outs[1]))
        assert np.array_equal(host(outs[0]), host(ref))
        if gh * gw <= 64:
            # and against the oracle's sampler (affordable at this size)
            mu64 = None if mu is None else float(np.float32(mu))
            want = o.sample(o.Weights(w), d, text_features(B, nt, 61), None, B, gh, gw, steps, 5.0, seed, mu=mu64,
                            phi=phi)
            got = host(outs[0])
            assert cos_sim(got, want) >= 0.99 and rel_l2(got, want) <= 5e-2, (cos_sim(got, want), rel_l2(got, want))
    finally:
        h2.destroy()


def test_step_sampler_state_rules(small):
    d, w, h = small
    B, gh, gw, nt = 1, 4, 4, 16
    Ec = dev(text_features(B, nt, 62))
    opt = _options(1.0, 0.0, None)
    v = torch.empty((B, gh * gw, 128), dtype=torch.float32, device="cuda")
    L.lens_sampler_prepare(h, Ec, None, B, nt, 16 * gh, 16 * gw, 2, opt, 3)
    L.lens_sampler_velocity(h, 1, v)
    with pytest.raises(L.LensError) as e:
        L.lens_sampler_velocity(h, 2, v)                       # k past the last step
    assert e.value.status == 2
    with pytest.raises(L.LensError) as e:
        L.lens_sampler_prepare(h, Ec, None, B, nt, 16 * gh, 16 * gw, 65, opt, 3)   # > max_timesteps
    assert e.value.status == 2
    L.lens_sampler_prepare(h, Ec, None, B, nt, 16 * gh, 16 * gw, 2, opt, 3)
    X = dev(np.zeros((B, gh * gw, 128), np.float32))
    L.lens_dit_forward(h, X, B, gh, gw, Ec, nt, [0.5], v)       # reuses the buffers: state dropped
    with pytest.raises(L.LensError) as e:
        L.lens_sampler_update(h, 0, v, None)
    assert e.value.status == 1
    _sync(h)


# ------------------------------------------------------------------ failure path (no fault: a flag the test raises)
@pytest.mark.parametrize("gh,gw,nt", [(8, 8, 16), (32, 32, 128)])
def test_abort_flag_reports_timeout_then_recovers(small, gh, gw, nt):
    """With the device abort flag raised (as an expired wait would raise it) every
    kernel that waits leaves at its first wait that does not complete at once, after
    draining its own TMA copies and MMAs; lens_dit_sync reports LENS_ERR_TIMEOUT (5)
    and clears the flag, and the next forward matches the oracle again.  Nothing
    faults or hangs: the flag is the designed abort path."""
    d, w, h = small
    B = 2
    X = image_tokens(B, gh * gw, 31)
    E = text_features(B, nt, 32)
    t = [0.6, 0.2]
    v = torch.empty((B, gh * gw, 128), dtype=torch.float32, device="cuda")
    L.lens_dit_debug_raise_abort(h)
    L.lens_dit_forward(h, dev(X), B, gh, gw, dev(E), nt, t, v)
    with pytest.raises(L.LensError) as e:
        L.lens_dit_sync(h)
    assert e.value.status == 5
    _sync(h)                                         # the flag was cleared
    v.fill_(float("nan"))
    L.lens_dit_forward(h, dev(X), B, gh, gw, dev(E), nt, t, v)
    _sync(h)
    ref = o.forward(o.Weights(w), d, X, gh, gw, E, t)
    got = host(v)
    assert np.all(np.isfinite(got))
    assert cos_sim(got, ref) > 0.9999 and rel_l2(got, ref) < 1e-2
