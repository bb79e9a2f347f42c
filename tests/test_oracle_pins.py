"""Pins for the CPU oracle: checks against what the pages and the mathematics fix,
never against a retyped copy of the oracle's own formula.  CPU only."""
import math
import os

import numpy as np
import pytest

from lens_inputs import LENS, TINY, f32_to_bf16_bits, make_weights, weight_specs
from oracle import lens_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = [l.split() for l in open(os.path.join(GOLDEN, name)) if l.strip() and not l.startswith("#")]
    return rows


@pytest.fixture(scope="module")
def tinyW():
    return o.Weights(make_weights(TINY, seed=11, std=0.2, bias_std=0.05, gain_std=0.2))


# ------------------------------------------------------------------ model size
def test_param_count_matches_blog_arithmetic():
    g = {k: float(v) for k, v in _golden("lens_param_arithmetic.txt")}
    pc = o.param_count(LENS)
    D, F = LENS.hidden, LENS.mlp_hidden
    assert abs(4 * D * D / 1e6 - g["attn_proj_M"]) < 0.01
    assert abs(3 * D * F / 1e6 - g["mlp_M"]) < 0.1
    # the page adds rounded parts (28.2 + 14.1), so allow its rounding
    assert abs(pc["stream_weights"] / 1e6 - g["stream_M"]) / g["stream_M"] < 0.005
    assert abs(2 * pc["stream_weights"] / 1e6 - g["block_M"]) / g["block_M"] < 0.005
    assert abs(pc["total"] * 2 / 1e9 - g["bf16_GB"]) < 0.05
    # the synthetic tensor list holds exactly these parameters
    assert sum(int(np.prod(s)) for _, s, _ in weight_specs(LENS)) == pc["total"]


# ------------------------------------------------------------------ patchify
def test_patchify_roundtrip_and_grouping():
    rng = np.random.default_rng(0)
    Z = rng.standard_normal((2, 32, 6, 10)).astype(np.float32)
    X = o.patchify(Z)
    assert X.shape == (2, 15, 128)                       # 2*2*32 = 128 per token
    assert np.array_equal(o.unpatchify(X, 3, 5, 32), Z)  # bijection, bit-exact
    # token (i, j) holds exactly the 2x2 spatial block at (2i.., 2j..) of every channel
    for b in range(2):
        for i in range(3):
            for j in range(5):
                blk = Z[b, :, 2 * i:2 * i + 2, 2 * j:2 * j + 2].ravel()
                assert sorted(X[b, i * 5 + j].tolist()) == sorted(blk.tolist())
    # reading: features channel-major, then patch row, then patch column
    assert X[1, 7, 4 * 3 + 2 * 1 + 0] == Z[1, 3, 2 * 1 + 1, 2 * 2 + 0]


# ------------------------------------------------------------------ RoPE
def test_rope_axes_cover_head_dim():
    assert sum(LENS.rope_axes) == LENS.head_dim == 64


def test_rope_complex_brute_force():
    """Rotation of pair k equals multiplying (x0 + i x1) by exp(i angle)."""
    rng = np.random.default_rng(1)
    ids = rng.integers(0, 50, size=(7, 3))
    ang = o.rope_angles(ids, (8, 28, 28), 1e4)
    x = rng.standard_normal((7, 64))
    y = o.apply_rope(x, ang)
    for n in range(7):
        for k in range(32):
            c = complex(x[n, 2 * k], x[n, 2 * k + 1]) * complex(math.cos(ang[n, k]), math.sin(ang[n, k]))
            assert abs(y[n, 2 * k] - c.real) < 1e-12 and abs(y[n, 2 * k + 1] - c.imag) < 1e-12
    # the first pair of each axis turns by exactly pos (omega = 1); the axis owns its segment
    assert np.allclose(ang[:, 0], ids[:, 0]) and np.allclose(ang[:, 4], ids[:, 1]) and np.allclose(ang[:, 18], ids[:, 2])


def test_rope_norm_identity_and_relative_position():
    rng = np.random.default_rng(2)
    ids = o.position_ids(5, 7, 3)
    ang = o.rope_angles(ids, (8, 28, 28), 1e4)
    q = rng.standard_normal((ids.shape[0], 64))
    k = rng.standard_normal((ids.shape[0], 64))
    rq, rk = o.apply_rope(q, ang), o.apply_rope(k, ang)
    assert np.allclose(np.linalg.norm(rq, axis=1), np.linalg.norm(q, axis=1), rtol=0, atol=1e-12)
    assert np.array_equal(rq[:3], q[:3])       # text ids (0,0,0): identity
    # <R(p) q, R(p') k> depends only on p - p': shift every id by a constant
    ang2 = o.rope_angles(ids + np.array([3, 11, 5]), (8, 28, 28), 1e4)
    d1 = o.apply_rope(q, ang) @ o.apply_rope(k, ang).T
    d2 = o.apply_rope(q, ang2) @ o.apply_rope(k, ang2).T
    assert np.allclose(d1, d2, rtol=0, atol=1e-9)
    # a displacement along the width axis moves only dims [36, 64)
    a0 = o.rope_angles(np.array([[0, 2, 3]]), (8, 28, 28), 1e4)
    a1 = o.rope_angles(np.array([[0, 2, 4]]), (8, 28, 28), 1e4)
    x = rng.standard_normal((1, 64))
    diff = np.abs(o.apply_rope(x, a0) - o.apply_rope(x, a1))[0]
    assert diff[:36].max() == 0 and diff[36:].max() > 0


def test_position_ids_layout():
    ids = o.position_ids(2, 3, 2)
    assert ids.tolist() == [[0, 0, 0], [0, 0, 0], [0, 0, 0], [0, 0, 1], [0, 0, 2], [0, 1, 0], [0, 1, 1], [0, 1, 2]]


# ------------------------------------------------------------------ norms, activations, sinusoid
def test_rms_norm_and_silu_closed_forms():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 33)) * 7.0
    y = o.rms_norm(x, 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-12)
    assert np.allclose(o.rms_norm(5.0 * x, 0.0), y, atol=1e-12)
    g = rng.standard_normal(33)
    assert np.allclose(o.rms_norm(x, 0.0, g), y * g, atol=1e-12)
    assert o.silu(np.array(0.0)) == 0.0
    assert abs(o.silu(np.array(1.0)) - 0.7310585786300049) < 1e-15      # 1 / (1 + e^-1)
    assert abs(o.silu(np.array(40.0)) - 40.0) < 1e-12
    assert abs(o.silu(np.array(-40.0))) < 1e-15


def test_timestep_features():
    e0 = o.timestep_features(np.array([0.0]), 256)[0]
    assert np.array_equal(e0, np.r_[np.ones(128), np.zeros(128)])
    t = 0.37
    e = o.timestep_features(np.array([t]), 256)[0]
    assert abs(e[0] - math.cos(370.0)) < 1e-12 and abs(e[128] - math.sin(370.0)) < 1e-12
    # lowest frequency is 10000^(-127/128)
    assert abs(e[127] - math.cos(370.0 * 10000 ** (-127 / 128))) < 1e-12
    assert np.allclose(e[:128] ** 2 + e[128:] ** 2, 1.0)


# ------------------------------------------------------------------ attention
def _attn_loops(q, k, v):
    Nq, d = q.shape
    out = np.zeros((Nq, v.shape[1]))
    for i in range(Nq):
        s = [sum(q[i, c] * k[j, c] for c in range(d)) / math.sqrt(d) for j in range(k.shape[0])]
        m = max(s)
        w = [math.exp(x - m) for x in s]
        z = sum(w)
        for j in range(k.shape[0]):
            out[i] += w[j] / z * v[j]
    return out


def test_attention_brute_force_and_invariances():
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, 2, 5, 4)) * 2 for _ in range(3))
    out = o.attention(q, k, v)
    for h in range(2):
        assert np.allclose(out[0, h], _attn_loops(q[0, h], k[0, h], v[0, h]), atol=1e-12)
    perm = rng.permutation(5)
    assert np.allclose(o.attention(q, k[:, :, perm], v[:, :, perm]), out, atol=1e-12)
    assert np.allclose(o.attention(q[:, :, perm], k, v), out[:, :, perm], atol=1e-12)
    assert np.allclose(o.attention(np.zeros_like(q), k, v), v.mean(axis=2, keepdims=True), atol=1e-12)


# ------------------------------------------------------------------ text input
def test_text_input_per_layer_normalisation(tinyW):
    rng = np.random.default_rng(5)
    E = rng.standard_normal((2, 3, 4, TINY.txt_dim))
    c = o.text_input(tinyW, E, 0.0)
    E2 = E.copy()
    E2[:, :, 2, :] *= 9.0                       # each layer slice is normalised on its own
    assert np.allclose(o.text_input(tinyW, E2, 0.0), c, atol=1e-9)
    E3 = E.copy()
    E3[:, :, :, :] *= np.array([1, 2, 3, 4])[None, None, :, None]   # unequal per-layer scales:
    assert np.allclose(o.text_input(tinyW, E3, 0.0), c, atol=1e-9)
    z = o.text_input(tinyW, np.zeros_like(E), TINY.eps)
    assert np.allclose(z, tinyW("txt_in.bias")[None, None, :], atol=1e-15)


# ------------------------------------------------------------------ block
def _block_inputs(dims, B=2, Ni=6, Nt=3, seed=6):
    rng = np.random.default_rng(seed)
    h_img = rng.standard_normal((B, Ni, dims.hidden))
    h_txt = rng.standard_normal((B, Nt, dims.hidden)) * 2
    temb = rng.standard_normal((B, dims.hidden))
    return h_img, h_txt, temb


def _edit(W, fn):
    t = dict(W.t)
    fn(t)
    return o.Weights(t)


def _zero_rows(t, name, lo, hi):
    w = t[name + ".weight"].copy(); w[lo:hi] = 0; t[name + ".weight"] = w
    b = t[name + ".bias"].copy(); b[lo:hi] = 0; t[name + ".bias"] = b


def test_block_zero_gates_is_identity(tinyW):
    D = TINY.hidden

    def zero_gates(t):
        for s in ("img_mod", "txt_mod"):
            _zero_rows(t, f"transformer_blocks.0.{s}", 2 * D, 3 * D)
            _zero_rows(t, f"transformer_blocks.0.{s}", 5 * D, 6 * D)
    W = _edit(tinyW, zero_gates)
    h_img, h_txt, temb = _block_inputs(TINY)
    ang = o.rope_angles(o.position_ids(2, 3, 3), TINY.rope_axes, TINY.rope_theta)
    hi, ht = o.block(W, 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps)
    assert np.array_equal(hi, h_img) and np.array_equal(ht, h_txt)


def test_block_gate_linearity(tinyW):
    """With the MLP gate closed the update is linear in the attention gate."""
    D = TINY.hidden

    def setup(scale):
        def fn(t):
            for s in ("img_mod", "txt_mod"):
                _zero_rows(t, f"transformer_blocks.0.{s}", 5 * D, 6 * D)
                w = o.upcast(t[f"transformer_blocks.0.{s}.weight"], np.float32)
                b = o.upcast(t[f"transformer_blocks.0.{s}.bias"], np.float32)
                w[2 * D:3 * D] *= scale; b[2 * D:3 * D] *= scale   # exact in bf16 (power of 2)
                t[f"transformer_blocks.0.{s}.weight"] = f32_to_bf16_bits(w)
                t[f"transformer_blocks.0.{s}.bias"] = f32_to_bf16_bits(b)
        return _edit(tinyW, fn)
    h_img, h_txt, temb = _block_inputs(TINY)
    ang = o.rope_angles(o.position_ids(2, 3, 3), TINY.rope_axes, TINY.rope_theta)
    a1 = o.block(setup(1.0), 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps)
    a2 = o.block(setup(2.0), 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps)
    assert np.allclose(a2[0] - h_img, 2 * (a1[0] - h_img), atol=1e-12)
    assert np.allclose(a2[1] - h_txt, 2 * (a1[1] - h_txt), atol=1e-12)
    assert np.abs(a1[0] - h_img).max() > 1e-3


def test_block_stream_symmetry(tinyW):
    """With identical weights in both streams the joint block treats [text; image]
    symmetrically: swapping the streams (and their positions) swaps the outputs."""
    def tie(t):
        p = "transformer_blocks.0."
        for a, b in (("img_mod", "txt_mod"), ("attn.img_qkv", "attn.txt_qkv"), ("attn.to_out", "attn.to_add_out"),
                     ("img_mlp.w1", "txt_mlp.w1"), ("img_mlp.w2", "txt_mlp.w2"), ("img_mlp.w3", "txt_mlp.w3")):
            t[p + b + ".weight"] = t[p + a + ".weight"]; t[p + b + ".bias"] = t[p + a + ".bias"]
        t[p + "attn.norm_added_q.weight"] = t[p + "attn.norm_q.weight"]
        t[p + "attn.norm_added_k.weight"] = t[p + "attn.norm_k.weight"]
    W = _edit(tinyW, tie)
    h_img, h_txt, temb = _block_inputs(TINY, Ni=4, Nt=4)
    rng = np.random.default_rng(7)
    ang = rng.uniform(-3, 3, size=(8, TINY.head_dim // 2))
    hi, ht = o.block(W, 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps)
    ang_sw = np.concatenate([ang[4:], ang[:4]])
    hi2, ht2 = o.block(W, 0, h_txt, h_img, temb, ang_sw, TINY.heads, TINY.eps)
    assert np.allclose(hi2, ht, atol=1e-10) and np.allclose(ht2, hi, atol=1e-10)


def test_block_token_permutation_equivariance(tinyW):
    h_img, h_txt, temb = _block_inputs(TINY, Ni=6, Nt=3)
    ang = o.rope_angles(o.position_ids(2, 3, 3), TINY.rope_axes, TINY.rope_theta)
    hi, ht = o.block(tinyW, 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps)
    perm = np.array([4, 0, 5, 2, 1, 3])
    ang_p = np.concatenate([ang[:3], ang[3:][perm]])
    hi_p, ht_p = o.block(tinyW, 0, h_img[:, perm], h_txt, temb, ang_p, TINY.heads, TINY.eps)
    assert np.allclose(hi_p, hi[:, perm], atol=1e-10) and np.allclose(ht_p, ht, atol=1e-10)


def test_block_single_token_attention_is_value(tinyW):
    """One token in total: softmax weight 1, so the attention output is that token's v
    (after nothing: RoPE never touches v)."""
    D, H = TINY.hidden, TINY.heads
    rng = np.random.default_rng(8)
    h_txt = rng.standard_normal((1, 1, D))
    h_img = np.zeros((1, 0, D))
    temb = rng.standard_normal((1, D))
    ang = rng.uniform(-3, 3, size=(1, TINY.head_dim // 2))

    def no_mlp(t):
        _zero_rows(t, "transformer_blocks.0.txt_mod", 5 * D, 6 * D)
    W = _edit(tinyW, no_mlp)
    _, ht = o.block(W, 0, h_img, h_txt, temb, ang, H, TINY.eps)
    m = o.linear(W, "transformer_blocks.0.txt_mod", o.silu(temb))
    sh, sc, g = m[:, :D], m[:, D:2 * D], m[:, 2 * D:3 * D]
    a = (1 + sc) * h_txt[0] / np.sqrt(np.mean(h_txt[0] ** 2) + TINY.eps) + sh
    v = o.linear(W, "transformer_blocks.0.attn.txt_qkv", a)[:, 2 * D:]
    ref = h_txt[0] + g * o.linear(W, "transformer_blocks.0.attn.to_add_out", v)
    assert np.allclose(ht[0], ref, atol=1e-10)


def test_block_row_selection_matches_full(tinyW):
    h_img, h_txt, temb = _block_inputs(TINY, Ni=6, Nt=3)
    ang = o.rope_angles(o.position_ids(2, 3, 3), TINY.rope_axes, TINY.rope_theta)
    hi, ht = o.block(tinyW, 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps)
    hs, ts = o.block(tinyW, 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps,
                     img_rows=np.array([5, 1]), txt_rows=np.array([2]))
    assert np.allclose(hs, hi[:, [5, 1]], atol=1e-12) and np.allclose(ts, ht[:, [2]], atol=1e-12)


def test_forward_runs_tiny(tinyW):
    rng = np.random.default_rng(9)
    X = rng.standard_normal((2, 6, TINY.in_channels))
    E = f32_to_bf16_bits(rng.standard_normal((2, 3, 4, TINY.txt_dim)).astype(np.float32))
    v = o.forward(tinyW, TINY, X, 2, 3, E, [0.3, 0.9])
    assert v.shape == (2, 6, TINY.in_channels) and np.all(np.isfinite(v))
    # batch elements are independent
    v1 = o.forward(tinyW, TINY, X[1:], 2, 3, E[1:], [0.9])
    assert np.allclose(v1[0], v[1], atol=1e-12)


# ------------------------------------------------------------------ sampler
def test_euler_lands_on_data_for_straight_paths():
    """x_t = (1-t) x0 + t x1 with v = x1 - x0: Euler is exact on straight lines."""
    rng = np.random.default_rng(10)
    x0, x1 = rng.standard_normal((2, 3, 8))
    vel = lambda x, t, c: x1 - x0
    for S in (1, 2, 4, 7, 20):
        assert np.allclose(o.sample_euler(vel, x1, S, 1.0), x0, atol=1e-12)
    # one step from t = 1 lands exactly on x0
    assert np.allclose(o.euler(x1, x1 - x0, 1.0), x0, atol=1e-15)
    # the exact velocity of the straight path at (x_t, t) is (x_t - x0) / t
    vel2 = lambda x, t, c: (x - x0) / t
    assert np.allclose(o.sample_euler(vel2, x1, 5, 1.0), x0, atol=1e-12)
    assert o.timesteps(4).tolist() == [1.0, 0.75, 0.5, 0.25]


def test_cfg_special_scales():
    rng = np.random.default_rng(11)
    c, u = rng.standard_normal((2, 10))
    assert np.allclose(o.cfg_combine(c, u, 1.0), c, atol=1e-15)
    assert np.array_equal(o.cfg_combine(c, u, 0.0), u)
    assert np.allclose(o.cfg_combine(c, u, 5.0), u + 5 * (c - u))
    calls = []
    vel = lambda x, t, cond: (calls.append(cond), np.full_like(x, 1.0 if cond else 3.0))[1]
    x = o.sample_euler(vel, np.zeros(4), 2, 5.0)          # v = 3 + 5 (1 - 3) = -7 each step
    assert np.allclose(x, 7.0) and calls.count(False) == 2
    calls.clear()
    o.sample_euler(vel, np.zeros(4), 2, 1.0)
    assert calls.count(False) == 0                        # guidance 1: no unconditional pass


# ------------------------------------------------------------------ sampler variants
def test_time_shift_fixed_points_values_and_group():
    t = np.linspace(0.0, 1.0, 11)
    assert np.array_equal(o.time_shift(t, 0.0), t)                 # mu = 0: identity
    for mu in (-1.3, 0.4, 1.06, 2.5):
        assert o.time_shift(0.0, mu) == 0.0 and o.time_shift(1.0, mu) == 1.0
        assert np.all(np.diff(o.time_shift(t, mu)) > 0)          # order of the grid kept
    # shift factor 3 (mu = ln 3), worked by hand: 1/2 -> 3/4, 1/4 -> 1/2, 1/10 -> 1/4
    assert abs(o.time_shift(0.5, math.log(3.0)) - 0.75) < 1e-15
    assert abs(o.time_shift(0.25, math.log(3.0)) - 0.5) < 1e-15
    assert abs(o.time_shift(0.1, math.log(3.0)) - 0.25) < 1e-15
    # shifts compose by adding mu (e^mu is the factor, not mu), and -mu undoes mu
    assert np.allclose(o.time_shift(o.time_shift(t, 0.7), -0.25), o.time_shift(t, 0.45), atol=1e-14)
    assert np.allclose(o.time_shift(o.time_shift(t, 1.06), -1.06), t, atol=1e-14)
    # mu > 0 moves every inner time towards the noise end t = 1
    assert np.all(o.time_shift(t[1:-1], 1.06) > t[1:-1])


def test_shift_mu_is_linear_through_both_anchors():
    # the pages' one anchor: 512^2 -> 32 x 32 = 1024 tokens at mu = 1.06
    assert o.shift_mu(1024, 1024, 1.06, 4096, 1.5) == pytest.approx(1.06, abs=1e-15)
    assert o.shift_mu(4096, 1024, 1.06, 4096, 1.5) == pytest.approx(1.5, abs=1e-15)
    assert o.shift_mu(2560, 1024, 1.06, 4096, 1.5) == pytest.approx(1.28, abs=1e-15)   # midpoint
    assert o.shift_mu(8100, 1024, 1.06, 4096, 1.06) == pytest.approx(1.06, abs=1e-15)  # flat line


def test_time_grid_uniform_and_shifted():
    assert o.time_grid(4).tolist() == [1.0, 0.75, 0.5, 0.25, 0.0]
    g = o.time_grid(7, 1.06)
    assert g[0] == 1.0 and g[-1] == 0.0 and len(g) == 8
    dt = -np.diff(g)
    assert np.all(dt > 0) and abs(dt.sum() - 1.0) < 1e-15         # steps telescope to 1
    assert dt[0] < 1.0 / 7 < dt[-1]                               # small steps near noise


def test_sampler_on_shifted_grid_worked_by_hand():
    # v(x, t) = x: Euler multiplies by (1 - dt_k).  S = 2, mu = ln 3: t = 1, 3/4, 0,
    # dt = 1/4, 3/4, so x -> x (3/4)(1/4) and the model sees t = 1 then t = 3/4
    seen = []
    vel = lambda x, t, c: (seen.append(t), x)[1]
    x = o.sample_euler(vel, np.full(3, 2.0), 2, 1.0, mu=math.log(3.0))
    assert np.allclose(x, 2.0 * 0.75 * 0.25, atol=1e-15)
    assert seen == pytest.approx([1.0, 0.75], abs=1e-15)
    # straight paths stay exact on any grid whose steps sum to 1
    rng = np.random.default_rng(12)
    x0, x1 = rng.standard_normal((2, 3, 8))
    assert np.allclose(o.sample_euler(lambda x, t, c: x1 - x0, x1, 5, 1.0, mu=1.3), x0, atol=1e-12)


def test_cfg_rescaled_values_and_invariants():
    # by hand: c = (3, 4), u = 0, s = 2 -> plain (6, 8), |c| = 5, |plain| = 10
    c = np.array([[3.0, 4.0]])
    u = np.zeros((1, 2))
    assert np.allclose(o.cfg_rescaled(c, u, 2.0, 1.0), [[3.0, 4.0]], atol=1e-15)
    assert np.allclose(o.cfg_rescaled(c, u, 2.0, 0.5), [[4.5, 6.0]], atol=1e-15)
    rng = np.random.default_rng(13)
    c, u = rng.standard_normal((2, 3, 4, 5))
    assert np.array_equal(o.cfg_rescaled(c, u, 5.0, 0.0), o.cfg_combine(c, u, 5.0))   # phi = 0: plain
    assert np.allclose(o.cfg_rescaled(c, u, 1.0, 1.0), c, atol=1e-14)                 # s = 1: cond
    v, p = o.cfg_rescaled(c, u, 5.0, 1.0), o.cfg_combine(c, u, 5.0)
    for b in range(3):                                  # per sample: |v| = |c|, same direction
        assert np.linalg.norm(v[b]) == pytest.approx(np.linalg.norm(c[b]), rel=1e-13)
        cosv = np.sum(v[b] * p[b]) / (np.linalg.norm(v[b]) * np.linalg.norm(p[b]))
        assert cosv == pytest.approx(1.0, abs=1e-13)
    c2 = c.copy()
    c2[1] *= 7.0
    assert np.array_equal(o.cfg_rescaled(c2, u, 5.0, 1.0)[0], v[0])   # samples are independent
    z = np.zeros((2, 6))
    assert np.array_equal(o.cfg_rescaled(z, z, 5.0, 1.0), z)          # zero velocity stays zero
    # inside the sampler: c = 1, u = 3 (4 elements): plain -7, rescaled to norm 2 -> -1
    vel = lambda x, t, cond: np.full_like(x, 1.0 if cond else 3.0)
    assert np.allclose(o.sample_euler(vel, np.zeros(4), 2, 5.0, phi=1.0), 1.0, atol=1e-15)


# ------------------------------------------------------------------ int4 weight-only
def test_w4_model_size_matches_the_page():
    g = {k: v for k, v in _golden("lens_int4_model.txt")}
    assert int(g["bits"]) == 4 and int(g["group_size"]) == o.W4_GROUP
    specs = [(n, s) for n, s, _ in weight_specs(LENS)]
    gb = o.w4_model_bytes(specs) / 1e9
    assert abs(gb - float(g["model_GB"])) < 0.01, gb          # 2.349 GB
    # the sensitive layers stay bf16, every 2-D block weight is quantized
    for name, shape in specs:
        q = o.w4_quantizable(name, len(shape))
        assert q == (len(shape) == 2 and name.startswith("transformer_blocks.")), name


def test_w4_hand_worked_groups():
    # codes 0..15 spread over a group: min 0, max 15 -> s = 1, b = 0, q = w, exact
    w = np.tile(np.arange(16, dtype=np.float32), 8).reshape(2, 64)
    q, sc, bi = o.quantize_w4(w)
    assert np.array_equal(q, w.astype(np.uint8)) and np.all(sc == 1.0) and np.all(bi == 0.0)
    assert np.array_equal(o.dequantize_w4(q, sc, bi), w)
    # a shifted, scaled copy: w = 0.5 + 0.25 k -> s = 0.25, b = 0.5, same codes
    q2, sc2, bi2 = o.quantize_w4(0.5 + 0.25 * w)
    assert np.array_equal(q2, q) and np.all(sc2 == 0.25) and np.all(bi2 == 0.5)
    # a constant group: s = 0, every code 0, the value comes back as its bf16 bias
    c = np.full((1, 64), 0.375, np.float32)
    q3, sc3, bi3 = o.quantize_w4(c)
    assert np.all(q3 == 0) and sc3[0, 0] == 0.0 and np.array_equal(o.dequantize_w4(q3, sc3, bi3), c)
    # rint ties go to even: 1.5 -> 2, 2.5 -> 2 (group min 0, max 15)
    t = np.zeros((1, 64), np.float32)
    t[0, 1], t[0, 2], t[0, 3] = 15.0, 1.5, 2.5
    assert o.quantize_w4(t)[0][0, 2] == 2 and o.quantize_w4(t)[0][0, 3] == 2


def test_w4_error_bound_and_order_on_random_weights():
    rng = np.random.default_rng(14)
    w = (rng.standard_normal((96, 1536)) * 0.02).astype(np.float32)
    q, sc, bi = o.quantize_w4(w)
    assert q.dtype == np.uint8 and q.max() <= 15 and sc.shape == (96, 24)
    err = np.abs(o.dequantize_w4(q, sc, bi) - w).reshape(96, 24, 64)
    g = w.reshape(96, 24, 64)
    # half a step, plus what rounding the bias to bf16 moved the grid
    bound = 0.5 * sc + np.abs(g.min(-1) - bi) + 1e-9
    assert np.all(err.max(-1) <= bound[...] + 0.5 * sc * 2.0 ** -7)
    # codes keep the order of the values inside a group
    order = np.argsort(g, axis=-1, kind="stable")
    qs = np.take_along_axis(q.reshape(96, 24, 64), order, -1)
    assert np.all(np.diff(qs.astype(int), axis=-1) >= 0)
    # the extremes of a group land on codes 0 and 15 (or one step inside)
    assert np.all(np.take_along_axis(q.reshape(96, 24, 64), order[..., :1], -1) <= 1)
    assert np.all(np.take_along_axis(q.reshape(96, 24, 64), order[..., -1:], -1) >= 14)


def test_w4_model_replaces_only_quantizable_weights():
    import dataclasses
    w = make_weights(dataclasses.replace(TINY, mlp_hidden=128), seed=3)      # every K a multiple of 64
    qm = o.quantize_model_w4(w)
    for name, t in w.items():
        if o.w4_quantizable(name, t.ndim):
            assert qm[name].dtype == np.float64 and not np.array_equal(qm[name], o.upcast(t))
        else:
            assert qm[name] is t


# ------------------------------------------------------------------ noise
def test_splitmix64_published_vectors():
    want = [int(r[0], 16) for r in _golden("splitmix64_seed0.txt")]
    gamma = 0x9E3779B97F4A7C15
    states = np.array([0, gamma, (2 * gamma) % 2 ** 64], np.uint64)
    assert [int(x) for x in o.splitmix64(states)] == want


def test_noise_is_standard_normal():
    from scipy import stats
    z = o.noise(42, 200_000).astype(np.float64)
    assert np.all(np.isfinite(z))
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1) < 0.01
    assert stats.kstest(z, "norm").pvalue > 1e-3
    # different seeds give different streams; same seed reproduces
    assert np.array_equal(o.noise(42, 1000), z[:1000].astype(np.float32))
    assert not np.array_equal(o.noise(43, 1000), o.noise(42, 1000))


def test_box_muller_closed_form():
    """u2 = 0 gives z = sqrt(-2 ln u1): check one element by hand from its words."""
    seed = 7
    n = np.arange(64, dtype=np.uint64)
    w1 = o.splitmix64(np.uint64(seed) ^ o.splitmix64(np.uint64(2) * n))
    w2 = o.splitmix64(np.uint64(seed) ^ o.splitmix64(np.uint64(2) * n + np.uint64(1)))
    z = o.noise(seed, 64)
    for i in (0, 17, 63):
        u1 = ((int(w1[i]) >> 11) + 1) / 2.0 ** 53
        u2 = (int(w2[i]) >> 11) / 2.0 ** 53
        assert 0.0 < u1 <= 1.0 and 0.0 <= u2 < 1.0
        assert z[i] == np.float32(math.sqrt(-2 * math.log(u1)) * math.cos(2 * math.pi * u2))


# ------------------------------------------------------------------ text padding mask
def test_masked_attention_brute_force_and_no_influence():
    rng = np.random.default_rng(12)
    q, k, v = (rng.standard_normal((2, 2, 6, 4)) for _ in range(3))
    mask = o.text_key_mask(2, 3, 3, [1, 3])        # sample 0 keeps 1 of 3 text keys
    out = o.attention(q, k, v, mask)
    for b in range(2):
        keep = np.where(mask[b])[0]
        for h in range(2):
            assert np.allclose(out[b, h], _attn_loops(q[b, h], k[b, h][keep], v[b, h][keep]), atol=1e-12)
    k2, v2 = k.copy(), v.copy()
    k2[0, :, 1:3] = 1e3 * rng.standard_normal((2, 2, 4))   # change only masked keys / values
    v2[0, :, 1:3] = -7.0
    assert np.allclose(o.attention(q, k2, v2, mask), out, atol=1e-12)
    assert np.allclose(o.attention(q, k, v, o.text_key_mask(2, 3, 3, [3, 3])), o.attention(q, k, v), atol=1e-12)
    assert o.text_key_mask(2, 3, 3, None) is None


def test_block_padding_has_no_influence(tinyW):
    h_img, h_txt, temb = _block_inputs(TINY, Ni=6, Nt=4)
    ang = o.rope_angles(o.position_ids(2, 3, 4), TINY.rope_axes, TINY.rope_theta)
    hi, ht = o.block(tinyW, 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps, txt_len=[2, 4])
    h_txt2 = h_txt.copy()
    h_txt2[0, 2:] = 50.0 * np.random.default_rng(13).standard_normal((2, TINY.hidden))
    hi2, ht2 = o.block(tinyW, 0, h_img, h_txt2, temb, ang, TINY.heads, TINY.eps, txt_len=[2, 4])
    assert np.allclose(hi2, hi, atol=1e-10) and np.allclose(ht2[:, :2], ht[:, :2], atol=1e-10)
    assert np.allclose(ht2[1], ht[1], atol=1e-10)
    # the unpadded sample equals the unmasked block
    hu, tu = o.block(tinyW, 0, h_img, h_txt, temb, ang, TINY.heads, TINY.eps)
    assert np.allclose(hi[1], hu[1], atol=1e-12) and not np.allclose(hi[0], hu[0], atol=1e-6)


# ------------------------------------------------------------------ closed-form pins of the remaining pieces
def _silu(x):
    return x / (1.0 + math.exp(-x))          # the sigmoid-weighted linear unit, by its definition


def test_gated_mlp_unit_vector_closed_form():
    """[blog] "Overview" (gate / up / down of 1536x4096) with the READING w1 = gated branch:
    unit rows in w1 and w3 pick x_i and x_j, a unit column of w2 routes their product to
    one output, so that output is silu(x_i) * x_j exactly.  A sum in place of the product,
    SiLU on the product, or SiLU on the w3 branch all give other numbers here."""
    D, F = 5, 3
    w1, w3, w2 = np.zeros((F, D)), np.zeros((F, D)), np.zeros((D, F))
    w1[0, 1], w3[0, 2], w2[4, 0] = 1.0, 1.0, 1.0        # out_4 = silu(x_1) * x_2
    w1[1, 2], w3[1, 1], w2[0, 1] = 1.0, 1.0, 1.0        # out_0 = silu(x_2) * x_1 (branches swapped)
    w1[2, 3], w3[2, 3], w2[2, 2] = 1.0, 1.0, 2.0        # out_2 = 2 silu(x_3) * x_3
    W = o.Weights({"m.w1.weight": w1, "m.w3.weight": w3, "m.w2.weight": w2,
                   "m.w2.bias": np.array([0.0, 0.0, 0.0, 0.5, 0.0])})
    x = np.array([[0.3, 1.0, -2.0, 0.5, 7.0]])
    y = o.gated_mlp(W, "m", x)[0]
    expect = [_silu(-2.0) * 1.0, 0.0, 2.0 * _silu(0.5) * 0.5, 0.5, _silu(1.0) * -2.0]
    assert np.allclose(y, expect, rtol=0, atol=1e-15)
    assert abs(expect[4] - (-1.4621171572600098)) < 1e-15  # silu(1) = 0.7310585786300049


def test_final_layer_closed_form():
    """[mlx] "Patchify 补丁化与输出投影": norm_out.linear then proj_out.  With zero
    norm_out weights its bias alone sets (scale, shift) (READING: scale first), and
    identity rows in proj_out expose (1 + scale) * x / rms(x) + shift column by column.
    The row [3, -4, 0, 0] has rms 2.5 (eps = 0), so x / rms(x) = [1.2, -1.6, 0, 0]."""
    D, C = 4, 3
    proj = np.zeros((C, D))
    proj[0, 0] = proj[1, 1] = proj[2, 2] = 1.0
    bias = np.array([1.0, 0.5, -1.0, 2.0, 0.25, -0.5, 3.0, 1.0])   # scale | shift
    W = o.Weights({"norm_out.linear.weight": np.zeros((2 * D, D)), "norm_out.linear.bias": bias,
                   "proj_out.weight": proj, "proj_out.bias": np.array([0.0, 0.0, 10.0])})
    h = np.array([[[3.0, -4.0, 0.0, 0.0], [0.0, 0.0, 5.0, 0.0]]])
    temb = np.array([[0.7, -1.0, 2.0, 0.0]])
    v = o.final_layer(W, h, temb, 0.0)[0]
    # row 0: [(1+1) 1.2 + 0.25, (1+0.5)(-1.6) - 0.5, 0 + 3 + 10]; row 1 has x/rms = [0, 0, 2, 0]
    assert np.allclose(v[0], [2.65, -2.9, 13.0], rtol=0, atol=1e-14)
    assert np.allclose(v[1], [0.25, -0.5, 0.0 * 2.0 + 3.0 + 10.0], rtol=0, atol=1e-14)
    # scale = shift = 0 is the plain RMSNorm
    W0 = o.Weights({"norm_out.linear.weight": np.zeros((2 * D, D)), "proj_out.weight": proj})
    assert np.allclose(o.final_layer(W0, h, temb, 0.0)[0, 0], [1.2, -1.6, 0.0], rtol=0, atol=1e-15)
    # the projection sees SiLU(temb): one unit weight makes scale_0 = 1 + silu(2)
    wn = np.zeros((2 * D, D))
    wn[0, 2] = 1.0
    W1 = o.Weights({"norm_out.linear.weight": wn, "norm_out.linear.bias": bias, "proj_out.weight": proj})
    assert abs(o.final_layer(W1, h, temb, 0.0)[0, 0, 0] - ((2.0 + _silu(2.0)) * 1.2 + 0.25)) < 1e-14


def test_modulation_closed_form():
    """AdaLN projection of a block stream ([blog] "Overview": shift, scale and gate for
    the attention and for the MLP; [mlx] "自适应调制": img_mod / txt_mod): Linear of
    SiLU(temb), split into six hidden-size chunks in the order (shift1, scale1, gate1,
    shift2, scale2, gate2).  Zero weights return the bias chunks in that order; one unit
    weight adds SiLU(temb_k) at one output column, not temb_k and not SiLU of the sum."""
    D = 3
    bias = np.arange(6 * D, dtype=np.float64) * 0.5 - 2.0
    temb = np.array([[0.4, -1.5, 2.5]])
    Wz = o.Weights({"blk.mod.weight": np.zeros((6 * D, D)), "blk.mod.bias": bias})
    parts = o.modulation(Wz, "blk.mod", temb, 6)
    assert len(parts) == 6
    for i, p in enumerate(parts):
        assert p.shape == (1, D) and np.array_equal(p[0], bias[i * D:(i + 1) * D])
    w = np.zeros((6 * D, D))
    w[2 * D + 1, 2] = 1.0                     # gate1, column 1 reads temb_2
    W1 = o.Weights({"blk.mod.weight": w, "blk.mod.bias": bias})
    g1 = o.modulation(W1, "blk.mod", temb, 6)[2][0]
    assert abs(g1[1] - (bias[2 * D + 1] + _silu(2.5))) < 1e-14
    assert np.array_equal(g1[[0, 2]], bias[[2 * D, 2 * D + 2]])


def test_timestep_embedding_mlp_closed_form():
    """temb = linear_2(SiLU(linear_1(e))) ([mlx] time_text_embed.timestep_embedder).  At
    t = 0 the features are [1 ... 1, 0 ... 0] (cos 0, sin 0), so unit rows in linear_1
    (with biases) give known pre-activations and linear_2 routes their SiLUs."""
    fd, D = 16, 4
    l1, b1 = np.zeros((D, fd)), np.array([0.0, -3.0, -0.5, 0.0])
    l1[0, 0] = 1.0                 # cos part: 1          -> silu(1)
    l1[1, 8] = 1.0                 # sin part: 0, bias -3 -> silu(-3)
    l1[2, 0] = l1[2, 1] = 1.0      # 2 - 0.5             -> silu(1.5)
    l2, b2 = np.zeros((D, D)), np.array([0.0, 0.0, 0.0, 1.0])
    l2[0, 2] = l2[1, 0] = l2[2, 1] = 1.0
    l2[3, 0] = 2.0
    p = "time_text_embed.timestep_embedder"
    W = o.Weights({p + ".linear_1.weight": l1, p + ".linear_1.bias": b1,
                   p + ".linear_2.weight": l2, p + ".linear_2.bias": b2})
    temb = o.timestep_embedding(W, np.array([0.0]), fd)[0]
    s1, sm3, s15 = 0.7310585786300049, -3.0 / (1.0 + math.exp(3.0)), 1.5 / (1.0 + math.exp(-1.5))
    assert np.allclose(temb, [s15, s1, sm3, 2.0 * s1 + 1.0], rtol=0, atol=1e-15)


def _zero_model_with_output_bias(d, b):
    w = {}
    for name, shape, _ in weight_specs(d):
        w[name] = np.zeros(shape)
    w["proj_out.bias"] = np.asarray(b, np.float64)
    return o.Weights(w)


@pytest.mark.parametrize("steps,mu,guidance", [(1, None, 1.0), (4, None, 1.0), (7, None, 5.0),
                                               (4, 0.7, 1.0), (7, -0.4, 3.0)])
def test_sample_constant_field_lands_exactly(steps, mu, guidance):
    """A model whose only nonzero weight is the proj_out bias b has v = b for every token,
    t and text, so the sampler returns noise(seed) - unpatchify(b) for any step count and
    any grid ([paper] "Flow Matching 训练目标": the grid runs from t = 1 to t = 0, so the
    steps add up to 1).  The expected latent is written out from the patch layout
    (channel c, patch row r, patch column s at feature 4c + 2r + s)."""
    d = TINY
    rng = np.random.default_rng(5)
    b = rng.standard_normal(d.in_channels)
    W = _zero_model_with_output_bias(d, b)
    gh, gw, B, seed = 2, 3, 2, 123
    E = rng.standard_normal((B, 3, d.txt_layers, d.txt_dim))
    x = o.sample(W, d, E, None, B, gh, gw, steps, guidance, seed, mu=mu)
    C = d.latent_channels
    z = o.noise(seed, B * C * 2 * gh * 2 * gw).astype(np.float64).reshape(B, C, 2 * gh, 2 * gw)
    shift = np.empty((C, 2 * gh, 2 * gw))
    for c in range(C):
        for yy in range(2 * gh):
            for xx in range(2 * gw):
                shift[c, yy, xx] = b[4 * c + 2 * (yy % 2) + (xx % 2)]
    assert np.allclose(x, z - shift[None], rtol=0, atol=1e-12)


def test_sample_wiring_with_guidance(tinyW):
    """Two CFG steps on the tiny random model, written out from the pinned parts:
    x1 = z - (1/2) g(z, 1), x2 = x1 - (1/2) g(x1, 1/2) with g = u + s (c - u), where c and
    u are the forward on the patchified latent with the conditional and unconditional
    text.  A swapped cond/uncond, a wrong t or a wrong dt all fail here."""
    d = TINY
    rng = np.random.default_rng(9)
    gh, gw, B, seed, s = 2, 2, 1, 77, 3.0
    Ec = rng.standard_normal((B, 3, d.txt_layers, d.txt_dim))
    Eu = rng.standard_normal((B, 3, d.txt_layers, d.txt_dim))
    C = d.latent_channels

    def f(x, t, E):
        return o.unpatchify(o.forward(tinyW, d, o.patchify(x), gh, gw, E, [t] * B), gh, gw, C)

    def g(x, t):
        c, u = f(x, t, Ec), f(x, t, Eu)
        assert np.linalg.norm(c - u) > 1e-3 * np.linalg.norm(c)   # text reaches the image
        return u + s * (c - u)

    z = o.noise(seed, B * C * 4 * gh * gw).astype(np.float64).reshape(B, C, 2 * gh, 2 * gw)
    x1 = z - 0.5 * g(z, 1.0)
    x2 = x1 - 0.5 * g(x1, 0.5)
    trace = []
    got = o.sample(tinyW, d, Ec, Eu, B, gh, gw, 2, s, seed, trace=trace)
    assert np.allclose(got, x2, rtol=0, atol=1e-12)
    assert [(t, c) for t, c, _, _ in trace] == [(1.0, True), (1.0, False), (0.5, True), (0.5, False)]
    # stop_after = 1 is the state after the first step of the same two-step grid
    assert np.allclose(o.sample(tinyW, d, Ec, Eu, B, gh, gw, 2, s, seed, stop_after=1), x1, rtol=0, atol=1e-12)


def test_sample_wiring_with_padding_masks(tinyW):
    """One CFG step with different valid text lengths for the two halves ([blog]
    "Exploring Text Encoder": padded text tokens are masked): the conditional half
    must use len_cond and the unconditional half len_uncond."""
    d = TINY
    rng = np.random.default_rng(10)
    gh, gw, B, seed, s = 2, 2, 1, 78, 4.0
    Ec = rng.standard_normal((B, 3, d.txt_layers, d.txt_dim))
    Eu = rng.standard_normal((B, 3, d.txt_layers, d.txt_dim))
    C = d.latent_channels
    z = o.noise(seed, B * C * 4 * gh * gw).astype(np.float64).reshape(B, C, 2 * gh, 2 * gw)

    def f(E, n):
        return o.unpatchify(o.forward(tinyW, d, o.patchify(z), gh, gw, E, [1.0] * B, txt_len=n), gh, gw, C)

    c, u = f(Ec, [1]), f(Eu, [3])
    assert np.linalg.norm(f(Ec, [3]) - c) > 1e-3 * np.linalg.norm(c)   # the mask matters here
    got = o.sample(tinyW, d, Ec, Eu, B, gh, gw, 1, s, seed, len_cond=[1], len_uncond=[3])
    assert np.allclose(got, z - (u + s * (c - u)), rtol=0, atol=1e-12)
