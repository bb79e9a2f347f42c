"""GPU parity of the single-operation entry points against the CPU oracle.
Indexing work is compared bit-exactly; floating point within stated bounds."""
import math

import numpy as np
import pytest

from lens_inputs import LENS, f32_to_bf16_bits
from oracle import lens_oracle as o
from tests.helpers import bf16_to_f64, cos_sim, dev, host, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import flow_matching_mmdit_b200 as L
    L.load_library()
    return torch


import flow_matching_mmdit_b200 as L  # noqa: E402


def _sync():
    import torch
    torch.cuda.synchronize()


# ------------------------------------------------------------------ indexing: bit-exact
@pytest.mark.parametrize("B,gh,gw", [(1, 8, 8), (2, 3, 5), (1, 64, 128), (2, 90, 90)])
def test_patchify_unpatchify_bit_exact(B, gh, gw):
    import torch
    rng = np.random.default_rng(gh * 1000 + gw)
    Z = rng.standard_normal((B, 32, 2 * gh, 2 * gw)).astype(np.float32)
    tok = torch.empty((B, gh * gw, 128), dtype=torch.float32, device="cuda")
    L.lens_op_patchify(dev(Z), B, gh, gw, tok)
    back = torch.empty((B, 32, 2 * gh, 2 * gw), dtype=torch.float32, device="cuda")
    L.lens_op_unpatchify(tok, B, gh, gw, back)
    _sync()
    assert np.array_equal(host(tok), o.patchify(Z))
    assert np.array_equal(host(back), Z)


@pytest.mark.parametrize("seed,B,gh,gw", [(0, 1, 8, 8), (42, 2, 64, 64), (5, 1, 90, 90), (2 ** 63 + 7, 1, 3, 7)])
def test_noise_tokens_match_oracle(seed, B, gh, gw):
    import torch
    tok = torch.empty((B, gh * gw, 128), dtype=torch.float32, device="cuda")
    L.lens_op_noise_tokens(seed, B, gh, gw, tok)
    _sync()
    ref = o.patchify(o.noise(seed, B * 32 * 4 * gh * gw).reshape(B, 32, 2 * gh, 2 * gw))
    got = host(tok)
    # both sides evaluate Box-Muller in double and round once to float
    assert np.allclose(got, ref, rtol=1e-6, atol=1e-6)
    assert np.mean(got == ref) > 0.999


@pytest.mark.parametrize("gh,gw,nt", [(8, 8, 16), (64, 128, 256), (90, 90, 0), (2, 3, 1)])
def test_rope_table(gh, gw, nt):
    import torch
    n = nt + gh * gw
    tab = torch.empty((n, 32, 2), dtype=torch.float32, device="cuda")
    L.lens_op_rope_table(gh, gw, nt, tab)
    _sync()
    ang = o.rope_angles(o.position_ids(gh, gw, nt), LENS.rope_axes, LENS.rope_theta)
    got = host(tab)
    assert np.allclose(got[..., 0], np.cos(ang), atol=2e-7, rtol=0)
    assert np.allclose(got[..., 1], np.sin(ang), atol=2e-7, rtol=0)
    if nt:
        assert np.array_equal(got[:nt, :, 0], np.ones((nt, 32), np.float32))
        assert np.array_equal(got[:nt, :, 1], np.zeros((nt, 32), np.float32))


# ------------------------------------------------------------------ floating point
def test_rmsnorm_modulate():
    import torch
    rng = np.random.default_rng(3)
    B, rows = 2, 333
    x = (rng.standard_normal((B * rows, 1536)) * 3).astype(np.float32)
    mod = (rng.standard_normal((B, 2, 1536)) * 0.3).astype(np.float32)
    y = torch.empty((B * rows, 1536), dtype=torch.int16, device="cuda")
    md = dev(mod)
    L.lens_op_rmsnorm_modulate(dev(x), B * rows, rows, md[:, 0], md[:, 1], 2 * 1536, 1e-6, y)
    _sync()
    xs = x.astype(np.float64).reshape(B, rows, 1536)
    ref = (1 + mod[:, None, 1].astype(np.float64)) * o.rms_norm(xs, 1e-6) + mod[:, None, 0]
    got = bf16_to_f64(host(y)).reshape(B, rows, 1536)
    # one bf16 rounding of the output: |err| <= 2^-8 |y| (plus fp32 slack)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 1536, 1536), (1000, 128, 1536), (77, 4608, 1536),
                                   (4352, 1536, 4096), (257, 96, 11520), (5, 32, 192)])
def test_gemm_bf16_tcgen05(M, N, K):
    import torch
    rng = np.random.default_rng(M + N + K)
    A = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    Bw = f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.05).astype(np.float32))
    bias = rng.standard_normal(N).astype(np.float32)
    C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    L.lens_op_gemm_bf16(dev(A), dev(Bw), dev(bias), C, M, N, K)
    _sync()
    ref = bf16_to_f64(A) @ bf16_to_f64(Bw).T + bias
    got = host(C)
    assert np.all(np.isfinite(got))
    # exact bf16 products, fp32 accumulation: error ~ sqrt(K) * 2^-24 * |terms|
    scale = np.sqrt(K) * 0.05
    assert np.max(np.abs(got - ref)) <= 1e-5 * scale * max(1.0, math.sqrt(K / 64)), np.max(np.abs(got - ref))
    # fp32 accumulation over K terms: relative error grows like sqrt(K) * 2^-24
    assert rel_l2(got, ref) < 3e-7 * math.sqrt(K) + 1e-6


@pytest.mark.parametrize("B,nt,ni", [(1, 16, 64), (2, 256, 1024), (1, 0, 333), (1, 7, 1), (2, 256, 4096)])
def test_joint_attention(B, nt, ni):
    import torch
    rng = np.random.default_rng(nt * 7 + ni)
    N = nt + ni
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((B, 24, N, 64)).astype(np.float32) * s) for s in (1.5, 1.5, 1))
    ot = torch.full((B, max(nt, 1), 1536), -1, dtype=torch.int16, device="cuda")
    oi = torch.full((B, max(ni, 1), 1536), -1, dtype=torch.int16, device="cuda")
    L.lens_op_attention(dev(q), dev(k), dev(v), B, nt, ni, ot, oi)
    _sync()
    heads = 24 if N <= 1100 else 4      # the oracle is O(N^2); sample heads at long N
    ref = o.attention(bf16_to_f64(q)[:, :heads], bf16_to_f64(k)[:, :heads], bf16_to_f64(v)[:, :heads])
    ref = ref.transpose(0, 2, 1, 3).reshape(B, N, heads * 64)
    got = np.concatenate([bf16_to_f64(host(ot))[:, :nt], bf16_to_f64(host(oi))[:, :ni]], axis=1)[..., :heads * 64]
    assert cos_sim(got, ref) > 0.9999
    assert rel_l2(got, ref) < 1e-2
    assert np.max(np.abs(got - ref)) < 0.05


@pytest.mark.parametrize("nt,ni", [(256, 4096), (7, 333)])
def test_joint_attention_rows_do_not_depend_on_the_batch(nt, ni):
    """Each batch row's output bits are the same computed alone or next to another row:
    no CTA's arithmetic depends on the rest of the launch (the CFG split across ranks
    is bit-exact against the batched CFG sampler because of it)."""
    import torch
    rng = np.random.default_rng(ni + 1)
    N = nt + ni
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((2, 24, N, 64)).astype(np.float32) * s) for s in (1.5, 1.5, 1))

    def run(rows):
        B = len(rows)
        ot = torch.full((B, nt, 1536), -1, dtype=torch.int16, device="cuda")
        oi = torch.full((B, ni, 1536), -1, dtype=torch.int16, device="cuda")
        qs, ks, vs = (dev(np.ascontiguousarray(a[rows])) for a in (q, k, v))
        L.lens_op_attention(qs, ks, vs, B, nt, ni, ot, oi)
        _sync()
        return host(ot), host(oi)

    bt, bi = run([0, 1])
    for r in (0, 1):
        at, ai = run([r])
        assert np.array_equal(at[0], bt[r]) and np.array_equal(ai[0], bi[r])


def test_euler_cfg_op():
    import torch
    rng = np.random.default_rng(9)
    n = 100_003
    x, vc, vu = (rng.standard_normal(n).astype(np.float32) for _ in range(3))
    xd = dev(x)
    L.lens_op_euler_cfg(xd, dev(vc), dev(vu), n, 0.25, 5.0)
    _sync()
    ref = o.euler(x.astype(np.float64), o.cfg_combine(vc.astype(np.float64), vu.astype(np.float64), 5.0), 0.25)
    assert np.allclose(host(xd), ref, rtol=1e-6, atol=1e-5)
    xd = dev(x)
    L.lens_op_euler_cfg(xd, dev(vc), None, n, 0.5, 1.0)
    _sync()
    assert np.allclose(host(xd), x - 0.5 * vc, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("B,nt,ni,lens", [(2, 16, 64, [5, 16]), (2, 256, 1024, [0, 200]), (3, 130, 333, [129, 1, 64])])
def test_joint_attention_text_padding(B, nt, ni, lens):
    """Text keys at and past each row's valid length are masked (length 0 masks
    whole key tiles before any valid key is seen)."""
    import torch
    rng = np.random.default_rng(nt + ni)
    N = nt + ni
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((B, 24, N, 64)).astype(np.float32) * s) for s in (1.5, 1.5, 1))
    ot = torch.full((B, nt, 1536), -1, dtype=torch.int16, device="cuda")
    oi = torch.full((B, ni, 1536), -1, dtype=torch.int16, device="cuda")
    L.lens_op_attention_masked(dev(q), dev(k), dev(v), B, nt, ni, lens, ot, oi)
    _sync()
    heads = 24 if N <= 600 else 4
    mask = o.text_key_mask(B, nt, ni, lens)
    ref = o.attention(bf16_to_f64(q)[:, :heads], bf16_to_f64(k)[:, :heads], bf16_to_f64(v)[:, :heads], mask)
    ref = ref.transpose(0, 2, 1, 3).reshape(B, N, heads * 64)
    got = np.concatenate([bf16_to_f64(host(ot)), bf16_to_f64(host(oi))], axis=1)[..., :heads * 64]
    assert np.all(np.isfinite(got))
    assert cos_sim(got, ref) > 0.9999 and rel_l2(got, ref) < 1e-2
