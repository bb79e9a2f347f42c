"""GPU parity of the int4 weight-only path against the CPU oracle: quantization
codes bit-exact (scales and biases equal), and the 4-bit GEMM against the oracle's
dequantized weights.  The kernel widens each weight once to bf16 (one rounding of
scale * code + bias), so against those bf16 values it must agree as tightly as the
bf16 GEMM does; against the exact dequantized weights the bf16 rounding bounds it."""
import numpy as np
import pytest

from lens_inputs import f32_to_bf16_bits
from oracle import lens_oracle as o
from tests.helpers import cos_sim, dev, host, rel_l2

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import flow_matching_mmdit_b200 as L  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L.load_library()


def _bits_to_f32(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32)


def unpack_codes(words: np.ndarray, rows: int, k: int) -> np.ndarray:
    """The documented device layout -> codes [rows, k]."""
    w = words.view(np.uint32).reshape(rows, k // 8)
    q = np.empty((rows, k // 8, 8), np.uint8)
    for j in range(4):
        q[:, :, 2 * j] = (w >> (4 * j)) & 0xF
        q[:, :, 2 * j + 1] = (w >> (16 + 4 * j)) & 0xF
    return q.reshape(rows, k)


def _quantize_gpu(wbits, rows, k):
    codes = torch.zeros((rows, k // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((k // 64, rows), dtype=torch.int32, device="cuda")
    L.lens_op_quantize_w4(dev(wbits), rows, k, codes, scales)
    torch.cuda.synchronize()
    return codes, scales


def _weights(rows, k, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((rows, k)) * 0.02).astype(np.float32)
    w[0, :64] = 0.375                                   # constant group: scale 0
    w[1, :64] = np.tile(np.arange(16, dtype=np.float32), 4) * 0.25 - 1.0   # codes on the grid
    if k >= 128:
        w[2, 64:128] = rng.standard_normal(64).astype(np.float32) * 40.0   # a wide group
    return f32_to_bf16_bits(w)


@pytest.mark.parametrize("rows,k", [(384, 1536), (128, 4096), (9216, 1536)])
def test_quantize_matches_oracle_bit_for_bit(rows, k):
    wb = _weights(rows, k, 5 + rows)
    codes, scales = _quantize_gpu(wb, rows, k)
    q_ref, s_ref, b_ref = o.quantize_w4(wb)
    q = unpack_codes(host(codes), rows, k)
    assert np.array_equal(q, q_ref)
    sw = host(scales).view(np.uint32).T                 # [rows, k / 64]
    assert np.array_equal(_bits_to_f32((sw & 0xFFFF).astype(np.uint16)), s_ref)
    assert np.array_equal(_bits_to_f32((sw >> 16).astype(np.uint16)), b_ref)


@pytest.mark.parametrize("M,N,K", [(128, 256, 1536), (300, 384, 1536), (4352, 1536, 4096), (1, 128, 64)])
def test_gemm_w4_matches_oracle(M, N, K):
    rng = np.random.default_rng(M + N + K)
    A = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    wb = _weights(N, K, 17 + N)
    bias = (rng.standard_normal(N) * 0.1).astype(np.float32)
    codes, scales = _quantize_gpu(wb, N, K)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    L.lens_op_gemm_w4(dev(A), codes, scales, dev(bias), C, M, N, K)
    torch.cuda.synchronize()
    got = host(C).astype(np.float64)
    Wq = o.dequantize_w4(*o.quantize_w4(wb))
    Af = o.upcast(A)
    # the same weights rounded once to bf16, as the kernel feeds them to the MMA
    Wb = o.upcast(f32_to_bf16_bits(Wq.astype(np.float32)))
    tight = Af @ Wb.T + bias
    assert rel_l2(got, tight) < 3e-7 * np.sqrt(K) + 1e-6, rel_l2(got, tight)
    exact = Af @ Wq.T + bias
    assert cos_sim(got, exact) > 0.99999 and rel_l2(got, exact) < 4e-3, (cos_sim(got, exact), rel_l2(got, exact))


# ------------------------------------------------------------------ the 4-bit model
from lens_inputs import LENS, image_tokens, make_weights, text_features  # noqa: E402
from tests.helpers import bf16_to_f64  # noqa: E402,F401


@pytest.fixture(scope="module")
def small_w4():
    """Two-block model with random biases and gains, created with weight_bits = 4; the
    oracle evaluates the same weights quantized by its own definition."""
    d = LENS.with_blocks(2)
    w = make_weights(d, seed=0, bias_std=0.02, gain_std=0.1)
    cfg = L.lens_dit_default_config()
    cfg.num_blocks, cfg.weight_bits = 2, 4
    cfg.max_batch, cfg.max_img_tokens, cfg.max_txt_tokens = 4, 4096, 256
    h = L.lens_dit_create(cfg, w)
    yield d, w, o.Weights(o.quantize_model_w4(w)), h
    h.destroy()


def test_w4_modulation_matches_oracle(small_w4):
    d, w, Wq, h = small_w4
    t = [0.7, 0.0, 1.0]
    modw = d.num_blocks * 2 * 9216 + 3072
    temb = torch.empty((len(t), 1536), dtype=torch.float32, device="cuda")
    mod = torch.empty((len(t), modw), dtype=torch.float32, device="cuda")
    L.lens_dit_op_timestep(h, t, temb, mod)
    L.lens_dit_sync(h)
    te = o.timestep_embedding(Wq, np.array(t), d.freq_dim)
    ref = np.concatenate([o.linear(Wq, f"transformer_blocks.{i}.{s}_mod", o.silu(te))
                          for i in range(d.num_blocks) for s in ("img", "txt")] +
                         [o.linear(Wq, "norm_out.linear", o.silu(te))], axis=1)
    got = host(mod)
    assert cos_sim(got, ref) > 0.99999 and rel_l2(got, ref) < 5e-3, (cos_sim(got, ref), rel_l2(got, ref))


@pytest.mark.parametrize("B,gh,gw,nt", [(1, 8, 8, 16), (2, 16, 12, 40)])
def test_w4_forward_matches_oracle(small_w4, B, gh, gw, nt):
    d, w, Wq, h = small_w4
    X = image_tokens(B, gh * gw, 3 + B)
    E = text_features(B, nt, 4 + B)
    t = [0.6, 0.25][:B]
    v = torch.empty((B, gh * gw, 128), dtype=torch.float32, device="cuda")
    L.lens_dit_forward(h, dev(X), B, gh, gw, dev(E), nt, t, v)
    L.lens_dit_sync(h)
    ref = o.forward(Wq, d, X, gh, gw, E, t)
    assert cos_sim(host(v), ref) >= 0.999 and rel_l2(host(v), ref) <= 2e-2, (cos_sim(host(v), ref), rel_l2(host(v), ref))


def test_w4_sampler_matches_oracle(small_w4):
    d, w, Wq, h = small_w4
    B, gh, gw, nt, seed, steps = 1, 8, 6, 16, 321, 3
    Ec = text_features(B, nt, 25)
    out = torch.empty((B, 32, 2 * gh, 2 * gw), dtype=torch.float32, device="cuda")
    L.lens_sample_euler(h, dev(Ec), None, B, nt, 16 * gh, 16 * gw, steps, 5.0, seed, out)
    L.lens_dit_sync(h)
    ref = o.sample(Wq, d, Ec, None, B, gh, gw, steps, 5.0, seed)
    got = host(out)
    assert cos_sim(got, ref) >= 0.99 and rel_l2(got, ref) <= 5e-2, (cos_sim(got, ref), rel_l2(got, ref))
