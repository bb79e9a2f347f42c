"""The allocation-free timestep embedding (for callers that cannot call cudaMalloc,
such as a plugin whose host owns all device memory) must agree with the handle's
timestep embedding, call after call, although every call shares one fixed device
array for its intermediates.  Collected last on purpose."""
import numpy as np
import pytest

from lens_inputs import LENS, make_weights
from oracle import lens_oracle as o
from tests.helpers import bf16_to_f64, dev, host, rel_l2

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import flow_matching_mmdit_b200 as L  # noqa: E402


def test_noalloc_timestep_embedding_matches_handle_path():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = LENS.with_blocks(1)
    w = make_weights(d, seed=5, bias_std=0.05)
    cfg = L.lens_dit_default_config()
    cfg.num_blocks = 1
    cfg.max_batch, cfg.max_img_tokens, cfg.max_txt_tokens = 1, 64, 16
    h = L.lens_dit_create(cfg, w)
    try:
        p = "time_text_embed.timestep_embedder."
        w1, w2 = dev(w[p + "linear_1.weight"]), dev(w[p + "linear_2.weight"])
        b1 = dev(bf16_to_f64(w[p + "linear_1.bias"]).astype(np.float32))
        b2 = dev(bf16_to_f64(w[p + "linear_2.bias"]).astype(np.float32))
        t64 = list(np.linspace(0.0, 1.0, 64))        # the largest T: the whole array in use
        for t in ([0.7, 0.0, 1.0, 0.333, 0.5], [0.25, 0.9, 0.01], t64, [0.125]):   # calls in a row
            T = len(t)
            ref = torch.empty((T, 1536), dtype=torch.float32, device="cuda")
            L.lens_dit_op_timestep(h, t, ref, None)
            got = torch.full((T, 1536), float("nan"), dtype=torch.float32, device="cuda")
            L.lens_op_timestep_embed_noalloc(t, w1, b1, w2, b2, got)
            torch.cuda.synchronize()
            assert np.all(np.isfinite(host(got)))
            assert rel_l2(host(got), host(ref)) < 1e-5
            # and directly against the oracle (fp64) on the same fp32 timesteps
            exact = o.timestep_embedding(o.Weights(w), np.asarray(t, np.float32).astype(np.float64), 256)
            assert rel_l2(host(got), exact) < 1e-3
        # sizes beyond the fixed array are rejected before any work is enqueued
        big = torch.empty((65, 1536), dtype=torch.float32, device="cuda")
        with pytest.raises(L.LensError) as ei:
            L.lens_op_timestep_embed_noalloc([0.5] * 65, w1, b1, w2, b2, big)
        assert ei.value.status == 2
        # misaligned weights are rejected: the rows are read 16 bytes at a time
        w1_off = torch.empty(w1.numel() + 8, dtype=w1.dtype, device="cuda")[1:1 + w1.numel()]
        with pytest.raises(L.LensError) as ei:
            L.lens_op_timestep_embed_noalloc([0.5], w1_off, b1, w2, b2, big)
        assert ei.value.status == 1
    finally:
        h.destroy()
