"""Seeded synthetic inputs for the Lens MMDiT denoiser: weights, latents, text features.

This module only draws numbers. It holds none of the denoiser's arithmetic, so the
CPU oracle and the CUDA library can both be fed from it without sharing any part of
the computation. Everything is deterministic in (seed, tensor index).

Shapes follow the Lens DiT configuration that the MLX port article
("Lens-Turbo-3.8B-bf16", config.json field list) and the 4-bit port article
("Lens-3.8B-4bit", DiT section) print: 48 dual-stream blocks, hidden 1536,
24 heads x 64, RoPE axes [8, 28, 28], 128-channel patchified input, 32-channel
latent, 2x2 patches, four GPT-OSS feature layers of 2880.  The gated MLP inner
size 4096 and the 9216-wide AdaLN projection come from the architecture arithmetic
on the Lens blog ("Overview": "1536x4096", "1536x9216").

Values (the plainest reading of the synthetic set-up):
  * matrices:   N(0, 1) * 0.02, rounded to bf16 (round to nearest even)
  * biases:     0
  * norm gains: 1.0
Options exist to draw random biases and gains, so tests can prove those terms are
applied.  Text features and image tokens are N(0, 1).
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np

__all__ = [
    "LensDims", "LENS", "TINY", "weight_specs", "make_weight", "make_weights",
    "f32_to_bf16_bits", "bf16_bits_to_f32", "text_features", "image_tokens",
    "latent_normal", "WORKLOADS", "Workload",
]


@dataclasses.dataclass(frozen=True)
class LensDims:
    num_blocks: int = 48
    hidden: int = 1536
    heads: int = 24
    head_dim: int = 64
    mlp_hidden: int = 4096
    latent_channels: int = 32
    patch: int = 2
    txt_layers: int = 4
    txt_dim: int = 2880
    rope_axes: Tuple[int, int, int] = (8, 28, 28)
    rope_theta: float = 10000.0
    eps: float = 1e-6
    freq_dim: int = 256          # sinusoidal timestep features

    @property
    def in_channels(self) -> int:
        return self.latent_channels * self.patch * self.patch

    @property
    def mod_dim(self) -> int:    # shift/scale/gate for attention and MLP
        return 6 * self.hidden

    def with_blocks(self, n: int) -> "LensDims":
        return dataclasses.replace(self, num_blocks=n)


LENS = LensDims()
# A toy model with the same structure, for fp64 oracle self-tests.
TINY = LensDims(num_blocks=2, hidden=64, heads=4, head_dim=16, mlp_hidden=96,
                latent_channels=4, patch=2, txt_layers=4, txt_dim=24,
                rope_axes=(4, 6, 6), freq_dim=16)


# ---------------------------------------------------------------- bf16 codec
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), round to nearest even. No NaNs expected."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------- weights
def weight_specs(d: LensDims = LENS) -> List[Tuple[str, Tuple[int, ...], str]]:
    """Canonical tensor list: (name, shape [out, in] for matrices, kind).

    Names are the tensor names the MLX port article lists for the Lens DiT
    (img_in, txt_in, txt_norm.0-3, time_text_embed.timestep_embedder, img_mod /
    txt_mod, attn.img_qkv / attn.txt_qkv, attn.norm_q / norm_k / norm_added_q /
    norm_added_k, attn.to_out / attn.to_add_out, img_mlp / txt_mlp w1 w2 w3,
    norm_out.linear, proj_out) under a `transformer_blocks.{i}.` prefix for blocks.
    The order fixes the per-tensor random stream.
    """
    D, F, hd = d.hidden, d.mlp_hidden, d.head_dim
    s: List[Tuple[str, Tuple[int, ...], str]] = []

    def lin(name, out_f, in_f):
        s.append((name + ".weight", (out_f, in_f), "matrix"))
        s.append((name + ".bias", (out_f,), "bias"))

    te = "time_text_embed.timestep_embedder"
    lin(te + ".linear_1", D, d.freq_dim)
    lin(te + ".linear_2", D, D)
    for l in range(d.txt_layers):
        s.append((f"txt_norm.{l}.weight", (d.txt_dim,), "gain"))
    lin("txt_in", D, d.txt_layers * d.txt_dim)
    lin("img_in", D, d.in_channels)
    for i in range(d.num_blocks):
        p = f"transformer_blocks.{i}."
        lin(p + "img_mod", d.mod_dim, D)
        lin(p + "txt_mod", d.mod_dim, D)
        lin(p + "attn.img_qkv", 3 * D, D)
        lin(p + "attn.txt_qkv", 3 * D, D)
        for g in ("norm_q", "norm_k", "norm_added_q", "norm_added_k"):
            s.append((p + f"attn.{g}.weight", (hd,), "gain"))
        lin(p + "attn.to_out", D, D)
        lin(p + "attn.to_add_out", D, D)
        for st in ("img_mlp", "txt_mlp"):
            lin(p + st + ".w1", F, D)
            lin(p + st + ".w3", F, D)
            lin(p + st + ".w2", D, F)
    lin("norm_out.linear", 2 * D, D)
    lin("proj_out", d.in_channels, D)
    return s


def _stream(seed: int, index: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(index)])))


def make_weight(spec_index: int, shape: Tuple[int, ...], kind: str, seed: int = 0,
                std: float = 0.02, bias_std: float = 0.0, gain_std: float = 0.0) -> np.ndarray:
    """One tensor as bf16 bits (uint16), drawn from stream (seed, spec_index)."""
    n = int(np.prod(shape))
    if kind == "matrix":
        x = _stream(seed, spec_index).standard_normal(n, dtype=np.float32)
        x *= np.float32(std)
    elif kind == "bias":
        if bias_std == 0.0:
            return np.zeros(shape, np.uint16)
        x = _stream(seed, spec_index).standard_normal(n, dtype=np.float32) * np.float32(bias_std)
    elif kind == "gain":
        if gain_std == 0.0:
            return np.full(shape, 0x3F80, np.uint16)      # bf16 1.0
        x = 1.0 + _stream(seed, spec_index).standard_normal(n, dtype=np.float32) * np.float32(gain_std)
    else:
        raise ValueError(kind)
    return f32_to_bf16_bits(x.astype(np.float32)).reshape(shape)


def make_weights(d: LensDims = LENS, seed: int = 0, std: float = 0.02, bias_std: float = 0.0,
                 gain_std: float = 0.0, names: Optional[Iterable[str]] = None,
                 threads: Optional[int] = None) -> Dict[str, np.ndarray]:
    """All (or the named) tensors as bf16 bits, generated in parallel threads."""
    specs = weight_specs(d)
    want = None if names is None else set(names)
    jobs = [(i, n, sh, k) for i, (n, sh, k) in enumerate(specs) if want is None or n in want]
    threads = threads or min(32, os.cpu_count() or 1)

    def one(job):
        i, n, sh, k = job
        return n, make_weight(i, sh, k, seed, std, bias_std, gain_std)

    with ThreadPoolExecutor(threads) as ex:
        return dict(ex.map(one, jobs))


# ---------------------------------------------------------------- activations
def text_features(B: int, n_txt: int, seed: int, d: LensDims = LENS) -> np.ndarray:
    """[B, n_txt, txt_layers, txt_dim] bf16 bits, N(0, 1)."""
    x = _stream(seed, 1_000_001).standard_normal((B, n_txt, d.txt_layers, d.txt_dim), dtype=np.float32)
    return f32_to_bf16_bits(x).reshape(B, n_txt, d.txt_layers, d.txt_dim)


def image_tokens(B: int, n_img: int, seed: int, d: LensDims = LENS) -> np.ndarray:
    """[B, n_img, in_channels] fp32, N(0, 1) (patchified latent tokens)."""
    return _stream(seed, 1_000_002).standard_normal((B, n_img, d.in_channels), dtype=np.float32)


def latent_normal(B: int, h_lat: int, w_lat: int, seed: int, d: LensDims = LENS) -> np.ndarray:
    """[B, latent_channels, h_lat, w_lat] fp32, N(0, 1)."""
    return _stream(seed, 1_000_003).standard_normal((B, d.latent_channels, h_lat, w_lat), dtype=np.float32)


# ---------------------------------------------------------------- workloads
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_blocks: int
    grid_h: int          # image tokens per column (latent height / 2)
    grid_w: int
    n_txt: int
    batch: int
    t: float = 0.5       # timestep for single-forward workloads
    steps: int = 0       # 0 = single forward
    guidance: float = 1.0
    seed: int = 0

    @property
    def n_img(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def height_px(self) -> int:   # one token = 16 x 16 pixels (8x VAE, 2x2 patch)
        return 16 * self.grid_h

    @property
    def width_px(self) -> int:
        return 16 * self.grid_w


WORKLOADS = {
    "block_8x8": Workload("one block, 8x8 image tokens + 16 text, t=0.7", 1, 8, 8, 16, 1, t=0.7, seed=0),
    "fwd_512": Workload("48-block forward at 512^2 (1024 img + 128 txt tokens)", 48, 32, 32, 128, 1, t=0.5, seed=2),
    "turbo_1024": Workload("4-step Euler sample at 1024^2 (4096 img + 256 txt), no CFG", 48, 64, 64, 256, 1,
                           steps=4, guidance=1.0, seed=3),
    "cfg_1024": Workload("20-step Euler sample at 1024^2 with CFG 5 (batched cond/uncond)", 48, 64, 64, 256, 1,
                         steps=20, guidance=5.0, seed=4),
    "cfg_1440": Workload("50-step Euler sample at 1440^2 (8100 img + 256 txt) with CFG 5", 48, 90, 90, 256, 1,
                         steps=50, guidance=5.0, seed=5),
    "cfg_1024x2048": Workload("50-step Euler sample at 1024x2048 (64x128 tokens) with CFG 5", 48, 64, 128, 256, 1,
                              steps=50, guidance=5.0, seed=6),
}
