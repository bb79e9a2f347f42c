"""CPU oracle for the Lens MMDiT denoiser and its flow-matching Euler sampler.

TEST INFRASTRUCTURE. This module is the plain, slow, obviously-correct restatement of
what the denoiser computes, written from the pages' description in numpy (fp64 by
default).  It is used only by the tests, by `__graft_entry__.smoke()` and by the
`cpu_baseline` / `--impl reference` legs of `bench.py`.  The CUDA library never
imports, links or calls it, and it shares no code with the library: it takes bf16
weights as raw bit patterns and upcasts them itself.

Sources (page title, section):
  [blog]    "Lens" blog post (zjwfufu.github.io), sections "Overview" (block arithmetic:
            48 blocks, hidden 1536, 24 heads, gate/up/down 1536x4096, AdaLN 1536x9216,
            dual stream), "Exploring Image Editing" (CFG combination; "norm-rescaled").
  [paper]   "Lens: 重新思考基础文生图模型的训练效率" summary page, sections "前置知识 /
            Flow Matching 训练目标" (x_t = (1-t) x0 + t x1, v = x1 - x0; mu(n) linear
            interpolation of the timestep schedule by resolution) and "方法步骤详情"
            (RMSNorm + RoPE dual stream; mu = 1.06 at 512^2; 20 steps CFG 5.0; Turbo 4).
  [mlx]     "深入 Lens-Turbo-3.8B-bf16 内核" article, sections "核心规格一览", "双流注意力机制",
            "自适应调制与 RMSNorm", "3D RoPE 旋转位置编码", "多层级文本特征融合",
            "Patchify 补丁化与输出投影", "guidance 1.0".
  [int4]    "从提示词到成图：Lens-3.8B-4bit完整管线解析", section 4 (DiT: 128-channel input,
            patch 2, 32-channel output, time_text_embed, axes [8, 28, 28]; int4 weights with
            group_size 64, sensitive layers in bf16, about 2.35 GB) and section 6
            (pipeline call with steps and seed).
  [survey]  "SOTA image generation" survey page, sections "CFG：无分类器引导" and
            "交叉注意力与条件注入" (joint attention over the concatenated sequence).

Where the pages leave a step open the plainest reading is taken; each such reading is
marked READING below.  Parity of the whole 48-block forward and of the sampler is
pinned only through the composition of the pinned parts (no worked example exists).
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Mapping, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64


# ============================================================ weights
def upcast(w, dtype=F64) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float, exactly (bf16 is the top half of fp32)."""
    w = np.asarray(w)
    if w.dtype == np.uint16:
        return (w.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(dtype)
    return w.astype(dtype)


class Weights:
    """Read-only view of a name -> bf16-bits mapping with on-demand upcast."""

    def __init__(self, tensors: Mapping[str, np.ndarray], dtype=F64):
        self.t = tensors
        self.dtype = dtype

    def __call__(self, name: str) -> np.ndarray:
        return upcast(self.t[name], self.dtype)

    def has(self, name: str) -> bool:
        return name in self.t


def linear(W: Weights, name: str, x: np.ndarray) -> np.ndarray:
    """y = x W^T + b with W stored [out, in]; a missing bias counts as zero.
    READING: every Linear may carry a bias (the pages do not say which do)."""
    y = x @ W(name + ".weight").T
    if W.has(name + ".bias"):
        y = y + W(name + ".bias")
    return y


# ============================================================ elementwise pieces
def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x)."""
    return x / (1.0 + np.exp(-x))


def rms_norm(x: np.ndarray, eps: float, gain: Optional[np.ndarray] = None) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis, times an optional gain.
    [mlx] "自适应调制与 RMSNorm": the block norm is RMSNorm (rms_norm: true).
    READING: eps = 1e-6 (not stated)."""
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if gain is None else y * gain


# ============================================================ patchify (a1, a13)
def patchify(Z: np.ndarray, p: int = 2) -> np.ndarray:
    """[B, C, p*h, p*w] latent -> [B, h*w, C*p*p] tokens.
    [mlx] "Patchify 补丁化与输出投影": 2x2 patches of the 32-channel latent give the
    128-channel input (2*2*32 = 128).
    READING: tokens in row-major (i, j) order; features channel-major, then the
    patch row, then the patch column: X[b, i*w+j, c*p*p + r*p + s] = Z[b, c, p*i+r, p*j+s]."""
    B, C, H, W_ = Z.shape
    h, w = H // p, W_ // p
    return Z.reshape(B, C, h, p, w, p).transpose(0, 2, 4, 1, 3, 5).reshape(B, h * w, C * p * p)


def unpatchify(X: np.ndarray, h: int, w: int, C: int, p: int = 2) -> np.ndarray:
    """Inverse of `patchify`: [B, h*w, C*p*p] -> [B, C, p*h, p*w]."""
    B = X.shape[0]
    return X.reshape(B, h, w, C, p, p).transpose(0, 3, 1, 4, 2, 5).reshape(B, C, p * h, p * w)


# ============================================================ positions and RoPE (a2)
def position_ids(grid_h: int, grid_w: int, n_txt: int) -> np.ndarray:
    """[n_txt + grid_h*grid_w, 3] ids for the joint sequence, text first.
    READING: text tokens get (0, 0, 0); image token (i, j) gets (0, i, j)."""
    ii, jj = np.meshgrid(np.arange(grid_h), np.arange(grid_w), indexing="ij")
    img = np.stack([np.zeros(grid_h * grid_w, np.int64), ii.ravel(), jj.ravel()], axis=1)
    return np.concatenate([np.zeros((n_txt, 3), np.int64), img], axis=0)


def rope_angles(ids: np.ndarray, axes: Sequence[int], theta: float) -> np.ndarray:
    """[N, sum(axes)/2] rotation angles.  [mlx] "3D RoPE 旋转位置编码": three axes of
    8, 28 and 28 dims, which add up to the head dim 64.
    READING: axis a owns a contiguous segment of the head dims; its pair m turns by
    pos_a * theta^(-2m/d_a), theta = 10000."""
    cols = []
    for a, da in enumerate(axes):
        m = np.arange(da // 2, dtype=F64)
        omega = theta ** (-2.0 * m / da)
        cols.append(ids[:, a:a + 1].astype(F64) * omega[None, :])
    return np.concatenate(cols, axis=1)


def apply_rope(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate adjacent pairs (2k, 2k+1) of the last axis by angles[token, k].
    x: [..., N, d]; angles: [N, d/2].  READING: interleaved pairs."""
    c, s = np.cos(angles), np.sin(angles)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ============================================================ timestep embedding (a4)
def timestep_features(t: np.ndarray, dim: int = 256) -> np.ndarray:
    """Sinusoidal features [len(t), dim]: first half cos, second half sin of
    1000*t*f_k with f_k = exp(-ln(10000) k / (dim/2)).
    [mlx] names the time_text_embed.timestep_embedder MLP; the 256-wide sinusoid and
    the 1000 scale are a READING (FLUX-family convention)."""
    half = dim // 2
    f = np.exp(-math.log(10000.0) * np.arange(half, dtype=F64) / half)
    arg = 1000.0 * np.asarray(t, F64)[:, None] * f[None, :]
    return np.concatenate([np.cos(arg), np.sin(arg)], axis=1)


def timestep_embedding(W: Weights, t: np.ndarray, freq_dim: int) -> np.ndarray:
    """temb = linear_2(SiLU(linear_1(sinusoid(t)))).  READING: temb depends on t only
    (text enters through txt_in)."""
    e = timestep_features(t, freq_dim).astype(W.dtype)
    p = "time_text_embed.timestep_embedder"
    return linear(W, p + ".linear_2", silu(linear(W, p + ".linear_1", e)))


def modulation(W: Weights, name: str, temb: np.ndarray, parts: int) -> Tuple[np.ndarray, ...]:
    """AdaLN projection of SiLU(temb) split into `parts` chunks of the hidden size.
    [blog] "Overview": a 1536x9216 projection per stream makes shift, scale and gate
    for the attention and for the gated MLP.  [mlx] "自适应调制": img_mod / txt_mod.
    READING: SiLU before the Linear; chunk order (shift1, scale1, gate1, shift2,
    scale2, gate2)."""
    m = linear(W, name, silu(temb))
    return tuple(np.split(m, parts, axis=-1))


# ============================================================ text input (a3)
def text_input(W: Weights, E: np.ndarray, eps: float) -> np.ndarray:
    """[B, T, L, Dt] features of L encoder layers -> [B, T, hidden].
    [mlx] "多层级文本特征融合": txt_norm.0..3 normalise the four layers, which are then
    fused; [paper] "方法步骤详情": the layers are concatenated to D = 1536.
    READING: RMSNorm each layer slice with its gain, concatenate layer-major, txt_in."""
    L = E.shape[2]
    parts = [rms_norm(E[:, :, l, :], eps, W(f"txt_norm.{l}.weight")) for l in range(L)]
    return linear(W, "txt_in", np.concatenate(parts, axis=-1))


# ============================================================ attention (a8)
def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, key_mask: Optional[np.ndarray] = None) -> np.ndarray:
    """softmax(q k^T / sqrt(d)) v per head.  q: [B, H, Nq, d]; k, v: [B, H, N, d];
    key_mask [B, N] (True = the key is attended) or None for no mask.
    [survey] "交叉注意力与条件注入": text and image tokens are concatenated into one
    sequence for joint attention; [mlx] "双流注意力机制"; [blog] "Exploring Text
    Encoder": zero-padded text tokens are masked out, so the DiT never sees them."""
    d = q.shape[-1]
    out = np.empty(q.shape[:-1] + (v.shape[-1],), dtype=np.result_type(q, v))
    for b in range(q.shape[0]):                   # heads are independent; one at a time
        for h in range(q.shape[1]):
            s = (q[b, h] @ k[b, h].T) / math.sqrt(d)
            if key_mask is not None:
                s = np.where(key_mask[b][None, :], s, -np.inf)
            s = s - s.max(axis=-1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=-1, keepdims=True)
            out[b, h] = p @ v[b, h]
    return out


# ============================================================ one dual-stream block (a6-a12)
def _heads(x: np.ndarray, H: int) -> np.ndarray:          # [B, N, H*d] -> [B, H, N, d]
    B, N, HD = x.shape
    return x.reshape(B, N, H, HD // H).transpose(0, 2, 1, 3)


def _unheads(x: np.ndarray) -> np.ndarray:                # [B, H, N, d] -> [B, N, H*d]
    B, H, N, d = x.shape
    return x.transpose(0, 2, 1, 3).reshape(B, N, H * d)


def gated_mlp(W: Weights, name: str, x: np.ndarray) -> np.ndarray:
    """w2(SiLU(w1 x) * w3 x).  [blog] "Overview": gate, up, down of 1536x4096;
    [mlx] gate_mlp: true with w1/w2/w3.  READING: w1 is the gated branch."""
    return linear(W, name + ".w2", silu(linear(W, name + ".w1", x)) * linear(W, name + ".w3", x))


def text_key_mask(B: int, n_txt: int, n_img: int, txt_len: Optional[Sequence[int]]) -> Optional[np.ndarray]:
    """[B, n_txt + n_img] attention key mask: text key n of sample b is attended iff
    n < txt_len[b]; image keys always.  None (no mask) when txt_len is None.
    READING: padding sits at the end of the text tokens ("zero-pad to the same size")."""
    if txt_len is None:
        return None
    m = np.ones((B, n_txt + n_img), bool)
    for b in range(B):
        m[b, int(txt_len[b]):n_txt] = False
    return m


def block(W: Weights, i: int, h_img: np.ndarray, h_txt: np.ndarray, temb: np.ndarray,
          angles: np.ndarray, heads: int, eps: float,
          img_rows: Optional[np.ndarray] = None, txt_rows: Optional[np.ndarray] = None,
          txt_len: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """One dual-stream MMDiT block on h_img [B, Ni, D], h_txt [B, Nt, D], temb [B, D].

    Each stream: AdaLN-modulated RMSNorm, its own fused QKV, per-head QK-RMSNorm
    (norm_q/norm_k for image, norm_added_q/norm_added_k for text), RoPE, then one
    joint attention over [text; image]; the outputs split back to to_add_out / to_out
    with a gated residual, then a gated SwiGLU MLP with a gated residual.
    [blog] "Overview"; [paper] "前置知识 / MMDiT" (per-stream RMSNorm-Attention-MLP with
    joint attention); [mlx] "双流注意力机制" and "自适应调制与 RMSNorm".
    READINGS: QKV rows are q | k | v, each head-major; QK-norm before RoPE; no gain on
    the pre-modulation RMSNorm; the gates multiply the branch output.

    img_rows / txt_rows select the query rows whose outputs are wanted (all when None);
    keys and values always cover every token.  txt_len [B] masks text keys at and past
    each sample's valid length (padding).  Returns the selected rows.
    """
    p = f"transformer_blocks.{i}."
    B, Ni, D = h_img.shape
    Nt = h_txt.shape[1]
    sh1i, sc1i, g1i, sh2i, sc2i, g2i = [m[:, None, :] for m in modulation(W, p + "img_mod", temb, 6)]
    sh1t, sc1t, g1t, sh2t, sc2t, g2t = [m[:, None, :] for m in modulation(W, p + "txt_mod", temb, 6)]

    a_img = (1.0 + sc1i) * rms_norm(h_img, eps) + sh1i
    a_txt = (1.0 + sc1t) * rms_norm(h_txt, eps) + sh1t
    qi, ki, vi = np.split(linear(W, p + "attn.img_qkv", a_img), 3, axis=-1)
    qt, kt, vt = np.split(linear(W, p + "attn.txt_qkv", a_txt), 3, axis=-1)
    qi = rms_norm(_heads(qi, heads), eps, W(p + "attn.norm_q.weight"))
    ki = rms_norm(_heads(ki, heads), eps, W(p + "attn.norm_k.weight"))
    qt = rms_norm(_heads(qt, heads), eps, W(p + "attn.norm_added_q.weight"))
    kt = rms_norm(_heads(kt, heads), eps, W(p + "attn.norm_added_k.weight"))
    vi, vt = _heads(vi, heads), _heads(vt, heads)

    Q = apply_rope(np.concatenate([qt, qi], axis=2), angles)
    K = apply_rope(np.concatenate([kt, ki], axis=2), angles)
    V = np.concatenate([vt, vi], axis=2)

    ir = np.arange(Ni) if img_rows is None else np.asarray(img_rows)
    tr = np.arange(Nt) if txt_rows is None else np.asarray(txt_rows)
    q_sel = np.concatenate([tr, Nt + ir])
    O = _unheads(attention(Q[:, :, q_sel, :], K, V, text_key_mask(B, Nt, Ni, txt_len)))
    O_txt, O_img = O[:, :len(tr)], O[:, len(tr):]

    hi = h_img[:, ir] + g1i * linear(W, p + "attn.to_out", O_img)
    ht = h_txt[:, tr] + g1t * linear(W, p + "attn.to_add_out", O_txt)
    hi = hi + g2i * gated_mlp(W, p + "img_mlp", (1.0 + sc2i) * rms_norm(hi, eps) + sh2i)
    ht = ht + g2t * gated_mlp(W, p + "txt_mlp", (1.0 + sc2t) * rms_norm(ht, eps) + sh2t)
    return hi, ht


# ============================================================ final layer (a13)
def final_layer(W: Weights, h_img: np.ndarray, temb: np.ndarray, eps: float) -> np.ndarray:
    """norm_out.linear (AdaLN-continuous) then proj_out to 128 = 2*2*32 per token.
    [mlx] "Patchify 补丁化与输出投影": norm_out.linear and proj_out project back.
    READING: chunk order (scale, shift)."""
    scale, shift = modulation(W, "norm_out.linear", temb, 2)
    y = (1.0 + scale[:, None, :]) * rms_norm(h_img, eps) + shift[:, None, :]
    return linear(W, "proj_out", y)


# ============================================================ whole forward
def forward(W: Weights, dims, X: np.ndarray, grid_h: int, grid_w: int, E: np.ndarray,
            t: Sequence[float], blocks: Optional[int] = None,
            txt_len: Optional[Sequence[int]] = None) -> np.ndarray:
    """Velocity v [B, Ni, 128] of the denoiser for tokens X [B, Ni, 128], text
    features E [B, Nt, 4, 2880] (valid lengths txt_len [B], None = all valid) and
    per-sample timesteps t [B]."""
    n_blocks = dims.num_blocks if blocks is None else blocks
    dt = W.dtype
    temb = timestep_embedding(W, np.asarray(t, F64), dims.freq_dim)
    h_img = linear(W, "img_in", np.asarray(X, dt))
    h_txt = text_input(W, upcast(E, dt), dims.eps)
    ang = rope_angles(position_ids(grid_h, grid_w, E.shape[1]), dims.rope_axes, dims.rope_theta)
    for i in range(n_blocks):
        h_img, h_txt = block(W, i, h_img, h_txt, temb, ang, dims.heads, dims.eps, txt_len=txt_len)
    return final_layer(W, h_img, temb, dims.eps)


# ============================================================ noise (a1)
_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(v: np.ndarray) -> np.ndarray:
    """SplitMix64 output for state v (Steele, Lea and Flood, OOPSLA 2014; Vigna's
    splitmix64.c): add the golden gamma, then the two xor-shift-multiply rounds."""
    z = np.asarray(v, np.uint64) + _GOLDEN
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def noise(seed: int, n: int) -> np.ndarray:
    """n standard normals (fp32) from a seed, by Box-Muller on two SplitMix64 words.
    Element i: w1 = sm(seed ^ sm(2i)), w2 = sm(seed ^ sm(2i+1));
    u1 = ((w1 >> 11) + 1) 2^-53 in (0, 1]; u2 = (w2 >> 11) 2^-53 in [0, 1);
    z = sqrt(-2 ln u1) cos(2 pi u2).  [int4] section 6: the pipeline call takes a seed.
    READING: the generator itself (the pages name none)."""
    i = np.arange(n, dtype=np.uint64)
    s = np.uint64(seed)
    w1 = splitmix64(s ^ splitmix64(np.uint64(2) * i))
    w2 = splitmix64(s ^ splitmix64(np.uint64(2) * i + np.uint64(1)))
    u1 = ((w1 >> np.uint64(11)).astype(F64) + 1.0) * 2.0 ** -53
    u2 = (w2 >> np.uint64(11)).astype(F64) * 2.0 ** -53
    return (np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)).astype(np.float32)


# ============================================================ sampler (a14)
def cfg_combine(v_cond: np.ndarray, v_uncond: np.ndarray, scale: float) -> np.ndarray:
    """uncond + scale * (cond - uncond).  [blog] "Exploring Image Editing" and [survey]
    "CFG：无分类器引导" print this combination.  READING: plain CFG (the blog calls it
    norm-rescaled but prints no rescale)."""
    return v_uncond + scale * (v_cond - v_uncond)


def timesteps(steps: int) -> np.ndarray:
    """Uniform grid t_k = 1 - k/S, k = 0..S-1 (model input at step k).
    READING: uniform grid with no resolution shift (the shift is stated for training)."""
    return 1.0 - np.arange(steps, dtype=F64) / steps


def cfg_rescaled(v_cond: np.ndarray, v_uncond: np.ndarray, scale: float, phi: float) -> np.ndarray:
    """Norm-rescaled CFG.  [blog] "Exploring Image Editing" names Lens's guidance
    "norm-rescaled CFG" and says it drives the difference of two guided velocities
    towards zero, but prints only u + s (c - u).  READING: form the plain combination
    v = u + s (c - u), then pull its L2 norm back to the conditional one,
        v <- phi * v * |c| / |v| + (1 - phi) * v,
    with each norm taken over one sample's whole velocity (every axis but the first).
    phi = 0 is plain CFG, phi = 1 the full rescale; |v| = 0 leaves v unchanged."""
    v = cfg_combine(v_cond, v_uncond, scale)
    axes = tuple(range(1, v.ndim))
    nc = np.sqrt(np.sum(v_cond.astype(F64) ** 2, axis=axes, keepdims=True))
    nv = np.sqrt(np.sum(v.astype(F64) ** 2, axis=axes, keepdims=True))
    r = np.where(nv > 0, nc / np.where(nv > 0, nv, 1.0), 1.0)
    return phi * r * v + (1.0 - phi) * v


def time_shift(t, mu: float):
    """Resolution shift of a flow-matching time, t' = e^mu t / (e^mu t + 1 - t).
    [paper] "Flow Matching 训练目标" ties the timestep schedule at each resolution to
    a mu(n) "linear interpolation" and [paper] "方法步骤详情" gives mu = 1.06 for the
    512^2 stage, but no formula is printed.  READING: the exponential shift of the
    published flow-matching schedule (Esser et al. 2024, resolution-dependent
    shifting of timestep schedules), with e^mu the shift factor: t = 0 and t = 1
    stay fixed, mu = 0 is the identity, mu > 0 spends more of the steps near t = 1."""
    t = np.asarray(t, dtype=F64)
    a = np.exp(F64(mu))
    return a * t / (a * t + (1.0 - t))


def shift_mu(n_img_tokens: int, n1: int, mu1: float, n2: int, mu2: float) -> float:
    """mu linear in the image token count n through (n1, mu1) and (n2, mu2) ([paper]
    "Flow Matching 训练目标": mu(n) is a linear interpolation).  The pages give one
    point only: 512^2 (32 x 32 = 1024 tokens) at mu = 1.06; the other anchor is the
    caller's."""
    return float(mu1 + (mu2 - mu1) * (n_img_tokens - n1) / (n2 - n1))


def time_grid(steps: int, mu: Optional[float] = None) -> np.ndarray:
    """t_0 .. t_S (S + 1 values): the uniform grid 1 - k/S, shifted by time_shift(., mu)
    when mu is given.  Step k feeds the model t_k and moves by t_k - t_{k+1}."""
    t = 1.0 - np.arange(steps + 1, dtype=F64) / steps
    return t if mu is None else time_shift(t, mu)


def euler(x: np.ndarray, v: np.ndarray, dt: float) -> np.ndarray:
    """x_{t-dt} = x_t - dt * v.  [paper] "Flow Matching 训练目标": x_t = (1-t) x0 + t x1
    with v = x1 - x0, so integrating from t = 1 (noise) to t = 0 (data) subtracts v."""
    return x - dt * v


def sample_euler(velocity: Callable[[np.ndarray, float, bool], np.ndarray], x1: np.ndarray,
                 steps: int, guidance: float, mu: Optional[float] = None, phi: float = 0.0,
                 stop_after: Optional[int] = None) -> np.ndarray:
    """Integrate from t = 1 to 0 with S Euler steps.  velocity(x, t, cond) gives the
    conditional (cond=True) or unconditional prediction.  guidance == 1 evaluates the
    conditional model only ([mlx] "guidance 1.0": no doubled forward).  mu shifts the
    time grid (time_grid), phi rescales the guided velocity (cfg_rescaled); with
    neither, the steps are the uniform 1/S.  stop_after = k returns the state after
    the first k steps of the S-step grid (None = all S)."""
    x = x1
    tg = time_grid(steps, mu)
    for k in range(steps if stop_after is None else min(stop_after, steps)):
        t = float(tg[k])
        dt = 1.0 / steps if mu is None else float(tg[k] - tg[k + 1])
        vc = velocity(x, t, True)
        if guidance == 1.0:
            v = vc
        else:
            vu = velocity(x, t, False)
            v = cfg_combine(vc, vu, guidance) if phi == 0.0 else cfg_rescaled(vc, vu, guidance, phi)
        x = euler(x, v, dt)
    return x


def sample(W: Weights, dims, E_cond: np.ndarray, E_uncond: Optional[np.ndarray], B: int,
           grid_h: int, grid_w: int, steps: int, guidance: float, seed: int,
           blocks: Optional[int] = None, len_cond: Optional[Sequence[int]] = None,
           len_uncond: Optional[Sequence[int]] = None, mu: Optional[float] = None,
           phi: float = 0.0, stop_after: Optional[int] = None,
           trace: Optional[list] = None) -> np.ndarray:
    """Full sampler: seeded noise latent [B, 32, 2h, 2w] -> latent at t = 0.
    The step loop is `sample_euler`; its velocity field is the denoiser `forward` on
    the patchified latent, with the conditional text for cond and the unconditional
    text otherwise (rows are independent, so running the two halves as one batch of
    2B, as the GPU does, computes the same thing).
    READING: unconditional text = zeros of the same shape when E_uncond is None.
    len_cond / len_uncond: valid text lengths per sample (None = all valid).
    mu: shifted time grid (time_grid); phi: norm-rescaled CFG (cfg_rescaled);
    stop_after: return the latent after that many steps of the S-step grid.
    trace: a list that receives (t, cond, tokens, velocity) for every forward."""
    C, p = dims.latent_channels, dims.patch
    z = noise(seed, B * C * p * grid_h * p * grid_w).reshape(B, C, p * grid_h, p * grid_w)
    if guidance != 1.0 and E_uncond is None:
        E_uncond = np.zeros_like(E_cond)
    Nt = E_cond.shape[1]
    lc = None if len_cond is None and len_uncond is None else \
        list(len_cond if len_cond is not None else [Nt] * B)
    lu = None if lc is None else list(len_uncond if len_uncond is not None else [Nt] * B)

    def velocity(x: np.ndarray, t: float, cond: bool) -> np.ndarray:
        X = patchify(x, p)
        v = forward(W, dims, X, grid_h, grid_w, E_cond if cond else E_uncond, [t] * B, blocks,
                    txt_len=lc if cond else lu)
        if trace is not None:
            trace.append((t, cond, X, v))
        return unpatchify(v, grid_h, grid_w, C, p)

    return sample_euler(velocity, z.astype(W.dtype), steps, guidance, mu, phi, stop_after)


# ============================================================ int4 weight-only (4-bit page)
W4_GROUP = 64
W4_SENSITIVE = ("img_in", "txt_in", "proj_out", "time_text_embed", "norm_out")


def _bf16_rne(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 (ties to even), returned as fp32 (finite inputs)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def w4_quantizable(name: str, ndim: int) -> bool:
    """[int4] section 4: the DiT stores its weights in 4 bits with group_size 64 and
    keeps img_in, txt_in, proj_out, time_text_embed and norm_out in bf16.  READING:
    every other Linear weight (all 2-D weights inside the 48 blocks: qkv, to_out,
    to_add_out, w1/w2/w3, img_mod/txt_mod) is quantized; gains and biases are not."""
    return ndim == 2 and name.endswith(".weight") and not name.startswith(W4_SENSITIVE)


def quantize_w4(w: np.ndarray, group: int = W4_GROUP):
    """Affine 4-bit quantization of a [N, K] weight in groups of `group` along K.
    [int4] section 4 gives the bit width and the group size only.  READING: per group
    scale s = (max - min) / 15 and bias b = min, both stored as bf16 (16 bits each:
    with 4-bit codes this is the 2.35 GB the page gives for the whole model), codes
    q = clamp(rint((w - b) / s), 0, 15) computed in fp32 with the stored s and b
    (q = 0 where s = 0).  w is fp32 (or bf16 bits).  Returns (q uint8 [N, K],
    s fp32 [N, K/group], b fp32 [N, K/group]); s and b hold bf16 values."""
    w = upcast(w, np.float32)
    N, K = w.shape
    if K % group:
        raise ValueError(f"K = {K} is not a multiple of the group size {group}")
    g = w.reshape(N, K // group, group)
    mn, mx = g.min(axis=-1), g.max(axis=-1)
    sc = _bf16_rne((mx - mn) / np.float32(15.0))
    bi = _bf16_rne(mn)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint((g - bi[..., None]) / sc[..., None])
    q = np.where(sc[..., None] > 0, q, 0.0)
    q = np.clip(q, 0, 15).astype(np.uint8).reshape(N, K)
    return q, sc, bi


def dequantize_w4(q: np.ndarray, sc: np.ndarray, bi: np.ndarray, group: int = W4_GROUP) -> np.ndarray:
    """w' = s q + b per group, exactly (fp64)."""
    N, K = q.shape
    g = q.reshape(N, K // group, group).astype(F64)
    return (g * sc.astype(F64)[..., None] + bi.astype(F64)[..., None]).reshape(N, K)


def quantize_model_w4(tensors: Mapping[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """The model the 4-bit pipeline evaluates: quantizable weights replaced by their
    dequantized values (fp64), everything else unchanged (bf16 bits)."""
    out = {}
    for name, w in tensors.items():
        out[name] = dequantize_w4(*quantize_w4(w)) if w4_quantizable(name, np.ndim(w)) else w
    return out


def w4_model_bytes(tensors_or_shapes) -> int:
    """Stored bytes of the 4-bit model: 4-bit codes plus a bf16 scale and a bf16 bias
    per group for quantizable weights, 2 bytes per value for the rest."""
    total = 0
    for name, shape in tensors_or_shapes:
        n = int(np.prod(shape))
        total += n // 2 + (n // W4_GROUP) * 4 if w4_quantizable(name, len(shape)) else 2 * n
    return total


# ============================================================ model size
def param_count(dims) -> Dict[str, int]:
    """Parameter counts implied by the tensor shapes this oracle consumes
    (weights and biases of every Linear, norm gains)."""
    D, F, hd = dims.hidden, dims.mlp_hidden, dims.head_dim
    lin = lambda o, i: o * i + o
    stream = lin(3 * D, D) + lin(D, D) + 2 * lin(F, D) + lin(D, F) + lin(6 * D, D) + 2 * hd
    stream_weights_only = 3 * D * D + D * D + 3 * D * F + 6 * D * D
    top = (lin(D, dims.freq_dim) + lin(D, D) + dims.txt_layers * dims.txt_dim
           + lin(D, dims.txt_layers * dims.txt_dim) + lin(D, dims.in_channels)
           + lin(2 * D, D) + lin(dims.in_channels, D))
    return {"stream_weights": stream_weights_only, "stream": stream, "block": 2 * stream,
            "total": dims.num_blocks * 2 * stream + top}
