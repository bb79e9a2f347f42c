/*
 * lens_dit.h — C ABI of the B200 (sm_100a) Lens MMDiT denoiser and its
 * flow-matching Euler sampler.
 *
 * What is computed (sources are web pages, cited by title and section):
 *   - "Lens" blog (zjwfufu.github.io), "Overview": 48 dual-stream MMDiT blocks,
 *     hidden 1536, 24 heads, gated MLP 1536x4096, AdaLN 1536x9216 per stream.
 *   - "深入 Lens-Turbo-3.8B-bf16 内核" (MLX bf16 port article), sections
 *     "核心规格一览", "双流注意力机制", "自适应调制与 RMSNorm", "3D RoPE",
 *     "多层级文本特征融合", "Patchify 补丁化与输出投影", "guidance 1.0": tensor
 *     names, RoPE axes [8, 28, 28], 2x2 patches of a 32-channel latent (128-d
 *     tokens), QK RMSNorm, four GPT-OSS feature layers of 2880.
 *   - "Lens: 重新思考基础文生图模型的训练效率" (paper summary), "Flow Matching 训练目标":
 *     x_t = (1-t) x0 + t x1, v = x1 - x0; "方法步骤详情": 20 steps with CFG 5.0,
 *     Turbo 4 steps without CFG.
 *   - "从提示词到成图：Lens-3.8B-4bit完整管线解析", section 6: pipeline(prompt,
 *     height, width, num_inference_steps, seed); this ABI starts after the text
 *     encoder (features in) and stops before the VAE (latent out).
 *
 * Conventions for every entry point:
 *   - Tensor pointers marked "dev" are caller-owned device memory on the current
 *     device; "host" pointers are read during the call only.
 *   - All GPU work is enqueued on `stream` (a cudaStream_t, NULL = legacy default
 *     stream).  Argument errors return synchronously and enqueue nothing.  Errors
 *     from kernels (including the device watchdog on internal waits) surface
 *     through lens_dit_sync() or the next call.
 *   - No entry point falls back to the CPU.  A handle is used by one stream at a
 *     time.  Forward and sample calls allocate nothing: the handle's workspace is
 *     sized at create time from the config's max_* fields.
 *   - bf16 tensors are raw IEEE bfloat16 bit patterns (uint16_t here).
 */
#ifndef LENS_DIT_H
#define LENS_DIT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LENS_API __attribute__((visibility("default")))
#else
#define LENS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lens_status {
  LENS_OK = 0,
  LENS_ERR_INVALID_ARG = 1,   /* null pointer, unknown tensor name, bad scalar */
  LENS_ERR_SHAPE = 2,         /* shape out of range or inconsistent with the config */
  LENS_ERR_OOM = 3,           /* device allocation failed at create */
  LENS_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  LENS_ERR_TIMEOUT = 5,       /* a kernel's bounded internal wait expired */
  LENS_ERR_UNSUPPORTED = 6    /* config value this build does not implement */
} lens_status;

/* Model and capacity configuration.  Model fields must keep the Lens values
 * (lens_dit_default_config); num_blocks may be 1..48 (fewer blocks run the first
 * num_blocks of the tensor list, for tests).  max_* size the workspace:
 * max_batch counts forward rows, i.e. 2 x samples when CFG is on. */
typedef struct lens_dit_config {
  int num_blocks;        /* 48 */
  int hidden;            /* 1536 */
  int heads;             /* 24 */
  int head_dim;          /* 64 */
  int mlp_hidden;        /* 4096 */
  int in_channels;       /* 128 = 2*2*32 */
  int latent_channels;   /* 32 */
  int patch;             /* 2 */
  int txt_layers;        /* 4 */
  int txt_dim;           /* 2880 */
  int rope_axes[3];      /* 8, 28, 28 */
  float rope_theta;      /* 10000 */
  float eps;             /* 1e-6, all RMSNorms */
  int freq_dim;          /* 256, sinusoidal timestep features */
  int max_batch;         /* forward rows (cond + uncond) */
  int max_img_tokens;    /* grid_h * grid_w */
  int max_txt_tokens;
  int max_timesteps;     /* distinct timesteps whose modulation is kept at once */
  int weight_bits;       /* 16: bf16 weights.  4: int4 weight-only ("从提示词到成图：
                            Lens-3.8B-4bit完整管线解析", section 4): every Linear inside the
                            blocks (qkv, to_out / to_add_out, w1 / w2 / w3, img_mod /
                            txt_mod) quantized at create (lens_op_quantize_w4's format),
                            img_in, txt_in, proj_out, the timestep MLP and norm_out kept
                            in bf16; about 2.35 GB of weights instead of 8.2 GB */
} lens_dit_config;

/* One named weight tensor, host bf16, row-major [out, in] for Linear weights.
 * Names (MLX bf16 port article, "双流注意力机制"/"自适应调制"/"多层级文本特征融合"):
 *   time_text_embed.timestep_embedder.linear_{1,2}.{weight,bias}
 *   txt_norm.{0..3}.weight, txt_in.{weight,bias}, img_in.{weight,bias}
 *   transformer_blocks.{i}.{img_mod,txt_mod}.{weight,bias}
 *   transformer_blocks.{i}.attn.{img_qkv,txt_qkv,to_out,to_add_out}.{weight,bias}
 *   transformer_blocks.{i}.attn.{norm_q,norm_k,norm_added_q,norm_added_k}.weight
 *   transformer_blocks.{i}.{img_mlp,txt_mlp}.{w1,w2,w3}.{weight,bias}
 *   norm_out.linear.{weight,bias}, proj_out.{weight,bias}
 * Every *.weight of a Linear is required; a missing bias is zero. */
typedef struct lens_weight {
  const char* name;
  const uint16_t* data;   /* host bf16 */
  int ndim;
  int64_t shape[4];
} lens_weight;

typedef struct lens_dit lens_dit;

/* Fill `cfg` with the Lens values and capacities for one 1024^2 CFG sample. */
LENS_API lens_status lens_dit_default_config(lens_dit_config* cfg);

/* Validate cfg, copy and pack the weights to the device (fused QKV as given,
 * w1|w3 interleaved per 32 columns, all AdaLN projections and norm_out
 * concatenated), and allocate the workspace.  The caller may free `w` on return.
 * Synchronous.  Errors: INVALID_ARG (null, duplicate or unknown name, missing
 * weight), SHAPE (a tensor shape differs from cfg), UNSUPPORTED (model fields
 * other than Lens's), OOM, CUDA. */
LENS_API lens_status lens_dit_create(const lens_dit_config* cfg, const lens_weight* w, int n_w,
                            void* stream, lens_dit** out);

LENS_API void lens_dit_destroy(lens_dit* h);

/* One denoiser forward: velocity of B rows at per-row timesteps.
 *   img_tokens  dev fp32 [B, grid_h*grid_w, 128]  patchified latent tokens
 *   txt         dev bf16 [B, n_txt, 4, 2880]      encoder features of 4 layers
 *   t           host fp32 [B]                     timesteps in [0, 1]
 *   v_out       dev fp32 [B, grid_h*grid_w, 128]  velocity tokens
 * Errors: INVALID_ARG (null), SHAPE (B > max_batch, B > max_timesteps, grid or
 * n_txt beyond the capacities, n_txt + grid_h*grid_w < 1). */
LENS_API lens_status lens_dit_forward(lens_dit* h, const float* img_tokens, int B, int grid_h, int grid_w,
                             const uint16_t* txt, int n_txt, const float* t, float* v_out,
                             void* stream);

/* lens_dit_forward with a text padding mask ("Lens" blog, "Exploring Text Encoder":
 * zero-padded text tokens are masked, so the DiT never sees them): text keys at and
 * past txt_len[b] are not attended by any query of batch row b.
 *   txt_len  host int [B], 0 <= txt_len[b] <= n_txt, or NULL (no padding).
 * B <= 64 when txt_len is given.  Errors as lens_dit_forward, plus SHAPE for a
 * length out of range. */
LENS_API lens_status lens_dit_forward_masked(lens_dit* h, const float* img_tokens, int B, int grid_h, int grid_w,
                                             const uint16_t* txt, int n_txt, const int* txt_len, const float* t,
                                             float* v_out, void* stream);

/* Flow-matching Euler sampler ("Flow Matching 训练目标": x_t = (1-t) x0 + t x1,
 * v = x1 - x0; integrate t from 1 to 0 with `steps` uniform steps,
 * x <- x - v / steps, model input t_k = 1 - k/steps).  With guidance != 1 the
 * conditional and unconditional rows run as one batch of 2B and combine as
 * uncond + guidance * (cond - uncond).
 *   txt_cond    dev bf16 [B, n_txt, 4, 2880]
 *   txt_uncond  dev bf16 [B, n_txt, 4, 2880], or NULL for zeros (ignored when
 *               guidance == 1)
 *   height_px, width_px: multiples of 16 (8x VAE, 2x2 patch)
 *   seed        initial noise N(0,1): Box-Muller over SplitMix64 words, latent
 *               element n uses words SM(seed ^ SM(2n)), SM(seed ^ SM(2n+1))
 *   latent_out  dev fp32 [B, 32, height_px/8, width_px/8]
 * Errors: INVALID_ARG (null, steps < 1, non-finite guidance), SHAPE (sizes not
 * multiples of 16, beyond capacities, forward rows > max_batch). */
LENS_API lens_status lens_sample_euler(lens_dit* h, const uint16_t* txt_cond, const uint16_t* txt_uncond,
                              int B, int n_txt, int height_px, int width_px, int steps,
                              float guidance, uint64_t seed, float* latent_out, void* stream);

/* lens_sample_euler with text padding masks: len_cond / len_uncond host int [B]
 * (valid text lengths of the conditional / unconditional features), either may be
 * NULL for "all n_txt valid".  2B <= 64 when a length array is given.
 * On a stream created by the caller, a call is captured as a CUDA graph and
 * replayed while every argument stays the same (this holds for lens_sample_euler
 * too); the legacy default stream runs the kernels directly. */
LENS_API lens_status lens_sample_euler_masked(lens_dit* h, const uint16_t* txt_cond, const int* len_cond,
                                              const uint16_t* txt_uncond, const int* len_uncond, int B, int n_txt,
                                              int height_px, int width_px, int steps, float guidance, uint64_t seed,
                                              float* latent_out, void* stream);

/* Sampler variants (plain value struct, filled by lens_sampler_default_options).
 *   guidance     CFG scale s; 1 evaluates the conditional model only.
 *   cfg_rescale  phi in [0, 1], used when guidance != 1: the guided velocity
 *                p = u + s (c - u) becomes (phi |c| / |p| + 1 - phi) p, both L2
 *                norms over one sample's whole velocity; |p| = 0 leaves p as is.
 *                Blog "Lens", section "Exploring Image Editing": Lens runs a
 *                "norm-rescaled CFG" (only u + s (c - u) is printed; this rescale
 *                toward the conditional norm is the reading taken).  0 = plain CFG.
 *   time_shift   nonzero: the uniform grid u_k = 1 - k/S is mapped through
 *                t_k = e^mu u_k / (e^mu u_k + 1 - u_k).  Summary page "Lens:
 *                重新思考基础文生图模型的训练效率", section "Flow Matching 训练目标":
 *                the timestep schedule at each resolution follows a mu(n) linear
 *                interpolation (section "方法步骤详情": mu = 1.06 at 512^2); the
 *                formula is not printed, the published resolution-dependent shift
 *                is taken.  Step k feeds the model t_k and moves by t_k - t_{k+1}.
 *   shift_mu     mu of the shift, |mu| <= 50 (see lens_shift_mu). */
typedef struct {
  float guidance;
  float cfg_rescale;
  int time_shift;
  float shift_mu;
} lens_sampler_options;

/* Defaults: guidance 1, cfg_rescale 0, time_shift 0, shift_mu 0 (the plain sampler).
 * Errors: INVALID_ARG for NULL. */
LENS_API lens_status lens_sampler_default_options(lens_sampler_options* opt);

/* mu(n) linear in the image token count n through (n1, mu1) and (n2, mu2).  The
 * pages give one point (512^2 = 1024 tokens: mu = 1.06); the second anchor is the
 * caller's.  Host only; returns NaN when n1 == n2. */
LENS_API double lens_shift_mu(int n_img_tokens, int n1, double mu1, int n2, double mu2);

/* The sampler's time grid t_0 .. t_steps (host double [steps + 1], caller-owned),
 * uniform or shifted as in lens_sampler_options.  Host only.
 * Errors: INVALID_ARG (NULL, steps < 1, non-finite mu or |mu| > 50). */
LENS_API lens_status lens_time_grid(int steps, int time_shift, double mu, double* t_out);

/* lens_sample_euler_masked with the variants of `opt` (host, not kept).  Arguments
 * and graph replay as lens_sample_euler_masked; the options are part of what must
 * stay the same for a replay.
 * Errors: as lens_sample_euler_masked, plus INVALID_ARG for a NULL opt,
 * cfg_rescale outside [0, 1] or |shift_mu| > 50 (or not finite). */
LENS_API lens_status lens_sample_euler_ex(lens_dit* h, const uint16_t* txt_cond, const int* len_cond,
                                          const uint16_t* txt_uncond, const int* len_uncond, int B, int n_txt,
                                          int height_px, int width_px, int steps, const lens_sampler_options* opt,
                                          uint64_t seed, float* latent_out, void* stream);

/* Step-wise sampler: the pieces of lens_sample_euler_ex as separate calls, for a
 * caller that evaluates the conditional and the unconditional half of CFG in two
 * processes (one per GPU) and exchanges the two velocities between steps.  The
 * velocity of one batch row does not depend on the other rows, so two handles
 * running the halves and exchanging velocities reproduce lens_sample_euler_ex.
 * Summary page "Lens: 重新思考基础文生图模型的训练效率", "方法步骤详情" (20 steps,
 * CFG 5.0) and blog "Lens", "Exploring Image Editing" (uncond + s (cond - uncond)):
 * each step needs both halves once.
 *
 * lens_sampler_prepare: seeded noise x (as lens_sample_euler), the text input of
 *   `txt` (dev bf16 [B, n_txt, 4, 2880]; NULL = zeros, the unconditional text of the
 *   plain sampler) with optional lengths txt_len (host int [B], NULL = all valid),
 *   and the modulation of every step (steps <= max_timesteps).  The state lives in
 *   the handle until the next call that is not one of these four.
 * lens_sampler_velocity: the velocity of this handle's rows at step k (0-based),
 *   v_out dev fp32 [B, (height/16)*(width/16), 128], 16-byte aligned.
 * lens_sampler_update: x -= dt_k v with v = v_cond when opt.guidance == 1, else the
 *   plain or norm-rescaled combination of v_cond and v_uncond (both dev fp32, same
 *   layout as v_out; v_uncond ignored when guidance == 1).
 * lens_sampler_finish: latent_out dev fp32 [B, 32, height/8, width/8] from x.
 * Errors: INVALID_ARG (NULL, bad options as lens_sample_euler_ex, steps < 1, a step
 * call without a prepared state, unaligned v_out), SHAPE (sizes as
 * lens_sample_euler, steps > max_timesteps, k outside [0, steps)). */
LENS_API lens_status lens_sampler_prepare(lens_dit* h, const uint16_t* txt, const int* txt_len, int B, int n_txt,
                                          int height_px, int width_px, int steps, const lens_sampler_options* opt,
                                          uint64_t seed, void* stream);
LENS_API lens_status lens_sampler_velocity(lens_dit* h, int k, float* v_out, void* stream);
LENS_API lens_status lens_sampler_update(lens_dit* h, int k, const float* v_cond, const float* v_uncond,
                                         void* stream);
LENS_API lens_status lens_sampler_finish(lens_dit* h, float* latent_out, void* stream);

/* Test hook: run blocks [first, last) in place on a residual stream.
 *   h_img dev fp32 [B, grid_h*grid_w, 1536], h_txt dev fp32 [B, n_txt, 1536]
 *   t host fp32 [B].  Errors as lens_dit_forward, plus SHAPE for a bad range. */
LENS_API lens_status lens_dit_debug_blocks(lens_dit* h, int first, int last, float* h_img, float* h_txt,
                                  int B, int grid_h, int grid_w, int n_txt, const float* t,
                                  void* stream);

/* Test hook for the failure path: raise the handle's device abort flag on `stream`,
 * as an expired wait would.  Kernels launched after it leave at their first wait
 * that does not complete at once, after draining their own copies and MMAs; the
 * next lens_dit_sync reports LENS_ERR_TIMEOUT and clears the flag, and calls after
 * that run normally.  Errors: INVALID_ARG (NULL handle), CUDA. */
LENS_API lens_status lens_dit_debug_raise_abort(lens_dit* h, void* stream);

/* Wait for the handle's work on `stream` and report kernel-side errors
 * (CUDA errors, TIMEOUT from the device watchdog).  Clears the watchdog flag. */
LENS_API lens_status lens_dit_sync(lens_dit* h, void* stream);

LENS_API const char* lens_status_string(lens_status s);

/* ---------------------------------------------------------------------------
 * Single-operation entry points (the same kernels the denoiser runs), for
 * parity tests of each step.  Handle-free unless stated; no allocation.
 * ------------------------------------------------------------------------- */

/* Seeded N(0,1) latent noise straight into patch tokens (noise definition as in
 * lens_sample_euler; patchify: token (i, j) of row-major order, feature
 * c*4 + 2*r + s = latent[c, 2i+r, 2j+s]).  tokens dev fp32 [B, gh*gw, 128]. */
LENS_API lens_status lens_op_noise_tokens(uint64_t seed, int B, int grid_h, int grid_w, float* tokens,
                                 void* stream);

/* Patchify a latent dev fp32 [B, 32, 2gh, 2gw] into tokens dev fp32
 * [B, gh*gw, 128] and back (MLX port article, "Patchify 补丁化与输出投影").
 * Bit-exact permutations. */
LENS_API lens_status lens_op_patchify(const float* latent, int B, int grid_h, int grid_w, float* tokens,
                             void* stream);
LENS_API lens_status lens_op_unpatchify(const float* tokens, int B, int grid_h, int grid_w, float* latent,
                               void* stream);

/* 3D RoPE table (MLX port article, "3D RoPE"): ids (0,0,0) for the n_txt text
 * tokens, then (0, i, j) for the image grid; pair m of axis a turns by
 * pos_a * 10000^(-2m/d_a), axes [8, 28, 28] own consecutive head-dim segments.
 * cos_sin dev fp32 [(n_txt + gh*gw), 32, 2] as (cos, sin) pairs. */
LENS_API lens_status lens_op_rope_table(int grid_h, int grid_w, int n_txt, float* cos_sin, void* stream);

/* y = (1 + scale[b]) * x / sqrt(mean(x^2) + eps) + shift[b] per row, rows of
 * sample b = row / rows_per_batch ("自适应调制与 RMSNorm").
 *   x dev fp32 [M, 1536]; shift, scale dev fp32 with row stride `mod_stride`
 *   per sample; y dev bf16 [M, 1536]. */
LENS_API lens_status lens_op_rmsnorm_modulate(const float* x, int M, int rows_per_batch,
                                     const float* shift, const float* scale, int64_t mod_stride,
                                     float eps, uint16_t* y, void* stream);

/* int4 weight-only ("从提示词到成图：Lens-3.8B-4bit完整管线解析", section 4: 4-bit
 * weights, group size 64).  lens_op_quantize_w4 quantizes a bf16 weight w [rows, k]
 * (dev, k a multiple of 64) per group of 64 along k: scale = bf16((max - min) / 15),
 * bias = bf16(min), code = clamp(rint((w - bias) / scale), 0, 15) in fp32 (0 where
 * scale = 0); w ~ scale * code + bias.  Caller-owned outputs:
 *   codes  dev uint8 [rows, k / 2], 16-byte aligned: 32-bit word j of a row holds
 *          the codes of k in [8j, 8j + 8); the code of k = 8j + 2i sits in bits
 *          [4i, 4i + 4), that of k = 8j + 2i + 1 in bits [16 + 4i, 20 + 4i)
 *   scales dev uint32 [k / 64, rows]: group g of row r at [g][r], bf16 scale in the
 *          low half, bf16 bias in the high half.
 * lens_op_gemm_w4: C[M,N] = A[M,K] W[N,K]^T (+ bias) with W given as codes/scales
 * of that layout (rows = N, k = K), widened to bf16 in shared memory before the
 * tcgen05 MMA; A dev bf16 [M, K], bias dev fp32 [N] or NULL, C dev fp32 [M, N].
 * N a multiple of 128, K of 64.  Errors: INVALID_ARG (NULL, misaligned), SHAPE. */
LENS_API lens_status lens_op_quantize_w4(const uint16_t* w, int64_t rows, int64_t k, uint8_t* codes,
                                         uint32_t* scales, void* stream);
LENS_API lens_status lens_op_gemm_w4(const uint16_t* A, const uint8_t* codes, const uint32_t* scales,
                                     const float* bias, float* C, int M, int N, int K, void* stream);

/* Plain bf16 GEMM on the tcgen05 tensor cores: C[M,N] = A[M,K] B[N,K]^T (+ bias),
 * fp32 out.  A, B dev bf16 K-contiguous; bias dev fp32 [N] or NULL; C dev fp32.
 * K and N multiples of 64 and 16; A, B, C 16-byte aligned rows. */
LENS_API lens_status lens_op_gemm_bf16(const uint16_t* A, const uint16_t* B, const float* bias, float* C,
                              int M, int N, int K, void* stream);

/* Joint attention over [text; image] tokens ("双流注意力机制"): per head
 * softmax(q k^T / 8) v, no mask.  q, k, v dev bf16 [B, 24, N, 64] with
 * N = n_txt + n_img, text rows first; out_txt dev bf16 [B, n_txt, 1536] and
 * out_img dev bf16 [B, n_img, 1536] (column = head*64 + d). */
LENS_API lens_status lens_op_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B,
                              int n_txt, int n_img, uint16_t* out_txt, uint16_t* out_img,
                              void* stream);

/* lens_op_attention with text padding: text keys at and past txt_len[b] (host int
 * [B], B <= 64; NULL = none) are not attended.  A batch row left with no key at
 * all (n_img = 0 and txt_len[b] = 0) has no defined softmax: LENS_ERR_SHAPE. */
LENS_API lens_status lens_op_attention_masked(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B,
                                              int n_txt, int n_img, const int* txt_len, uint16_t* out_txt,
                                              uint16_t* out_img, void* stream);

/* Euler step with optional CFG on tokens: x -= dt * (vu + g (vc - vu)), or
 * x -= dt * vc when v_uncond is NULL.  x, v_cond, v_uncond dev fp32 [n]. */
LENS_API lens_status lens_op_euler_cfg(float* x, const float* v_cond, const float* v_uncond, int64_t n,
                              float dt, float guidance, void* stream);

/* Euler step with norm-rescaled CFG (see lens_sampler_options.cfg_rescale) on B
 * samples of per_sample values each: x -= dt (phi |c| / |p| + 1 - phi) p with
 * p = u + guidance (c - u), norms per sample.  x, v_cond, v_uncond dev fp32
 * [B, per_sample].  Uses the handle's workspace, so calls on one handle must not
 * overlap.  Errors: INVALID_ARG (NULL, non-finite dt or guidance, phi outside
 * [0, 1]), SHAPE (B < 1, B > max_batch, per_sample < 1). */
LENS_API lens_status lens_dit_op_euler_cfg_rescaled(lens_dit* h, float* x, const float* v_cond,
                                                    const float* v_uncond, int B, int64_t per_sample, float dt,
                                                    float guidance, float phi, void* stream);

/* Handle ops: the timestep embedding temb [T, 1536] (dev fp32) of host t[T], and
 * the AdaLN modulation of every block plus norm_out for those timesteps,
 * mod dev fp32 [T, 48*2*9216 + 3072] laid out block-major, then img/txt, then
 * (shift1, scale1, gate1, shift2, scale2, gate2) x 1536; norm_out last as
 * (scale, shift).  T <= max_timesteps. */
LENS_API lens_status lens_dit_op_timestep(lens_dit* h, const float* t, int T, float* temb, float* mod,
                                 void* stream);

/* Handle op: text input head, txt dev bf16 [B, n_txt, 4, 2880] -> c dev fp32
 * [B, n_txt, 1536] (txt_norm.0..3, concatenation, txt_in). */
LENS_API lens_status lens_dit_op_text_input(lens_dit* h, const uint16_t* txt, int B, int n_txt, float* c,
                                   void* stream);

/* Timestep embedding without any allocation.  The paper has no counterpart: this
 * entry point exists for callers that cannot call cudaMalloc, for instance a plugin
 * in a host application that owns and budgets all device memory, or a
 * latency-critical loop that cannot afford cudaMalloc's implicit synchronisation.
 * It computes the same temb as lens_dit_op_timestep (sinusoid -> linear_1 -> SiLU
 * -> linear_2) from caller-supplied weights:
 *   t     host fp32 [T], 1 <= T <= 64 (larger T returns LENS_ERR_SHAPE)
 *   w1    dev bf16 [1536, 256],  b1 dev fp32 [1536] or NULL
 *   w2    dev bf16 [1536, 1536], b2 dev fp32 [1536] or NULL
 *   temb  dev fp32 [T, 1536]
 * w1 and w2 must be 16-byte aligned (LENS_ERR_INVALID_ARG otherwise).
 * The intermediates live in one fixed 448 KiB device array inside the library.
 * The first call on each device looks up that array's device address with the
 * device current; under lazy module loading (the CUDA default) that lookup is
 * also what loads the library's kernels on the device and reserves the array,
 * an implicit driver allocation that may synchronise and may fail (returned as
 * LENS_ERR_OOM).  So make the first call on each device during set-up, before
 * any stream capture; later calls allocate nothing, and the array stays reserved
 * until the process exits.  All calls share the array and it keeps the last
 * call's contents (every value is written before it is read), so calls whose GPU
 * work overlaps (e.g. on two streams at once) race.
 * Calls no cudaMalloc, cudaFree or other allocating routine. */
LENS_API lens_status lens_op_timestep_embed_noalloc(const float* t, int T, const uint16_t* w1, const float* b1,
                                                    const uint16_t* w2, const float* b2, float* temb,
                                                    void* stream);

/* ---------------------------------------------------------------------------
 * Measurement hooks.
 * ------------------------------------------------------------------------- */
typedef enum lens_kernel {
  LENS_KERNEL_NONE = 0,
  LENS_KERNEL_ATTENTION = 1,     /* joint attention */
  LENS_KERNEL_GEMM_QKV = 2,      /* QKV GEMM + QK-norm + RoPE epilogue */
  LENS_KERNEL_GEMM_OUT = 3,      /* to_out / to_add_out GEMM + gated residual */
  LENS_KERNEL_GEMM_W13 = 4,      /* w1|w3 GEMM + SwiGLU epilogue */
  LENS_KERNEL_GEMM_W2 = 5,       /* w2 GEMM + gated residual */
  LENS_KERNEL_RMSNORM_MOD = 6,   /* RMSNorm + AdaLN modulation */
  LENS_KERNEL_GEMM_MOD = 7       /* all-block AdaLN modulation GEMM */
} lens_kernel;

/* Time every launch of one kernel family with a CUDA event pair recorded on the
 * launching stream (up to `capacity` launches; later ones are not timed).
 * kernel = LENS_KERNEL_NONE switches timing off.  Resets the record.  Creating
 * the events is the only allocation; the call is synchronous. */
LENS_API lens_status lens_dit_profile_kernel(lens_dit* h, lens_kernel kernel, int capacity);

/* Synchronise the recorded events and report the timed launches and their summed
 * device time in milliseconds. */
LENS_API lens_status lens_dit_profile_read(lens_dit* h, int* launches, double* total_ms);

/* Kernels this handle has launched since create (memcpy/memset not counted). */
LENS_API int64_t lens_dit_launch_count(lens_dit* h);

/* Number of streaming multiprocessors the kernels size their grids by. */
LENS_API int lens_device_sm_count(void);

#ifdef __cplusplus
}
#endif
#endif /* LENS_DIT_H */
