// C ABI of the Lens MMDiT denoiser and flow-matching Euler sampler (include/lens_dit.h).
//
// The handle owns the packed weights (one device arena) and a workspace sized at
// create time; forward / sample never allocate.  Every step of the path runs in
// this library's kernels: tcgen05 GEMMs with fused epilogues, the joint-attention
// kernel and the memory-bound kernels in elementwise.cu.
#include <math.h>
#include <string.h>

#include <string>
#include <unordered_map>
#include <vector>

#include "gemm.h"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "lens_dit.h"
#include "smem_attr.h"

using namespace lens;

namespace {

// the largest block weight staged at create with weight_bits = 4 (one stream's AdaLN)
constexpr size_t kStageElems = (size_t)kModPerStream * kHidden;

// 4-bit block GEMMs on 256-row tiles (one widened B tile feeds two 128-row MMAs):
// 128 wide for w1|w3 and QKV, 96 wide for the 1536-wide to_out and w2 (272 tiles)
constexpr int kBnW13W4 = 128, kBnQkvW4 = 128, kBnResW4 = 96;

constexpr int kBnQkv = 256, kBnOut = 192, kBnW13 = 256, kBnW2 = 192, kBnImgIn = 256, kBnTxtIn = 128,
              kBnProj = 128;

// a 4-bit weight (weight_bits = 4): codes and scales in lens_op_quantize_w4's layout
struct QW {
  uint8_t* codes = nullptr;
  uint32_t* scales = nullptr;
  CUtensorMap tq, ts;
};

struct StreamW {
  __nv_bfloat16 *qkv, *out, *w13, *w2;   // bf16 weights (null with weight_bits = 4)
  QW q_qkv, q_out, q_w13, q_w2;          // 4-bit weights (weight_bits = 4)
  float *b_qkv, *b_out, *b_w13, *b_w2, *gq, *gk;
  CUtensorMap t_qkv, t_out, t_w13, t_w2;
  // the same weights with B boxes for 2- and 4-way column slices of a tile (the tail
  // round of a CTA-pair launch; see launch_gemm_pair)
  CUtensorMap n_qkv[2], n_out[2], n_w13[2], n_w2[2];
  // a bias that is absent or all zero is not added at all
  bool has_b_qkv = false, has_b_out = false, has_b_w13 = false, has_b_w2 = false;
};
struct BlockW {
  StreamW s[2];   // 0 = image stream, 1 = text stream
};

// Bump allocator used twice: once to size (base 0), once to hand out pointers.
struct Bump {
  uintptr_t base = 0;
  size_t off = 0;
  template <class T>
  T* take(size_t n) {
    off = (off + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base + off);
    off += n * sizeof(T);
    return p;
  }
};

inline bool any_nonzero_bf16(const uint16_t* p, size_t n) {
  if (!p) return false;
  for (size_t i = 0; i < n; ++i)
    if (p[i] & 0x7FFF) return true;
  return false;
}

inline float bf16_to_f32(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

}  // namespace

struct lens_dit {
  lens_dit_config cfg{};
  int device = 0, sms = 148;
  int64_t modw = 0;   // modulation floats per timestep
  // weights
  void* warena = nullptr;
  __nv_bfloat16 *w_t1, *w_t2, *w_txt_in, *w_img_in, *w_proj, *w_mod;
  float *b_t1, *b_t2, *b_txt_in, *b_img_in, *b_proj, *b_mod, *g_txt;
  bool has_b_txt_in = false, has_b_img_in = false, has_b_proj = false;
  CUtensorMap t_txt_in, t_img_in, t_proj, t_mod;
  // weight_bits = 4: block AdaLN rows as 4-bit, norm_out rows in bf16 (w_no)
  bool w4 = false;
  QW q_mod;
  __nv_bfloat16* w_no = nullptr;
  CUtensorMap t_no;
  __nv_bfloat16* wstage = nullptr;      // create-time staging of one bf16 matrix
  std::vector<BlockW> blk;
  // workspace
  void* ws = nullptr;
  __nv_bfloat16 *xin, *a_img, *a_txt, *q, *k, *v, *o_img, *o_txt, *u_img, *u_txt, *txt_cat, *stemb;
  float *h_img, *h_txt, *h_txt0, *vtok, *xtok, *tfeat, *hid, *temb, *mod;
  float2* rope;
  double* cfgpart;     // per-sample partial norms of the norm-rescaled CFG
  int* err;
  // the last sampler call, captured as a CUDA graph and replayed for identical calls
  struct SampleGraph {
    bool valid = false;
    const void *txt_cond, *txt_uncond, *latent_out;
    cudaStream_t stream;
    int B, n_txt, height_px, width_px, steps;
    float guidance, cfg_rescale, shift_mu;
    int time_shift;
    uint64_t seed;
    int prof_kind;
    bool masked;
    TextLengths lens;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    int64_t launches = 0;        // kernels one replay runs
  } sg;
  // step-wise sampler (lens_sampler_prepare .. lens_sampler_finish); cleared by every
  // call that reuses the modulation, text or token buffers
  struct StepSampler {
    bool ready = false;
    int B = 0, gh = 0, gw = 0, n_txt = 0, steps = 0;
    lens_sampler_options opt{};
    bool masked = false;
    TextLengths tl{};
    double grid[kMaxTimesteps + 1];
  } ss;
  // measurement
  int64_t launches = 0;
  int prof_kind = 0, prof_cap = 0, prof_n = 0;
  std::vector<cudaEvent_t> prof_ev;
};

static void drop_sample_graph(lens_dit* h);

// ============================================================ helpers
static const char* kStatusStr[] = {"ok", "invalid argument", "shape out of range", "out of device memory",
                                   "CUDA error", "device wait timed out", "unsupported configuration"};

#define LENS_CUDA(x)                              \
  do {                                            \
    cudaError_t e_ = (x);                         \
    if (e_ != cudaSuccess) return LENS_ERR_CUDA;  \
  } while (0)

// Launch accounting: count every kernel, and time the selected family.
// One event record of the profiling hooks.  While the stream is being captured the
// record must be an external one to become an event node of the graph; outside a
// capture it is a plain record.  A failed record is cleared so that it is not
// reported as the next launch's error.
static bool prof_record(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const cudaError_t e = cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal)
                                                            : cudaEventRecord(ev, st);
  if (e != cudaSuccess) cudaGetLastError();
  return e == cudaSuccess;
}

struct KScope {
  lens_dit* h;
  cudaStream_t st;
  bool on;
  KScope(lens_dit* h_, int kind, cudaStream_t st_) : h(h_), st(st_), on(false) {
    ++h->launches;
    if (h->prof_kind == kind && h->prof_n < h->prof_cap) on = prof_record(h->prof_ev[2 * h->prof_n], st);
    // a timed launch sits between two event records: no programmatic overlap with it
    pdl_suspended() = on;
  }
  ~KScope() {
    pdl_suspended() = false;
    if (on && prof_record(h->prof_ev[2 * h->prof_n + 1], st)) ++h->prof_n;
  }
};

#define LENS_LAUNCH(h, kind, st, x) \
  do {                              \
    KScope ks_(h, kind, st);        \
    LENS_CUDA(x);                   \
  } while (0)

static int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

static GemmArgs make_args(int* err) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.err = err;
  return a;
}

static GemmProblem base_problem(int M, int N, int K) {
  GemmProblem p;
  memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.K = K;
  p.rows_per_batch = 1;
  p.heads = kHeads;
  return p;
}

// ============================================================ module-level error flag
// Used by the handle-free op entry points.
__device__ int g_op_err;
static int* op_err_ptr() {
  int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_op_err) != cudaSuccess) return nullptr;
  return p;
}

// ============================================================ weight loading
namespace {
struct Loader {
  std::unordered_map<std::string, const lens_weight*> by_name;
  lens_status st = LENS_OK;

  const uint16_t* get(const std::string& name, std::initializer_list<int64_t> shape, bool required) {
    auto it = by_name.find(name);
    if (it == by_name.end()) {
      if (required && st == LENS_OK) st = LENS_ERR_INVALID_ARG;
      return nullptr;
    }
    const lens_weight* w = it->second;
    if (!w->data) {
      if (st == LENS_OK) st = LENS_ERR_INVALID_ARG;
      return nullptr;
    }
    if (w->ndim != (int)shape.size()) {
      if (st == LENS_OK) st = LENS_ERR_SHAPE;
      return nullptr;
    }
    int i = 0;
    for (int64_t s : shape)
      if (w->shape[i++] != s) {
        if (st == LENS_OK) st = LENS_ERR_SHAPE;
        return nullptr;
      }
    return w->data;
  }
};

// bf16 host -> device bf16 (straight copy)
lens_status put_bf16(__nv_bfloat16* dst, const uint16_t* src, size_t n) {
  if (cudaMemcpy(dst, src, n * 2, cudaMemcpyHostToDevice) != cudaSuccess) return LENS_ERR_CUDA;
  return LENS_OK;
}
// bf16 host (or zeros / a constant when src is null) -> device fp32
lens_status put_f32(float* dst, const uint16_t* src, size_t n, float fill, std::vector<float>& stage) {
  stage.resize(n);
  for (size_t i = 0; i < n; ++i) stage[i] = src ? bf16_to_f32(src[i]) : fill;
  if (cudaMemcpy(dst, stage.data(), n * 4, cudaMemcpyHostToDevice) != cudaSuccess) return LENS_ERR_CUDA;
  return LENS_OK;
}
}  // namespace

static void layout_weights(lens_dit* h, Bump& b) {
  const int nb = h->cfg.num_blocks;
  h->w_t1 = b.take<__nv_bfloat16>((size_t)kHidden * kFreqDim);
  h->w_t2 = b.take<__nv_bfloat16>((size_t)kHidden * kHidden);
  h->w_txt_in = b.take<__nv_bfloat16>((size_t)kHidden * kTxtLayers * kTxtDim);
  h->w_img_in = b.take<__nv_bfloat16>((size_t)kHidden * 2 * kInCh);
  h->w_proj = b.take<__nv_bfloat16>((size_t)kInCh * kHidden);
  if (h->w4) {
    const size_t mrows = (size_t)nb * kModPerBlock;
    h->w_mod = nullptr;
    h->w_no = b.take<__nv_bfloat16>((size_t)2 * kHidden * kHidden);
    h->q_mod.codes = b.take<uint8_t>(mrows * kHidden / 2);
    h->q_mod.scales = b.take<uint32_t>(mrows * (kHidden / 64));
  } else {
    h->w_mod = b.take<__nv_bfloat16>((size_t)h->modw * kHidden);
  }
  h->b_t1 = b.take<float>(kHidden);
  h->b_t2 = b.take<float>(kHidden);
  h->b_txt_in = b.take<float>(kHidden);
  h->b_img_in = b.take<float>(kHidden);
  h->b_proj = b.take<float>(kInCh);
  h->b_mod = b.take<float>(h->modw);
  h->g_txt = b.take<float>(kTxtLayers * kTxtDim);
  h->blk.resize(nb);
  for (int i = 0; i < nb; ++i)
    for (int s = 0; s < 2; ++s) {
      StreamW& w = h->blk[i].s[s];
      if (h->w4) {
        auto take_q = [&b](QW& q, size_t rows, size_t k) {
          q.codes = b.take<uint8_t>(rows * k / 2);
          q.scales = b.take<uint32_t>(rows * (k / 64));
        };
        w.qkv = w.out = w.w13 = w.w2 = nullptr;
        take_q(w.q_qkv, 3 * kHidden, kHidden);
        take_q(w.q_out, kHidden, kHidden);
        take_q(w.q_w13, 2 * kMlp, kHidden);
        take_q(w.q_w2, kHidden, kMlp);
      } else {
        w.qkv = b.take<__nv_bfloat16>((size_t)3 * kHidden * kHidden);
        w.out = b.take<__nv_bfloat16>((size_t)kHidden * kHidden);
        w.w13 = b.take<__nv_bfloat16>((size_t)2 * kMlp * kHidden);
        w.w2 = b.take<__nv_bfloat16>((size_t)kHidden * kMlp);
      }
      w.b_qkv = b.take<float>(3 * kHidden);
      w.b_out = b.take<float>(kHidden);
      w.b_w13 = b.take<float>(2 * kMlp);
      w.b_w2 = b.take<float>(kHidden);
      w.gq = b.take<float>(kHeadDim);
      w.gk = b.take<float>(kHeadDim);
    }
}

// A block Linear weight [rows, k]: bf16 straight copy, or (weight_bits = 4) staged
// on the device and quantized into q at row offset row0 of a matrix of scale_ld rows.
static lens_status put_block_weight(lens_dit* h, __nv_bfloat16* dst, QW* q, const uint16_t* src, size_t rows,
                                    size_t k, size_t row0 = 0, size_t scale_ld = 0) {
  if (!h->w4) return put_bf16(dst, src, rows * k);
  if (!h->wstage || rows * k > kStageElems) return LENS_ERR_CUDA;
  if (cudaMemcpy(h->wstage, src, rows * k * 2, cudaMemcpyHostToDevice) != cudaSuccess) return LENS_ERR_CUDA;
  if (launch_quantize_w4(h->wstage, (int64_t)rows, (int64_t)k, q->codes + row0 * k / 2, q->scales + row0,
                         (int64_t)(scale_ld ? scale_ld : rows), nullptr) != cudaSuccess)
    return LENS_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return LENS_ERR_CUDA;   // wstage is reused by the next weight
  return LENS_OK;
}

static lens_status load_weights(lens_dit* h, const lens_weight* ws, int n_w) {
  Loader L;
  for (int i = 0; i < n_w; ++i) {
    if (!ws[i].name) return LENS_ERR_INVALID_ARG;
    if (!L.by_name.emplace(ws[i].name, &ws[i]).second) return LENS_ERR_INVALID_ARG;   // duplicate
  }
  const int nb = h->cfg.num_blocks;
  // every supplied name must be one this model consumes
  {
    size_t known = 0;
    auto count = [&](const std::string& n) { known += L.by_name.count(n); };
    const char* lin_top[] = {"time_text_embed.timestep_embedder.linear_1", "time_text_embed.timestep_embedder.linear_2",
                             "txt_in", "img_in", "norm_out.linear", "proj_out"};
    for (const char* n : lin_top) {
      count(std::string(n) + ".weight");
      count(std::string(n) + ".bias");
    }
    for (int l = 0; l < kTxtLayers; ++l) count("txt_norm." + std::to_string(l) + ".weight");
    const char* lin_blk[] = {"img_mod", "txt_mod", "attn.img_qkv", "attn.txt_qkv", "attn.to_out", "attn.to_add_out",
                             "img_mlp.w1", "img_mlp.w2", "img_mlp.w3", "txt_mlp.w1", "txt_mlp.w2", "txt_mlp.w3"};
    const char* gains[] = {"attn.norm_q", "attn.norm_k", "attn.norm_added_q", "attn.norm_added_k"};
    for (int i = 0; i < nb; ++i) {
      const std::string p = "transformer_blocks." + std::to_string(i) + ".";
      for (const char* n : lin_blk) {
        count(p + n + ".weight");
        count(p + n + ".bias");
      }
      for (const char* n : gains) count(p + n + ".weight");
    }
    // tensors of blocks beyond num_blocks are allowed (a 48-block list with a shorter config)
    size_t extra_blocks = 0;
    for (auto& kv : L.by_name) {
      const std::string& n = kv.first;
      if (n.rfind("transformer_blocks.", 0) == 0) {
        const int idx = atoi(n.c_str() + strlen("transformer_blocks."));
        if (idx >= nb) ++extra_blocks;
      }
    }
    if (known + extra_blocks != L.by_name.size()) return LENS_ERR_INVALID_ARG;
  }

  std::vector<float> stage;
  std::vector<uint16_t> pack;
  lens_status st;
  const int D = kHidden;
  // timestep MLP
  const char* te = "time_text_embed.timestep_embedder";
  const uint16_t* w;
  if (!(w = L.get(std::string(te) + ".linear_1.weight", {D, kFreqDim}, true))) return L.st;
  if ((st = put_bf16(h->w_t1, w, (size_t)D * kFreqDim))) return st;
  if ((st = put_f32(h->b_t1, L.get(std::string(te) + ".linear_1.bias", {D}, false), D, 0.f, stage))) return st;
  if (!(w = L.get(std::string(te) + ".linear_2.weight", {D, D}, true))) return L.st;
  if ((st = put_bf16(h->w_t2, w, (size_t)D * D))) return st;
  if ((st = put_f32(h->b_t2, L.get(std::string(te) + ".linear_2.bias", {D}, false), D, 0.f, stage))) return st;
  // text input
  for (int l = 0; l < kTxtLayers; ++l) {
    const uint16_t* g = L.get("txt_norm." + std::to_string(l) + ".weight", {kTxtDim}, true);
    if (!g) return L.st;
    if ((st = put_f32(h->g_txt + l * kTxtDim, g, kTxtDim, 1.f, stage))) return st;
  }
  if (!(w = L.get("txt_in.weight", {D, kTxtLayers * kTxtDim}, true))) return L.st;
  if ((st = put_bf16(h->w_txt_in, w, (size_t)D * kTxtLayers * kTxtDim))) return st;
  h->has_b_txt_in = any_nonzero_bf16(L.get("txt_in.bias", {D}, false), D);
  if ((st = put_f32(h->b_txt_in, L.get("txt_in.bias", {D}, false), D, 0.f, stage))) return st;
  // image input, packed [W | W] so the [hi | lo] operand reproduces fp32 tokens
  if (!(w = L.get("img_in.weight", {D, kInCh}, true))) return L.st;
  pack.resize((size_t)D * 2 * kInCh);
  for (int r = 0; r < D; ++r) {
    memcpy(&pack[(size_t)r * 2 * kInCh], w + (size_t)r * kInCh, kInCh * 2);
    memcpy(&pack[(size_t)r * 2 * kInCh + kInCh], w + (size_t)r * kInCh, kInCh * 2);
  }
  if ((st = put_bf16(h->w_img_in, pack.data(), pack.size()))) return st;
  h->has_b_img_in = any_nonzero_bf16(L.get("img_in.bias", {D}, false), D);
  if ((st = put_f32(h->b_img_in, L.get("img_in.bias", {D}, false), D, 0.f, stage))) return st;
  // final layer
  if (!(w = L.get("proj_out.weight", {kInCh, D}, true))) return L.st;
  if ((st = put_bf16(h->w_proj, w, (size_t)kInCh * D))) return st;
  h->has_b_proj = any_nonzero_bf16(L.get("proj_out.bias", {kInCh}, false), kInCh);
  if ((st = put_f32(h->b_proj, L.get("proj_out.bias", {kInCh}, false), kInCh, 0.f, stage))) return st;
  // all AdaLN projections: block-major, image then text, then norm_out
  const int64_t no_off = (int64_t)nb * kModPerBlock;
  if (!(w = L.get("norm_out.linear.weight", {2 * D, D}, true))) return L.st;
  if ((st = put_bf16(h->w4 ? h->w_no : h->w_mod + no_off * D, w, (size_t)2 * D * D))) return st;
  if ((st = put_f32(h->b_mod + no_off, L.get("norm_out.linear.bias", {2 * D}, false), 2 * D, 0.f, stage)))
    return st;

  for (int i = 0; i < nb; ++i) {
    const std::string p = "transformer_blocks." + std::to_string(i) + ".";
    for (int s = 0; s < 2; ++s) {
      StreamW& sw = h->blk[i].s[s];
      const std::string mod = p + (s == 0 ? "img_mod" : "txt_mod");
      const int64_t moff = (int64_t)i * kModPerBlock + s * kModPerStream;
      if (!(w = L.get(mod + ".weight", {kModPerStream, D}, true))) return L.st;
      if ((st = put_block_weight(h, h->w4 ? nullptr : h->w_mod + moff * D, &h->q_mod, w, kModPerStream, D, moff,
                                 (size_t)nb * kModPerBlock)))
        return st;
      if ((st = put_f32(h->b_mod + moff, L.get(mod + ".bias", {kModPerStream}, false), kModPerStream, 0.f, stage)))
        return st;

      const std::string qkv = p + (s == 0 ? "attn.img_qkv" : "attn.txt_qkv");
      if (!(w = L.get(qkv + ".weight", {3 * D, D}, true))) return L.st;
      if ((st = put_block_weight(h, sw.qkv, &sw.q_qkv, w, 3 * D, D))) return st;
      sw.has_b_qkv = any_nonzero_bf16(L.get(qkv + ".bias", {3 * D}, false), 3 * D);
      if ((st = put_f32(sw.b_qkv, L.get(qkv + ".bias", {3 * D}, false), 3 * D, 0.f, stage))) return st;
      const std::string nq = p + (s == 0 ? "attn.norm_q" : "attn.norm_added_q");
      const std::string nk = p + (s == 0 ? "attn.norm_k" : "attn.norm_added_k");
      const uint16_t* g;
      if (!(g = L.get(nq + ".weight", {kHeadDim}, true))) return L.st;
      if ((st = put_f32(sw.gq, g, kHeadDim, 1.f, stage))) return st;
      if (!(g = L.get(nk + ".weight", {kHeadDim}, true))) return L.st;
      if ((st = put_f32(sw.gk, g, kHeadDim, 1.f, stage))) return st;

      const std::string out = p + (s == 0 ? "attn.to_out" : "attn.to_add_out");
      if (!(w = L.get(out + ".weight", {D, D}, true))) return L.st;
      if ((st = put_block_weight(h, sw.out, &sw.q_out, w, D, D))) return st;
      sw.has_b_out = any_nonzero_bf16(L.get(out + ".bias", {D}, false), D);
      if ((st = put_f32(sw.b_out, L.get(out + ".bias", {D}, false), D, 0.f, stage))) return st;

      const std::string mlp = p + (s == 0 ? "img_mlp" : "txt_mlp");
      const uint16_t* w1 = L.get(mlp + ".w1.weight", {kMlp, D}, true);
      const uint16_t* w3 = L.get(mlp + ".w3.weight", {kMlp, D}, true);
      const uint16_t* w2 = L.get(mlp + ".w2.weight", {D, kMlp}, true);
      if (!w1 || !w3 || !w2) return L.st;
      // interleave per 32 output features: rows [64c, 64c+32) = w1 rows [32c, 32c+32),
      // rows [64c+32, 64c+64) = w3 rows [32c, 32c+32)
      pack.resize((size_t)2 * kMlp * D);
      for (int c = 0; c < kMlp / 32; ++c) {
        memcpy(&pack[(size_t)(64 * c) * D], w1 + (size_t)(32 * c) * D, (size_t)32 * D * 2);
        memcpy(&pack[(size_t)(64 * c + 32) * D], w3 + (size_t)(32 * c) * D, (size_t)32 * D * 2);
      }
      if ((st = put_block_weight(h, sw.w13, &sw.q_w13, pack.data(), 2 * kMlp, D))) return st;
      const uint16_t* b1 = L.get(mlp + ".w1.bias", {kMlp}, false);
      const uint16_t* b3 = L.get(mlp + ".w3.bias", {kMlp}, false);
      if (L.st) return L.st;
      sw.has_b_w13 = any_nonzero_bf16(b1, kMlp) || any_nonzero_bf16(b3, kMlp);
      stage.resize(2 * kMlp);
      for (int c = 0; c < kMlp / 32; ++c)
        for (int j = 0; j < 32; ++j) {
          stage[64 * c + j] = b1 ? bf16_to_f32(b1[32 * c + j]) : 0.f;
          stage[64 * c + 32 + j] = b3 ? bf16_to_f32(b3[32 * c + j]) : 0.f;
        }
      if (cudaMemcpy(sw.b_w13, stage.data(), 2 * kMlp * 4, cudaMemcpyHostToDevice) != cudaSuccess)
        return LENS_ERR_CUDA;
      if ((st = put_block_weight(h, sw.w2, &sw.q_w2, w2, D, kMlp))) return st;
      sw.has_b_w2 = any_nonzero_bf16(L.get(mlp + ".w2.bias", {D}, false), D);
      if ((st = put_f32(sw.b_w2, L.get(mlp + ".w2.bias", {D}, false), D, 0.f, stage))) return st;
    }
  }
  return L.st;
}

static lens_status make_weight_maps(lens_dit* h) {
  const int D = kHidden;
  bool ok = encode_tmap_bf16(&h->t_txt_in, h->w_txt_in, D, kTxtLayers * kTxtDim, kTxtLayers * kTxtDim, kBnTxtIn) &&
            encode_tmap_bf16(&h->t_img_in, h->w_img_in, D, 2 * kInCh, 2 * kInCh, kBnImgIn) &&
            encode_tmap_bf16(&h->t_proj, h->w_proj, kInCh, D, D, kBnProj);
  if (h->w4) {
    auto qmaps = [](QW& q, uint64_t rows, uint64_t k, uint32_t box) {
      return encode_tmap_w4_codes(&q.tq, q.codes, rows, k, box) && encode_tmap_w4_scales(&q.ts, q.scales, rows, k, box);
    };
    ok = ok && encode_tmap_bf16(&h->t_no, h->w_no, 2 * D, D, D, 128) &&
         qmaps(h->q_mod, (uint64_t)h->cfg.num_blocks * kModPerBlock, D, 128);
    for (auto& b : h->blk)
      for (auto& s : b.s)     // 4-bit block GEMMs run on single CTAs: the B box is the whole tile width
        ok = ok && qmaps(s.q_qkv, 3 * D, D, kBnQkvW4) && qmaps(s.q_out, D, D, kBnResW4) &&
             qmaps(s.q_w13, 2 * kMlp, D, kBnW13W4) && qmaps(s.q_w2, D, kMlp, kBnResW4);
    return ok ? LENS_OK : LENS_ERR_CUDA;
  }
  ok = ok && encode_tmap_bf16(&h->t_mod, h->w_mod, h->modw, D, D, 128);
  for (auto& b : h->blk)
    for (auto& s : b.s)
      // block GEMMs run on CTA pairs: each CTA stages half of the B tile
      ok = ok && encode_tmap_bf16(&s.t_qkv, s.qkv, 3 * D, D, D, kBnQkv / 2) &&
           encode_tmap_bf16(&s.t_out, s.out, D, D, D, kBnOut / 2) &&
           encode_tmap_bf16(&s.t_w13, s.w13, 2 * kMlp, D, D, kBnW13 / 2) &&
           encode_tmap_bf16(&s.t_w2, s.w2, D, kMlp, kMlp, kBnW2 / 2);
  for (auto& b : h->blk)
    for (auto& s : b.s)
      for (int i = 0; i < 2; ++i) {   // half of a 2- or 4-way column slice per CTA
        const int q = 4 << i;
        ok = ok && encode_tmap_bf16(&s.n_qkv[i], s.qkv, 3 * D, D, D, kBnQkv / q) &&
             encode_tmap_bf16(&s.n_out[i], s.out, D, D, D, kBnOut / q) &&
             encode_tmap_bf16(&s.n_w13[i], s.w13, 2 * kMlp, D, D, kBnW13 / q) &&
             encode_tmap_bf16(&s.n_w2[i], s.w2, D, kMlp, kMlp, kBnW2 / q);
      }
  return ok ? LENS_OK : LENS_ERR_CUDA;
}

static size_t layout_workspace(lens_dit* h, Bump& b) {
  const lens_dit_config& c = h->cfg;
  const size_t Bm = c.max_batch, Ni = c.max_img_tokens, Nt = c.max_txt_tokens, N = Ni + Nt;
  const size_t Tm = c.max_timesteps;
  h->xin = b.take<__nv_bfloat16>(Bm * Ni * 2 * kInCh);
  h->a_img = b.take<__nv_bfloat16>(Bm * Ni * kHidden);
  h->a_txt = b.take<__nv_bfloat16>(Bm * Nt * kHidden + 1);
  h->q = b.take<__nv_bfloat16>(Bm * kHeads * N * kHeadDim);
  h->k = b.take<__nv_bfloat16>(Bm * kHeads * N * kHeadDim);
  h->v = b.take<__nv_bfloat16>(Bm * kHeads * N * kHeadDim);
  h->o_img = b.take<__nv_bfloat16>(Bm * Ni * kHidden);
  h->o_txt = b.take<__nv_bfloat16>(Bm * Nt * kHidden + 1);
  h->u_img = b.take<__nv_bfloat16>(Bm * Ni * kMlp);
  h->u_txt = b.take<__nv_bfloat16>(Bm * Nt * kMlp + 1);
  h->txt_cat = b.take<__nv_bfloat16>(Bm * Nt * kTxtLayers * kTxtDim + 1);
  h->stemb = b.take<__nv_bfloat16>((size_t)kMaxTimesteps * kHidden);
  h->h_img = b.take<float>(Bm * Ni * kHidden);
  h->h_txt = b.take<float>(Bm * Nt * kHidden + 1);
  h->h_txt0 = b.take<float>(Bm * Nt * kHidden + 1);
  h->vtok = b.take<float>(Bm * Ni * kInCh);
  h->xtok = b.take<float>(Bm * Ni * kInCh);
  h->tfeat = b.take<float>((size_t)kMaxTimesteps * kFreqDim);
  h->hid = b.take<float>((size_t)kMaxTimesteps * kHidden);
  h->temb = b.take<float>((size_t)kMaxTimesteps * kHidden);
  h->mod = b.take<float>(Tm * h->modw);
  h->rope = b.take<float2>(N * 32);
  h->cfgpart = b.take<double>(Bm * kCfgNormParts * 2);
  h->err = b.take<int>(1);
  return b.off;
}

// ============================================================ path pieces
static lens_status compute_modulation(lens_dit* h, const float* t, int T, cudaStream_t st) {
  TimestepList tl;
  tl.T = T;
  for (int i = 0; i < T; ++i) tl.t[i] = t[i];
  const int Tpad = T <= 16 ? 16 : (T <= 32 ? 32 : 64);
  LENS_LAUNCH(h, 0, st, launch_timestep_features(tl, h->tfeat, st));
  LENS_LAUNCH(h, 0, st, launch_small_linear(h->tfeat, T, kFreqDim, h->w_t1, h->b_t1, kHidden, false, h->hid, nullptr, 0, st));
  LENS_LAUNCH(h, 0, st, launch_small_linear(h->hid, T, kHidden, h->w_t2, h->b_t2, kHidden, true, h->temb, h->stemb, Tpad, st));
  CUtensorMap tb;
  if (!encode_tmap_bf16(&tb, h->stemb, Tpad, kHidden, kHidden, Tpad)) return LENS_ERR_CUDA;
  GemmArgs a = make_args(h->err);
  a.num_problems = 1;
  a.p[0] = base_problem((int)h->modw, Tpad, kHidden);
  a.p[0].out_f32 = h->mod;
  a.p[0].ld_out = h->modw;
  a.p[0].bias = h->b_mod;
  a.p[0].n_valid = T;
  if (h->w4) {
    // 4-bit block AdaLN rows, then the bf16 norm_out rows into the same buffer
    const int mrows = h->cfg.num_blocks * kModPerBlock;
    a.p[0].M = mrows;
    LENS_LAUNCH(h, LENS_KERNEL_GEMM_MOD, st, launch_gemm_w4(128, Tpad, EPI_F32_T, true, nullptr, &tb, &h->q_mod.tq, &h->q_mod.ts, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, a, h->sms, st));
    GemmArgs a2 = make_args(h->err);
    a2.num_problems = 1;
    a2.p[0] = base_problem(2 * kHidden, Tpad, kHidden);
    a2.p[0].out_f32 = h->mod + mrows;
    a2.p[0].ld_out = h->modw;
    a2.p[0].bias = h->b_mod + mrows;
    a2.p[0].n_valid = T;
    LENS_LAUNCH(h, LENS_KERNEL_GEMM_MOD, st, launch_gemm(Tpad, EPI_F32_T, &h->t_no, &tb, nullptr, nullptr, nullptr, nullptr, a2, h->sms, st));
    return LENS_OK;
  }
  LENS_LAUNCH(h, LENS_KERNEL_GEMM_MOD, st, launch_gemm(Tpad, EPI_F32_T, &h->t_mod, &tb, nullptr, nullptr, nullptr, nullptr, a, h->sms, st));
  return LENS_OK;
}

// txt [B*n_txt, 4, 2880] (or zeros when txt is null) -> h->txt_cat rows [row0, row0 + rows)
static lens_status text_norm_rows(lens_dit* h, const uint16_t* txt, int rows, int row0, cudaStream_t st) {
  __nv_bfloat16* dst = h->txt_cat + (size_t)row0 * kTxtLayers * kTxtDim;
  if (rows <= 0) return LENS_OK;
  if (!txt) {
    LENS_CUDA(cudaMemsetAsync(dst, 0, (size_t)rows * kTxtLayers * kTxtDim * 2, st));
    return LENS_OK;
  }
  LENS_LAUNCH(h, 0, st, launch_text_norm(reinterpret_cast<const __nv_bfloat16*>(txt), rows, h->g_txt, h->cfg.eps, dst, st));
  return LENS_OK;
}

static lens_status text_in_gemm(lens_dit* h, int rows, float* out, cudaStream_t st) {
  if (rows <= 0) return LENS_OK;
  CUtensorMap ta, tc;
  if (!encode_tmap_bf16(&ta, h->txt_cat, rows, kTxtLayers * kTxtDim, kTxtLayers * kTxtDim, 128) ||
      !encode_tmap_out(&tc, out, 4, rows, kHidden, kHidden))
    return LENS_ERR_CUDA;
  GemmArgs a = make_args(h->err);
  a.num_problems = 1;
  a.p[0] = base_problem(rows, kHidden, kTxtLayers * kTxtDim);
  a.p[0].out_f32 = out;
  a.p[0].ld_out = kHidden;
  a.p[0].bias = h->has_b_txt_in ? h->b_txt_in : nullptr;
  LENS_LAUNCH(h, 0, st, launch_gemm(kBnTxtIn, EPI_F32, &ta, &h->t_txt_in, nullptr, nullptr, &tc, nullptr, a, h->sms, st));
  return LENS_OK;
}

// Tensor maps of one forward's activations: GEMM A operands (a, o, u as bf16, box
// 128 rows) and TMA-store targets (residual streams h as fp32, u as bf16).
struct ActMaps {
  CUtensorMap a_img, a_txt, o_img, o_txt, u_img, u_txt;      // A operands
  CUtensorMap h_img, h_txt, uo_img, uo_txt;                  // epilogue outputs
  bool has_txt;
};

static lens_status make_act_maps(lens_dit* h, int Mi, int Mt, float* hi, float* ht, ActMaps& m) {
  m.has_txt = Mt > 0;
  bool ok = encode_tmap_bf16(&m.a_img, h->a_img, Mi, kHidden, kHidden, 128) &&
            encode_tmap_bf16(&m.o_img, h->o_img, Mi, kHidden, kHidden, 128) &&
            encode_tmap_bf16(&m.u_img, h->u_img, Mi, kMlp, kMlp, 128) &&
            encode_tmap_out(&m.h_img, hi, 4, Mi, kHidden, kHidden) &&
            encode_tmap_out(&m.uo_img, h->u_img, 2, Mi, kMlp, kMlp);
  if (m.has_txt)
    ok = ok && encode_tmap_bf16(&m.a_txt, h->a_txt, Mt, kHidden, kHidden, 128) &&
         encode_tmap_bf16(&m.o_txt, h->o_txt, Mt, kHidden, kHidden, 128) &&
         encode_tmap_bf16(&m.u_txt, h->u_txt, Mt, kMlp, kMlp, 128) &&
         encode_tmap_out(&m.h_txt, ht, 4, Mt, kHidden, kHidden) &&
         encode_tmap_out(&m.uo_txt, h->u_txt, 2, Mt, kMlp, kMlp);
  return ok ? LENS_OK : LENS_ERR_CUDA;
}

// One dual-stream block on residual streams hi [B*Ni, 1536], ht [B*Nt, 1536].
static lens_status run_block(lens_dit* h, int i, float* hi, float* ht, int B, int Ni, int Nt, const float* mod,
                             int64_t mstride, const ActMaps& am, const TextLengths* tl, cudaStream_t st) {
  const float eps = h->cfg.eps;
  const int Mi = B * Ni, Mt = B * Nt, N = Ni + Nt;
  const float* mI = mod + (int64_t)i * kModPerBlock;
  const float* mT = mI + kModPerStream;
  const StreamW& wi = h->blk[i].s[0];
  const StreamW& wt = h->blk[i].s[1];
  const int np = am.has_txt ? 2 : 1;

  // attention branch (both streams in one launch)
  {
    const RmsSeg si{hi, mI, mI + kHidden, h->a_img, Mi, Ni, mstride};
    const RmsSeg stx{ht, mT, mT + kHidden, h->a_txt, np > 1 ? Mt : 0, Nt > 0 ? Nt : 1, mstride};
    LENS_LAUNCH(h, LENS_KERNEL_RMSNORM_MOD, st, launch_rmsnorm_modulate(si, stx, eps, st));
  }
  {
    GemmArgs a = make_args(h->err);
    a.num_problems = np;
    for (int s = 0; s < np; ++s) {
      const StreamW& w = h->blk[i].s[s];
      GemmProblem p = base_problem(s == 0 ? Mi : Mt, 3 * kHidden, kHidden);
      p.bias = w.has_b_qkv ? w.b_qkv : nullptr;
      p.q = h->q;
      p.k = h->k;
      p.v = h->v;
      p.gain_q = w.gq;
      p.gain_k = w.gk;
      p.rope = h->rope;
      p.n_tok = N;
      p.tok_offset = s == 0 ? Nt : 0;
      p.rows_per_batch = s == 0 ? Ni : Nt;
      p.eps = eps;
      a.p[s] = p;
    }
    if (h->w4) {
      LENS_LAUNCH(h, LENS_KERNEL_GEMM_QKV, st, launch_gemm_w4(256, kBnQkvW4, EPI_QKV, false, &am.a_img, nullptr, &wi.q_qkv.tq, &wi.q_qkv.ts,
                            np > 1 ? &am.a_txt : nullptr, nullptr, np > 1 ? &wt.q_qkv.tq : nullptr, np > 1 ? &wt.q_qkv.ts : nullptr,
                            nullptr, nullptr, a, h->sms, st));
    } else {
      const NarrowB nb{{&wi.n_qkv[0], &wi.n_qkv[1]}, {&wt.n_qkv[0], &wt.n_qkv[1]}};
      LENS_LAUNCH(h, LENS_KERNEL_GEMM_QKV, st, launch_gemm_pair(kBnQkv, EPI_QKV, &am.a_img, &wi.t_qkv, np > 1 ? &am.a_txt : nullptr,
                            np > 1 ? &wt.t_qkv : nullptr, nullptr, nullptr, a, h->sms, st, &nb));
    }
  }
  LENS_LAUNCH(h, LENS_KERNEL_ATTENTION, st, launch_joint_attention(h->q, h->k, h->v, B, kHeads, Nt, Ni, h->o_txt, h->o_img, tl, h->err, st));
  {
    GemmArgs a = make_args(h->err);
    a.num_problems = np;
    for (int s = 0; s < np; ++s) {
      const StreamW& w = h->blk[i].s[s];
      GemmProblem p = base_problem(s == 0 ? Mi : Mt, kHidden, kHidden);
      p.out_f32 = s == 0 ? hi : ht;
      p.ld_out = kHidden;
      p.bias = w.has_b_out ? w.b_out : nullptr;
      p.gate = (s == 0 ? mI : mT) + 2 * kHidden;
      p.gate_stride = mstride;
      p.rows_per_batch = s == 0 ? Ni : Nt;
      a.p[s] = p;
    }
    if (h->w4) {
      LENS_LAUNCH(h, LENS_KERNEL_GEMM_OUT, st, launch_gemm_w4(256, kBnResW4, EPI_RESID, false, &am.o_img, nullptr, &wi.q_out.tq, &wi.q_out.ts,
                            np > 1 ? &am.o_txt : nullptr, nullptr, np > 1 ? &wt.q_out.tq : nullptr, np > 1 ? &wt.q_out.ts : nullptr,
                            &am.h_img, np > 1 ? &am.h_txt : nullptr, a, h->sms, st));
    } else {
      const NarrowB nb{{&wi.n_out[0], &wi.n_out[1]}, {&wt.n_out[0], &wt.n_out[1]}};
      LENS_LAUNCH(h, LENS_KERNEL_GEMM_OUT, st, launch_gemm_pair(kBnOut, EPI_RESID, &am.o_img, &wi.t_out, np > 1 ? &am.o_txt : nullptr,
                            np > 1 ? &wt.t_out : nullptr, &am.h_img, np > 1 ? &am.h_txt : nullptr, a, h->sms, st, &nb));
    }
  }
  // MLP branch
  {
    const RmsSeg si{hi, mI + 3 * kHidden, mI + 4 * kHidden, h->a_img, Mi, Ni, mstride};
    const RmsSeg stx{ht, mT + 3 * kHidden, mT + 4 * kHidden, h->a_txt, np > 1 ? Mt : 0, Nt > 0 ? Nt : 1, mstride};
    LENS_LAUNCH(h, LENS_KERNEL_RMSNORM_MOD, st, launch_rmsnorm_modulate(si, stx, eps, st));
  }
  {
    GemmArgs a = make_args(h->err);
    a.num_problems = np;
    for (int s = 0; s < np; ++s) {
      const StreamW& w = h->blk[i].s[s];
      GemmProblem p = base_problem(s == 0 ? Mi : Mt, 2 * kMlp, kHidden);
      p.out_bf16 = s == 0 ? h->u_img : h->u_txt;
      p.bias = w.has_b_w13 ? w.b_w13 : nullptr;
      a.p[s] = p;
    }
    if (h->w4) {
      LENS_LAUNCH(h, LENS_KERNEL_GEMM_W13, st, launch_gemm_w4(256, kBnW13W4, EPI_SWIGLU, false, &am.a_img, nullptr, &wi.q_w13.tq, &wi.q_w13.ts,
                            np > 1 ? &am.a_txt : nullptr, nullptr, np > 1 ? &wt.q_w13.tq : nullptr, np > 1 ? &wt.q_w13.ts : nullptr,
                            &am.uo_img, np > 1 ? &am.uo_txt : nullptr, a, h->sms, st));
    } else {
      const NarrowB nb{{&wi.n_w13[0], &wi.n_w13[1]}, {&wt.n_w13[0], &wt.n_w13[1]}};
      LENS_LAUNCH(h, LENS_KERNEL_GEMM_W13, st, launch_gemm_pair(kBnW13, EPI_SWIGLU, &am.a_img, &wi.t_w13, np > 1 ? &am.a_txt : nullptr,
                            np > 1 ? &wt.t_w13 : nullptr, &am.uo_img, np > 1 ? &am.uo_txt : nullptr, a, h->sms, st, &nb));
    }
  }
  {
    GemmArgs a = make_args(h->err);
    a.num_problems = np;
    for (int s = 0; s < np; ++s) {
      const StreamW& w = h->blk[i].s[s];
      GemmProblem p = base_problem(s == 0 ? Mi : Mt, kHidden, kMlp);
      p.out_f32 = s == 0 ? hi : ht;
      p.ld_out = kHidden;
      p.bias = w.has_b_w2 ? w.b_w2 : nullptr;
      p.gate = (s == 0 ? mI : mT) + 5 * kHidden;
      p.gate_stride = mstride;
      p.rows_per_batch = s == 0 ? Ni : Nt;
      a.p[s] = p;
    }
    if (h->w4) {
      LENS_LAUNCH(h, LENS_KERNEL_GEMM_W2, st, launch_gemm_w4(256, kBnResW4, EPI_RESID, false, &am.u_img, nullptr, &wi.q_w2.tq, &wi.q_w2.ts,
                            np > 1 ? &am.u_txt : nullptr, nullptr, np > 1 ? &wt.q_w2.tq : nullptr, np > 1 ? &wt.q_w2.ts : nullptr,
                            &am.h_img, np > 1 ? &am.h_txt : nullptr, a, h->sms, st));
    } else {
      const NarrowB nb{{&wi.n_w2[0], &wi.n_w2[1]}, {&wt.n_w2[0], &wt.n_w2[1]}};
      LENS_LAUNCH(h, LENS_KERNEL_GEMM_W2, st, launch_gemm_pair(kBnW2, EPI_RESID, &am.u_img, &wi.t_w2, np > 1 ? &am.u_txt : nullptr,
                            np > 1 ? &wt.t_w2 : nullptr, &am.h_img, np > 1 ? &am.h_txt : nullptr, a, h->sms, st, &nb));
    }
  }
  return LENS_OK;
}

// Whole forward: h->xin holds the [hi | lo] token operand [B*Ni, 256] and h->h_txt0
// the text input [B*Nt, 1536]; velocity tokens go to v_dst [B*Ni, 128].
static lens_status run_forward_core(lens_dit* h, int B, int gh, int gw, int Nt, const float* mod, int64_t mstride,
                                    float* v_dst, const TextLengths* tl, cudaStream_t st) {
  const int Ni = gh * gw, Mi = B * Ni, Mt = B * Nt;
  lens_status s;
  LENS_LAUNCH(h, 0, st, launch_rope_table(gh, gw, Nt, h->rope, st));
  {
    CUtensorMap tx, th;
    if (!encode_tmap_bf16(&tx, h->xin, Mi, 2 * kInCh, 2 * kInCh, 128) ||
        !encode_tmap_out(&th, h->h_img, 4, Mi, kHidden, kHidden))
      return LENS_ERR_CUDA;
    GemmArgs a = make_args(h->err);
    a.num_problems = 1;
    a.p[0] = base_problem(Mi, kHidden, 2 * kInCh);
    a.p[0].out_f32 = h->h_img;
    a.p[0].ld_out = kHidden;
    a.p[0].bias = h->has_b_img_in ? h->b_img_in : nullptr;
    LENS_LAUNCH(h, 0, st, launch_gemm(kBnImgIn, EPI_F32, &tx, &h->t_img_in, nullptr, nullptr, &th, nullptr, a, h->sms, st));
  }
  if (Mt > 0) LENS_CUDA(cudaMemcpyAsync(h->h_txt, h->h_txt0, (size_t)Mt * kHidden * 4, cudaMemcpyDeviceToDevice, st));
  ActMaps am;
  if ((s = make_act_maps(h, Mi, Mt, h->h_img, h->h_txt, am))) return s;
  for (int i = 0; i < h->cfg.num_blocks; ++i)
    if ((s = run_block(h, i, h->h_img, h->h_txt, B, Ni, Nt, mod, mstride, am, tl, st))) return s;
  const float* no = mod + (int64_t)h->cfg.num_blocks * kModPerBlock;   // (scale, shift)
  LENS_LAUNCH(h, LENS_KERNEL_RMSNORM_MOD, st, launch_rmsnorm_modulate(h->h_img, Mi, Ni, no + kHidden, no, mstride, h->cfg.eps, h->a_img, st));
  {
    CUtensorMap tv;
    if (!encode_tmap_out(&tv, v_dst, 4, Mi, kInCh, kInCh)) return LENS_ERR_INVALID_ARG;
    GemmArgs a = make_args(h->err);
    a.num_problems = 1;
    a.p[0] = base_problem(Mi, kInCh, kHidden);
    a.p[0].out_f32 = v_dst;
    a.p[0].ld_out = kInCh;
    a.p[0].bias = h->has_b_proj ? h->b_proj : nullptr;
    LENS_LAUNCH(h, 0, st, launch_gemm(kBnProj, EPI_F32, &am.a_img, &h->t_proj, nullptr, nullptr, &tv, nullptr, a, h->sms, st));
  }
  return LENS_OK;
}

static lens_status check_model_fields(const lens_dit_config* c) {
  lens_dit_config d;
  lens_dit_default_config(&d);
  if (c->hidden != d.hidden || c->heads != d.heads || c->head_dim != d.head_dim || c->mlp_hidden != d.mlp_hidden ||
      c->in_channels != d.in_channels || c->latent_channels != d.latent_channels || c->patch != d.patch ||
      c->txt_layers != d.txt_layers || c->txt_dim != d.txt_dim || c->rope_axes[0] != d.rope_axes[0] ||
      c->rope_axes[1] != d.rope_axes[1] || c->rope_axes[2] != d.rope_axes[2] || c->rope_theta != d.rope_theta ||
      c->freq_dim != d.freq_dim)
    return LENS_ERR_UNSUPPORTED;
  if (c->num_blocks < 1 || c->num_blocks > 48) return LENS_ERR_UNSUPPORTED;
  if (c->weight_bits != 16 && c->weight_bits != 4) return LENS_ERR_UNSUPPORTED;
  if (!(c->eps > 0.f) || !isfinite(c->eps)) return LENS_ERR_INVALID_ARG;
  if (c->max_batch < 1 || c->max_img_tokens < 1 || c->max_txt_tokens < 0 || c->max_timesteps < 1 ||
      c->max_timesteps > kMaxTimesteps)
    return LENS_ERR_SHAPE;
  return LENS_OK;
}

static void drop_sample_graph(lens_dit* h) {
  if (h->sg.exec) cudaGraphExecDestroy(h->sg.exec);
  if (h->sg.graph) cudaGraphDestroy(h->sg.graph);
  h->sg = lens_dit::SampleGraph();
}

// t_0 .. t_S of the sampler: the uniform grid 1 - k/S, optionally mapped through the
// resolution shift t' = e^mu t / (e^mu t + 1 - t) (summary page "Lens: 重新思考基础文生图
// 模型的训练效率", "Flow Matching 训练目标": the schedule at each resolution follows a
// mu(n) linear interpolation; the published resolution-dependent shift is taken).
static void sampler_time_grid(int steps, bool shift, double mu, double* t) {
  const double a = exp(mu);
  for (int k = 0; k <= steps; ++k) {
    const double u = 1.0 - (double)k / (double)steps;
    t[k] = shift ? a * u / (a * u + (1.0 - u)) : u;
  }
  t[steps] = 0.0;
}

// Enqueue one sampler call on `st` (validated arguments).
static lens_status enqueue_sample(lens_dit* h, const uint16_t* txt_cond, const uint16_t* txt_uncond, int B,
                                  int n_txt, int gh, int gw, int steps, const lens_sampler_options& o, uint64_t seed,
                                  float* latent_out, const TextLengths* tl, cudaStream_t st) {
  const float guidance = o.guidance;
  const bool cfg = guidance != 1.0f;
  const bool rescale = cfg && o.cfg_rescale != 0.0f;
  const bool shift = o.time_shift != 0;
  const int Ni = gh * gw;
  const int Bf = cfg ? 2 * B : B;
  const int64_t per_sample = (int64_t)Ni * kInCh;
  lens_status s;
  LENS_LAUNCH(h, 0, st, launch_noise_tokens(seed, B, gh, gw, h->xtok, st));
  LENS_LAUNCH(h, 0, st, launch_tokens_to_operand(h->xtok, (int64_t)B * Ni, cfg ? 2 : 1, (int64_t)B * Ni, h->xin, st));
  if ((s = text_norm_rows(h, txt_cond, B * n_txt, 0, st))) return s;
  if (cfg && (s = text_norm_rows(h, txt_uncond, B * n_txt, B * n_txt, st))) return s;
  if ((s = text_in_gemm(h, Bf * n_txt, h->h_txt0, st))) return s;

  const int chunk = h->cfg.max_timesteps;
  std::vector<double> grid(steps + 1);
  sampler_time_grid(steps, shift, o.shift_mu, grid.data());
  float tv[kMaxTimesteps];
  for (int k0 = 0; k0 < steps; k0 += chunk) {
    const int T = steps - k0 < chunk ? steps - k0 : chunk;
    for (int j = 0; j < T; ++j) tv[j] = (float)grid[k0 + j];
    if ((s = compute_modulation(h, tv, T, st))) return s;
    for (int j = 0; j < T; ++j) {
      // uniform grid: every step is exactly 1/S, as in the plain sampler
      const float dt = shift ? (float)(grid[k0 + j] - grid[k0 + j + 1]) : 1.0f / (float)steps;
      if ((s = run_forward_core(h, Bf, gh, gw, n_txt, h->mod + (int64_t)j * h->modw, 0, h->vtok, tl, st))) return s;
      if (rescale) {
        const float* vu = h->vtok + (int64_t)B * per_sample;
        LENS_LAUNCH(h, 0, st, launch_cfg_norm_partials(h->vtok, vu, per_sample, B, guidance, h->cfgpart, st));
        LENS_LAUNCH(h, 0, st, launch_euler_cfg_rescaled(h->xtok, h->vtok, vu, per_sample, B, dt, guidance,
                                                        o.cfg_rescale, h->cfgpart, h->xin, 2, st));
      } else {
        LENS_LAUNCH(h, 0, st, launch_euler_cfg(h->xtok, h->vtok, per_sample, B, cfg, dt, guidance, h->xin, st));
      }
    }
  }
  LENS_LAUNCH(h, 0, st, launch_unpatchify(h->xtok, B, gh, gw, latent_out, st));
  return LENS_OK;
}

// ============================================================ C ABI
extern "C" {

const char* lens_status_string(lens_status s) {
  if ((int)s < 0 || (int)s > 6) return "unknown status";
  return kStatusStr[(int)s];
}

int lens_device_sm_count(void) { return device_sms(); }

lens_status lens_dit_default_config(lens_dit_config* c) {
  if (!c) return LENS_ERR_INVALID_ARG;
  c->num_blocks = 48;
  c->hidden = 1536;
  c->heads = 24;
  c->head_dim = 64;
  c->mlp_hidden = 4096;
  c->in_channels = 128;
  c->latent_channels = 32;
  c->patch = 2;
  c->txt_layers = 4;
  c->txt_dim = 2880;
  c->rope_axes[0] = 8;
  c->rope_axes[1] = 28;
  c->rope_axes[2] = 28;
  c->rope_theta = 10000.f;
  c->eps = 1e-6f;
  c->freq_dim = 256;
  c->max_batch = 2;
  c->max_img_tokens = 4096;
  c->max_txt_tokens = 256;
  c->max_timesteps = 64;
  c->weight_bits = 16;
  return LENS_OK;
}

lens_status lens_dit_create(const lens_dit_config* cfg, const lens_weight* w, int n_w, void* stream,
                            lens_dit** out) {
  if (!cfg || !w || n_w <= 0 || !out) return LENS_ERR_INVALID_ARG;
  *out = nullptr;
  lens_status s = check_model_fields(cfg);
  if (s) return s;
  lens_dit* h = new lens_dit();
  h->cfg = *cfg;
  h->w4 = cfg->weight_bits == 4;
  h->modw = (int64_t)cfg->num_blocks * kModPerBlock + 2 * kHidden;
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return LENS_ERR_CUDA;
  }
  h->sms = device_sms();
  Bump wb;
  layout_weights(h, wb);
  const size_t wbytes = wb.off;
  Bump sb;
  layout_workspace(h, sb);
  const size_t sbytes = sb.off;
  if (cudaMalloc(&h->warena, wbytes) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return LENS_ERR_OOM;
  }
  if (cudaMalloc(&h->ws, sbytes) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(h->warena);
    delete h;
    return LENS_ERR_OOM;
  }
  wb = Bump();
  wb.base = reinterpret_cast<uintptr_t>(h->warena);
  layout_weights(h, wb);
  sb = Bump();
  sb.base = reinterpret_cast<uintptr_t>(h->ws);
  layout_workspace(h, sb);
  // weight_bits = 4: one bf16 matrix at a time is staged on the device and quantized
  if (h->w4 && cudaMalloc(&h->wstage, kStageElems * 2) != cudaSuccess) {
    cudaGetLastError();
    lens_dit_destroy(h);
    return LENS_ERR_OOM;
  }
  s = load_weights(h, w, n_w);
  if (h->wstage) {
    cudaDeviceSynchronize();
    cudaFree(h->wstage);
    h->wstage = nullptr;
  }
  if (s == LENS_OK) s = make_weight_maps(h);
  if (s == LENS_OK && cudaMemsetAsync(h->err, 0, sizeof(int), (cudaStream_t)stream) != cudaSuccess)
    s = LENS_ERR_CUDA;
  if (s == LENS_OK && cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) s = LENS_ERR_CUDA;
  if (s != LENS_OK) {
    lens_dit_destroy(h);
    return s;
  }
  *out = h;
  return LENS_OK;
}

void lens_dit_destroy(lens_dit* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  drop_sample_graph(h);
  for (cudaEvent_t e : h->prof_ev) cudaEventDestroy(e);
  if (h->wstage) cudaFree(h->wstage);
  if (h->ws) cudaFree(h->ws);
  if (h->warena) cudaFree(h->warena);
  delete h;
}

lens_status lens_dit_debug_raise_abort(lens_dit* h, void* stream) {
  if (!h) return LENS_ERR_INVALID_ARG;
  // the flag is a little-endian int that is otherwise 0: its low byte makes it 1
  if (cudaMemsetAsync(h->err, 1, 1, (cudaStream_t)stream) != cudaSuccess) return LENS_ERR_CUDA;
  return LENS_OK;
}

lens_status lens_dit_sync(lens_dit* h, void* stream) {
  if (!h) return LENS_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LENS_ERR_CUDA;
  int e = 0;
  if (cudaMemcpy(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LENS_ERR_CUDA;
  if (e) {
    cudaMemset(h->err, 0, sizeof(int));
    return LENS_ERR_TIMEOUT;
  }
  return LENS_OK;
}

static lens_status check_sizes(lens_dit* h, int B, int gh, int gw, int n_txt) {
  if (B < 1 || gh < 1 || gw < 1 || n_txt < 0) return LENS_ERR_SHAPE;
  if (B > h->cfg.max_batch || (int64_t)gh * gw > h->cfg.max_img_tokens || n_txt > h->cfg.max_txt_tokens)
    return LENS_ERR_SHAPE;
  return LENS_OK;
}

lens_status lens_dit_forward(lens_dit* h, const float* img_tokens, int B, int grid_h, int grid_w,
                             const uint16_t* txt, int n_txt, const float* t, float* v_out, void* stream) {
  return lens_dit_forward_masked(h, img_tokens, B, grid_h, grid_w, txt, n_txt, nullptr, t, v_out, stream);
}

lens_status lens_dit_forward_masked(lens_dit* h, const float* img_tokens, int B, int grid_h, int grid_w,
                                    const uint16_t* txt, int n_txt, const int* txt_len, const float* t, float* v_out,
                                    void* stream) {
  if (!h || !img_tokens || !t || !v_out || (n_txt > 0 && !txt)) return LENS_ERR_INVALID_ARG;
  h->ss.ready = false;
  TextLengths tl;
  if (txt_len) {
    if (B > kMaxRows) return LENS_ERR_SHAPE;
    for (int b = 0; b < B; ++b) {
      if (txt_len[b] < 0 || txt_len[b] > n_txt) return LENS_ERR_SHAPE;
      tl.n[b] = txt_len[b];
    }
  }
  lens_status s = check_sizes(h, B, grid_h, grid_w, n_txt);
  if (s) return s;
  if (B > h->cfg.max_timesteps) return LENS_ERR_SHAPE;
  for (int i = 0; i < B; ++i)
    if (!isfinite(t[i])) return LENS_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int Ni = grid_h * grid_w;
  if ((s = compute_modulation(h, t, B, st))) return s;
  LENS_LAUNCH(h, 0, st, launch_tokens_to_operand(img_tokens, (int64_t)B * Ni, 1, 0, h->xin, st));
  if ((s = text_norm_rows(h, txt, B * n_txt, 0, st))) return s;
  if ((s = text_in_gemm(h, B * n_txt, h->h_txt0, st))) return s;
  return run_forward_core(h, B, grid_h, grid_w, n_txt, h->mod, h->modw, v_out, txt_len ? &tl : nullptr, st);
}

lens_status lens_dit_debug_blocks(lens_dit* h, int first, int last, float* h_img, float* h_txt, int B, int grid_h,
                                  int grid_w, int n_txt, const float* t, void* stream) {
  if (!h || !h_img || !t || (n_txt > 0 && !h_txt)) return LENS_ERR_INVALID_ARG;
  h->ss.ready = false;
  lens_status s = check_sizes(h, B, grid_h, grid_w, n_txt);
  if (s) return s;
  if (B > h->cfg.max_timesteps) return LENS_ERR_SHAPE;
  if (first < 0 || last > h->cfg.num_blocks || first > last) return LENS_ERR_SHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  const int Ni = grid_h * grid_w;
  if ((s = compute_modulation(h, t, B, st))) return s;
  LENS_LAUNCH(h, 0, st, launch_rope_table(grid_h, grid_w, n_txt, h->rope, st));
  if ((reinterpret_cast<uintptr_t>(h_img) | reinterpret_cast<uintptr_t>(h_txt)) & 15) return LENS_ERR_INVALID_ARG;
  ActMaps am;
  if ((s = make_act_maps(h, B * Ni, B * n_txt, h_img, h_txt, am))) return s;
  for (int i = first; i < last; ++i)
    if ((s = run_block(h, i, h_img, h_txt, B, Ni, n_txt, h->mod, h->modw, am, nullptr, st))) return s;
  return LENS_OK;
}

lens_status lens_sample_euler(lens_dit* h, const uint16_t* txt_cond, const uint16_t* txt_uncond, int B, int n_txt,
                              int height_px, int width_px, int steps, float guidance, uint64_t seed,
                              float* latent_out, void* stream) {
  return lens_sample_euler_masked(h, txt_cond, nullptr, txt_uncond, nullptr, B, n_txt, height_px, width_px, steps,
                                  guidance, seed, latent_out, stream);
}

lens_status lens_sample_euler_masked(lens_dit* h, const uint16_t* txt_cond, const int* len_cond,
                                     const uint16_t* txt_uncond, const int* len_uncond, int B, int n_txt,
                                     int height_px, int width_px, int steps, float guidance, uint64_t seed,
                                     float* latent_out, void* stream) {
  lens_sampler_options o;
  lens_sampler_default_options(&o);
  o.guidance = guidance;
  return lens_sample_euler_ex(h, txt_cond, len_cond, txt_uncond, len_uncond, B, n_txt, height_px, width_px, steps,
                              &o, seed, latent_out, stream);
}

lens_status lens_sampler_default_options(lens_sampler_options* o) {
  if (!o) return LENS_ERR_INVALID_ARG;
  o->guidance = 1.0f;
  o->cfg_rescale = 0.0f;
  o->time_shift = 0;
  o->shift_mu = 0.0f;
  return LENS_OK;
}

double lens_shift_mu(int n_img_tokens, int n1, double mu1, int n2, double mu2) {
  if (n1 == n2) return NAN;
  return mu1 + (mu2 - mu1) * (double)(n_img_tokens - n1) / (double)(n2 - n1);
}

lens_status lens_time_grid(int steps, int time_shift, double mu, double* t_out) {
  if (!t_out || steps < 1 || !isfinite(mu) || fabs(mu) > 50.0) return LENS_ERR_INVALID_ARG;
  sampler_time_grid(steps, time_shift != 0, mu, t_out);
  return LENS_OK;
}

lens_status lens_sample_euler_ex(lens_dit* h, const uint16_t* txt_cond, const int* len_cond,
                                 const uint16_t* txt_uncond, const int* len_uncond, int B, int n_txt, int height_px,
                                 int width_px, int steps, const lens_sampler_options* opt, uint64_t seed,
                                 float* latent_out, void* stream) {
  if (!h || !opt || !latent_out || (n_txt > 0 && !txt_cond)) return LENS_ERR_INVALID_ARG;
  h->ss.ready = false;
  const float guidance = opt->guidance;
  if (steps < 1 || !isfinite(guidance)) return LENS_ERR_INVALID_ARG;
  if (!(opt->cfg_rescale >= 0.0f && opt->cfg_rescale <= 1.0f) || !isfinite(opt->shift_mu) ||
      fabsf(opt->shift_mu) > 50.0f)
    return LENS_ERR_INVALID_ARG;
  if (height_px <= 0 || width_px <= 0 || height_px % 16 || width_px % 16) return LENS_ERR_SHAPE;
  const bool cfg = guidance != 1.0f;
  const int gh = height_px / 16, gw = width_px / 16;
  const int Bf = cfg ? 2 * B : B;
  lens_status s = check_sizes(h, Bf, gh, gw, n_txt);
  if (s) return s;
  if (B < 1) return LENS_ERR_SHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  if (!cfg) {
    txt_uncond = nullptr;
    len_uncond = nullptr;
  }
  // valid text lengths of the forward rows: cond rows, then uncond rows
  const bool masked = len_cond || len_uncond;
  TextLengths tl;
  if (masked) {
    if (Bf > kMaxRows) return LENS_ERR_SHAPE;
    for (int b = 0; b < B; ++b) {
      const int lc = len_cond ? len_cond[b] : n_txt, lu = len_uncond ? len_uncond[b] : n_txt;
      if (lc < 0 || lc > n_txt || lu < 0 || lu > n_txt) return LENS_ERR_SHAPE;
      tl.n[b] = lc;
      if (cfg) tl.n[B + b] = lu;
    }
  }
  const TextLengths* tlp = masked ? &tl : nullptr;
  // On a created stream the call is captured once as a CUDA graph and replayed
  // while the arguments stay the same (the legacy default stream cannot capture).
  if (st == nullptr)
    return enqueue_sample(h, txt_cond, txt_uncond, B, n_txt, gh, gw, steps, *opt, seed, latent_out, tlp, st);
  lens_dit::SampleGraph& g = h->sg;
  if (g.valid && g.txt_cond == txt_cond && g.txt_uncond == txt_uncond && g.latent_out == latent_out &&
      g.stream == st && g.B == B && g.n_txt == n_txt && g.height_px == height_px && g.width_px == width_px &&
      g.steps == steps && g.guidance == guidance && g.cfg_rescale == opt->cfg_rescale &&
      g.time_shift == (opt->time_shift != 0) && g.shift_mu == opt->shift_mu && g.seed == seed &&
      g.prof_kind == h->prof_kind &&
      g.masked == masked && (!masked || memcmp(g.lens.n, tl.n, sizeof(int) * Bf) == 0)) {
    LENS_CUDA(cudaGraphLaunch(g.exec, st));
    h->launches += g.launches;
    return LENS_OK;
  }
  drop_sample_graph(h);
  const int64_t l0 = h->launches;
  if (cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return LENS_ERR_CUDA;
  s = enqueue_sample(h, txt_cond, txt_uncond, B, n_txt, gh, gw, steps, *opt, seed, latent_out, tlp, st);
  cudaGraph_t graph = nullptr;
  const cudaError_t ce = cudaStreamEndCapture(st, &graph);
  if (s != LENS_OK || ce != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    return s != LENS_OK ? s : LENS_ERR_CUDA;
  }
  cudaGraphExec_t exec = nullptr;
  if (cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
    cudaGraphDestroy(graph);
    return LENS_ERR_CUDA;
  }
  g.valid = true;
  g.txt_cond = txt_cond;
  g.txt_uncond = txt_uncond;
  g.latent_out = latent_out;
  g.stream = st;
  g.B = B;
  g.n_txt = n_txt;
  g.height_px = height_px;
  g.width_px = width_px;
  g.steps = steps;
  g.guidance = guidance;
  g.cfg_rescale = opt->cfg_rescale;
  g.time_shift = opt->time_shift != 0;
  g.shift_mu = opt->shift_mu;
  g.seed = seed;
  g.prof_kind = h->prof_kind;
  g.masked = masked;
  g.lens = tl;
  g.graph = graph;
  g.exec = exec;
  g.launches = h->launches - l0;
  LENS_CUDA(cudaGraphLaunch(exec, st));
  return LENS_OK;
}

lens_status lens_dit_profile_kernel(lens_dit* h, lens_kernel kernel, int capacity) {
  if (!h || capacity < 0) return LENS_ERR_INVALID_ARG;
  if ((int)kernel < 0 || (int)kernel > 7) return LENS_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return LENS_ERR_CUDA;
  drop_sample_graph(h);                 // a captured graph may record the old events
  for (cudaEvent_t e : h->prof_ev) cudaEventDestroy(e);
  h->prof_ev.clear();
  h->prof_kind = 0;
  h->prof_cap = 0;
  h->prof_n = 0;
  if (kernel == LENS_KERNEL_NONE || capacity == 0) return LENS_OK;
  h->prof_ev.resize(2 * (size_t)capacity);
  for (auto& e : h->prof_ev)
    if (cudaEventCreate(&e) != cudaSuccess) return LENS_ERR_CUDA;
  h->prof_kind = (int)kernel;
  h->prof_cap = capacity;
  return LENS_OK;
}

lens_status lens_dit_profile_read(lens_dit* h, int* launches, double* total_ms) {
  if (!h || !launches || !total_ms) return LENS_ERR_INVALID_ARG;
  double tot = 0;
  for (int i = 0; i < h->prof_n; ++i) {
    if (cudaEventSynchronize(h->prof_ev[2 * i + 1]) != cudaSuccess) return LENS_ERR_CUDA;
    float ms = 0;
    if (cudaEventElapsedTime(&ms, h->prof_ev[2 * i], h->prof_ev[2 * i + 1]) != cudaSuccess) return LENS_ERR_CUDA;
    tot += ms;
  }
  *launches = h->prof_n;
  *total_ms = tot;
  return LENS_OK;
}

int64_t lens_dit_launch_count(lens_dit* h) { return h ? h->launches : 0; }

lens_status lens_dit_op_timestep(lens_dit* h, const float* t, int T, float* temb, float* mod, void* stream) {
  if (!h || !t || (!temb && !mod)) return LENS_ERR_INVALID_ARG;
  if (T < 1 || T > h->cfg.max_timesteps) return LENS_ERR_SHAPE;
  h->ss.ready = false;
  cudaStream_t st = (cudaStream_t)stream;
  lens_status s = compute_modulation(h, t, T, st);
  if (s) return s;
  if (temb) LENS_CUDA(cudaMemcpyAsync(temb, h->temb, (size_t)T * kHidden * 4, cudaMemcpyDeviceToDevice, st));
  if (mod) LENS_CUDA(cudaMemcpyAsync(mod, h->mod, (size_t)T * h->modw * 4, cudaMemcpyDeviceToDevice, st));
  return LENS_OK;
}

lens_status lens_dit_op_text_input(lens_dit* h, const uint16_t* txt, int B, int n_txt, float* c, void* stream) {
  if (!h || !txt || !c) return LENS_ERR_INVALID_ARG;
  if (B < 1 || n_txt < 1 || B > h->cfg.max_batch || n_txt > h->cfg.max_txt_tokens) return LENS_ERR_SHAPE;
  h->ss.ready = false;
  cudaStream_t st = (cudaStream_t)stream;
  lens_status s = text_norm_rows(h, txt, B * n_txt, 0, st);
  if (s) return s;
  return text_in_gemm(h, B * n_txt, c, st);
}

lens_status lens_op_noise_tokens(uint64_t seed, int B, int grid_h, int grid_w, float* tokens, void* stream) {
  if (!tokens) return LENS_ERR_INVALID_ARG;
  if (B < 1 || grid_h < 1 || grid_w < 1) return LENS_ERR_SHAPE;
  LENS_CUDA(launch_noise_tokens(seed, B, grid_h, grid_w, tokens, (cudaStream_t)stream));
  return LENS_OK;
}

lens_status lens_op_patchify(const float* latent, int B, int grid_h, int grid_w, float* tokens, void* stream) {
  if (!latent || !tokens) return LENS_ERR_INVALID_ARG;
  if (B < 1 || grid_h < 1 || grid_w < 1) return LENS_ERR_SHAPE;
  LENS_CUDA(launch_patchify(latent, B, grid_h, grid_w, tokens, (cudaStream_t)stream));
  return LENS_OK;
}

lens_status lens_op_unpatchify(const float* tokens, int B, int grid_h, int grid_w, float* latent, void* stream) {
  if (!latent || !tokens) return LENS_ERR_INVALID_ARG;
  if (B < 1 || grid_h < 1 || grid_w < 1) return LENS_ERR_SHAPE;
  LENS_CUDA(launch_unpatchify(tokens, B, grid_h, grid_w, latent, (cudaStream_t)stream));
  return LENS_OK;
}

lens_status lens_op_rope_table(int grid_h, int grid_w, int n_txt, float* cos_sin, void* stream) {
  if (!cos_sin) return LENS_ERR_INVALID_ARG;
  if (grid_h < 1 || grid_w < 1 || n_txt < 0) return LENS_ERR_SHAPE;
  LENS_CUDA(launch_rope_table(grid_h, grid_w, n_txt, reinterpret_cast<float2*>(cos_sin), (cudaStream_t)stream));
  return LENS_OK;
}

lens_status lens_op_rmsnorm_modulate(const float* x, int M, int rows_per_batch, const float* shift,
                                     const float* scale, int64_t mod_stride, float eps, uint16_t* y, void* stream) {
  if (!x || !shift || !scale || !y) return LENS_ERR_INVALID_ARG;
  if (M < 1 || rows_per_batch < 1 || mod_stride < 0 || mod_stride % 4) return LENS_ERR_SHAPE;
  if (!(eps > 0.f)) return LENS_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(shift) | reinterpret_cast<uintptr_t>(scale) |
       reinterpret_cast<uintptr_t>(y)) & 15)
    return LENS_ERR_INVALID_ARG;
  LENS_CUDA(launch_rmsnorm_modulate(x, M, rows_per_batch, shift, scale, mod_stride, eps,
                                    reinterpret_cast<__nv_bfloat16*>(y), (cudaStream_t)stream));
  return LENS_OK;
}

lens_status lens_op_quantize_w4(const uint16_t* w, int64_t rows, int64_t k, uint8_t* codes, uint32_t* scales,
                                void* stream) {
  if (!w || !codes || !scales) return LENS_ERR_INVALID_ARG;
  if (rows < 1 || k < 64 || k % 64) return LENS_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(codes) & 15) return LENS_ERR_INVALID_ARG;
  LENS_CUDA(launch_quantize_w4(w, rows, k, codes, scales, rows, (cudaStream_t)stream));
  return LENS_OK;
}

lens_status lens_op_gemm_w4(const uint16_t* A, const uint8_t* codes, const uint32_t* scales, const float* bias,
                            float* C, int M, int N, int K, void* stream) {
  if (!A || !codes || !scales || !C) return LENS_ERR_INVALID_ARG;
  if (M < 1 || N < 128 || K < 64 || K % 64 || N % 128) return LENS_ERR_SHAPE;
  const int bn = N % 256 == 0 ? 256 : 128;
  const int bm = bn == 128 && M >= 256 ? 256 : 128;   // 256-row tiles with the 128-wide B tile
  CUtensorMap ta, tq, ts, tc;
  if (!encode_tmap_bf16(&ta, A, M, K, K, 128) || !encode_tmap_w4_codes(&tq, codes, N, K, bn) ||
      !encode_tmap_w4_scales(&ts, scales, N, K, bn) || !encode_tmap_out(&tc, C, 4, M, N, N))
    return LENS_ERR_INVALID_ARG;
  int* err = op_err_ptr();
  if (!err) return LENS_ERR_CUDA;
  GemmArgs a = make_args(err);
  a.num_problems = 1;
  a.p[0] = base_problem(M, N, K);
  a.p[0].out_f32 = C;
  a.p[0].ld_out = N;
  a.p[0].bias = bias;
  LENS_CUDA(launch_gemm_w4(bm, bn, EPI_F32, false, &ta, nullptr, &tq, &ts, nullptr, nullptr, nullptr, nullptr, &tc,
                           nullptr, a, device_sms(), (cudaStream_t)stream));
  return LENS_OK;
}

lens_status lens_op_gemm_bf16(const uint16_t* A, const uint16_t* Bm, const float* bias, float* C, int M, int N,
                              int K, void* stream) {
  if (!A || !Bm || !C) return LENS_ERR_INVALID_ARG;
  if (M < 1 || N < 32 || K < 64 || K % 64 || N % 32) return LENS_ERR_SHAPE;
  const int bn = N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : (N % 64 == 0 ? 64 : 32));
  const bool pair = M >= 256 && bn >= 128;     // CTA pairs when a 256-row tile is not mostly padding
  CUtensorMap ta, tb;
  if (!encode_tmap_bf16(&ta, A, M, K, K, 128) || !encode_tmap_bf16(&tb, Bm, N, K, K, pair ? bn / 2 : bn))
    return LENS_ERR_INVALID_ARG;
  CUtensorMap tc;
  if (!encode_tmap_out(&tc, C, 4, M, N, N)) return LENS_ERR_INVALID_ARG;
  int* err = op_err_ptr();
  if (!err) return LENS_ERR_CUDA;
  GemmArgs a = make_args(err);
  a.num_problems = 1;
  a.p[0] = base_problem(M, N, K);
  a.p[0].out_f32 = C;
  a.p[0].ld_out = N;
  a.p[0].bias = bias;
  if (pair)
    LENS_CUDA(launch_gemm_pair(bn, EPI_F32, &ta, &tb, nullptr, nullptr, &tc, nullptr, a, device_sms(),
                               (cudaStream_t)stream));
  else
    LENS_CUDA(launch_gemm(bn, EPI_F32, &ta, &tb, nullptr, nullptr, &tc, nullptr, a, device_sms(),
                          (cudaStream_t)stream));
  return LENS_OK;
}

lens_status lens_op_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int n_txt, int n_img,
                              uint16_t* out_txt, uint16_t* out_img, void* stream) {
  return lens_op_attention_masked(q, k, v, B, n_txt, n_img, nullptr, out_txt, out_img, stream);
}

lens_status lens_op_attention_masked(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int n_txt,
                                     int n_img, const int* txt_len, uint16_t* out_txt, uint16_t* out_img,
                                     void* stream) {
  if (!q || !k || !v || (n_txt > 0 && !out_txt) || (n_img > 0 && !out_img)) return LENS_ERR_INVALID_ARG;
  TextLengths tl;
  if (txt_len) {
    if (B > kMaxRows) return LENS_ERR_SHAPE;
    for (int b = 0; b < B; ++b) {
      if (txt_len[b] < 0 || txt_len[b] > n_txt) return LENS_ERR_SHAPE;
      tl.n[b] = txt_len[b];
    }
  }
  if (B < 1 || n_txt < 0 || n_img < 0 || n_txt + n_img < 1) return LENS_ERR_SHAPE;
  // a batch row with no image token and no valid text token has no key to attend:
  // its softmax is undefined, so the call is refused
  if (txt_len && n_img == 0)
    for (int b = 0; b < B; ++b)
      if (txt_len[b] == 0) return LENS_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15)
    return LENS_ERR_INVALID_ARG;
  int* err = op_err_ptr();
  if (!err) return LENS_ERR_CUDA;
  LENS_CUDA(launch_joint_attention(
      reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(k),
      reinterpret_cast<const __nv_bfloat16*>(v), B, kHeads, n_txt, n_img, reinterpret_cast<__nv_bfloat16*>(out_txt),
      reinterpret_cast<__nv_bfloat16*>(out_img), txt_len ? &tl : nullptr, err, (cudaStream_t)stream));
  return LENS_OK;
}

// ------------------------------------------------------------ step-wise sampler
static lens_status check_options(const lens_sampler_options* o) {
  if (!o || !isfinite(o->guidance)) return LENS_ERR_INVALID_ARG;
  if (!(o->cfg_rescale >= 0.0f && o->cfg_rescale <= 1.0f) || !isfinite(o->shift_mu) || fabsf(o->shift_mu) > 50.0f)
    return LENS_ERR_INVALID_ARG;
  return LENS_OK;
}

lens_status lens_sampler_prepare(lens_dit* h, const uint16_t* txt, const int* txt_len, int B, int n_txt,
                                 int height_px, int width_px, int steps, const lens_sampler_options* opt,
                                 uint64_t seed, void* stream) {
  if (!h) return LENS_ERR_INVALID_ARG;
  h->ss.ready = false;
  lens_status s = check_options(opt);
  if (s) return s;
  if (steps < 1) return LENS_ERR_INVALID_ARG;
  if (height_px <= 0 || width_px <= 0 || height_px % 16 || width_px % 16) return LENS_ERR_SHAPE;
  const int gh = height_px / 16, gw = width_px / 16, Ni = gh * gw;
  if ((s = check_sizes(h, B, gh, gw, n_txt))) return s;
  if (steps > h->cfg.max_timesteps) return LENS_ERR_SHAPE;
  lens_dit::StepSampler& ss = h->ss;
  ss.masked = txt_len != nullptr;
  if (ss.masked) {
    if (B > kMaxRows) return LENS_ERR_SHAPE;
    for (int b = 0; b < B; ++b) {
      if (txt_len[b] < 0 || txt_len[b] > n_txt) return LENS_ERR_SHAPE;
      ss.tl.n[b] = txt_len[b];
    }
  }
  cudaStream_t st = (cudaStream_t)stream;
  sampler_time_grid(steps, opt->time_shift != 0, opt->shift_mu, ss.grid);
  LENS_LAUNCH(h, 0, st, launch_noise_tokens(seed, B, gh, gw, h->xtok, st));
  LENS_LAUNCH(h, 0, st, launch_tokens_to_operand(h->xtok, (int64_t)B * Ni, 1, (int64_t)B * Ni, h->xin, st));
  if ((s = text_norm_rows(h, txt, B * n_txt, 0, st))) return s;     // NULL text: zeros
  if ((s = text_in_gemm(h, B * n_txt, h->h_txt0, st))) return s;
  float tv[kMaxTimesteps];
  for (int k = 0; k < steps; ++k) tv[k] = (float)ss.grid[k];
  if ((s = compute_modulation(h, tv, steps, st))) return s;
  ss.B = B;
  ss.gh = gh;
  ss.gw = gw;
  ss.n_txt = n_txt;
  ss.steps = steps;
  ss.opt = *opt;
  ss.ready = true;
  return LENS_OK;
}

lens_status lens_sampler_velocity(lens_dit* h, int k, float* v_out, void* stream) {
  if (!h || !v_out || !h->ss.ready) return LENS_ERR_INVALID_ARG;
  const lens_dit::StepSampler& ss = h->ss;
  if (k < 0 || k >= ss.steps) return LENS_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(v_out) & 15) return LENS_ERR_INVALID_ARG;
  return run_forward_core(h, ss.B, ss.gh, ss.gw, ss.n_txt, h->mod + (int64_t)k * h->modw, 0, v_out,
                          ss.masked ? &ss.tl : nullptr, (cudaStream_t)stream);
}

lens_status lens_sampler_update(lens_dit* h, int k, const float* v_cond, const float* v_uncond, void* stream) {
  if (!h || !v_cond || !h->ss.ready) return LENS_ERR_INVALID_ARG;
  const lens_dit::StepSampler& ss = h->ss;
  if (k < 0 || k >= ss.steps) return LENS_ERR_SHAPE;
  const float g = ss.opt.guidance;
  const bool cfg = g != 1.0f;
  if (cfg && !v_uncond) return LENS_ERR_INVALID_ARG;
  const bool shift = ss.opt.time_shift != 0;
  const float dt = shift ? (float)(ss.grid[k] - ss.grid[k + 1]) : 1.0f / (float)ss.steps;
  const int64_t per_sample = (int64_t)ss.gh * ss.gw * kInCh;
  cudaStream_t st = (cudaStream_t)stream;
  if (cfg && ss.opt.cfg_rescale != 0.0f) {
    LENS_LAUNCH(h, 0, st, launch_cfg_norm_partials(v_cond, v_uncond, per_sample, ss.B, g, h->cfgpart, st));
    LENS_LAUNCH(h, 0, st, launch_euler_cfg_rescaled(h->xtok, v_cond, v_uncond, per_sample, ss.B, dt, g,
                                                    ss.opt.cfg_rescale, h->cfgpart, h->xin, 1, st));
  } else {
    LENS_LAUNCH(h, 0, st, launch_euler_step(h->xtok, v_cond, cfg ? v_uncond : nullptr, per_sample * ss.B, dt, g,
                                            h->xin, st));
  }
  return LENS_OK;
}

lens_status lens_sampler_finish(lens_dit* h, float* latent_out, void* stream) {
  if (!h || !latent_out || !h->ss.ready) return LENS_ERR_INVALID_ARG;
  const lens_dit::StepSampler& ss = h->ss;
  cudaStream_t st = (cudaStream_t)stream;
  LENS_LAUNCH(h, 0, st, launch_unpatchify(h->xtok, ss.B, ss.gh, ss.gw, latent_out, st));
  return LENS_OK;
}

lens_status lens_dit_op_euler_cfg_rescaled(lens_dit* h, float* x, const float* v_cond, const float* v_uncond, int B,
                                           int64_t per_sample, float dt, float guidance, float phi, void* stream) {
  if (!h || !x || !v_cond || !v_uncond) return LENS_ERR_INVALID_ARG;
  if (!isfinite(dt) || !isfinite(guidance) || !(phi >= 0.0f && phi <= 1.0f)) return LENS_ERR_INVALID_ARG;
  if (B < 1 || B > h->cfg.max_batch || per_sample < 1) return LENS_ERR_SHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  LENS_LAUNCH(h, 0, st, launch_cfg_norm_partials(v_cond, v_uncond, per_sample, B, guidance, h->cfgpart, st));
  LENS_LAUNCH(h, 0, st, launch_euler_cfg_rescaled(x, v_cond, v_uncond, per_sample, B, dt, guidance, phi, h->cfgpart,
                                                  nullptr, 1, st));
  return LENS_OK;
}

lens_status lens_op_euler_cfg(float* x, const float* v_cond, const float* v_uncond, int64_t n, float dt,
                              float guidance, void* stream) {
  if (!x || !v_cond) return LENS_ERR_INVALID_ARG;
  if (n < 1) return LENS_ERR_SHAPE;
  if (!isfinite(dt) || !isfinite(guidance)) return LENS_ERR_INVALID_ARG;
  LENS_CUDA(launch_euler_plain(x, v_cond, v_uncond, n, dt, guidance, (cudaStream_t)stream));
  return LENS_OK;
}

}  // extern "C"
