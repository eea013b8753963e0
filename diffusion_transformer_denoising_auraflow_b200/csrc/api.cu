// api.cu -- the C ABI (include/af.h): weight pack, scratch, block and forward
// orchestration.  Every compute step runs in this library's kernels
// (gemm.cu, attention.cu, kernels.cu); this file only checks arguments,
// lays out memory and sequences launches on the caller's stream.
//
// Sequencing follows "Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级
// 使用指南", §前向传播流程 (embed -> joint blocks -> cat(text, image) ->
// single blocks -> image slice -> pre-final -> proj_out -> unpatchify), with
// the block internals of §联合注意力块 / §单 DiT 块.
#include <array>
#include <cstdio>
#include <cstring>
#include <string>
#include <unordered_map>
#include <vector>

#include "af.h"
#include "af_internal.h"

using namespace af;

namespace {

thread_local std::string g_last_error;

af_status cuda_fail(cudaError_t e) {
  g_last_error = cudaGetErrorString(e);
  return AF_ERR_CUDA;
}

#define AF_CUDA(x)                              \
  do {                                          \
    cudaError_t e_ = (x);                       \
    if (e_ != cudaSuccess) return cuda_fail(e_); \
  } while (0)

int isqrt_exact(int n) {
  int g = 0;
  while ((g + 1) * (g + 1) <= n) ++g;
  return g * g == n ? g : -1;
}

int find_multiple(int n, int k) { return n % k == 0 ? n : n + k - n % k; }

struct Derived {
  int D, F, G, H, hd;
};

af_status derive(const af_config* c, Derived* d) {
  if (!c) return AF_ERR_INVALID_ARG;
  if (c->patch_size <= 0 || c->in_channels <= 0 || c->out_channels <= 0 || c->num_mmdit_layers < 0 ||
      c->num_single_dit_layers < 0 || c->attention_head_dim <= 0 || c->num_attention_heads <= 0 ||
      c->joint_attention_dim <= 0 || c->pos_embed_max_size <= 0 || c->num_register_tokens < 0 ||
      c->timestep_channels <= 0 || c->timestep_channels % 2 != 0 || c->ffn_inner < 0 || !(c->ln_eps >= 0.f))
    return AF_ERR_INVALID_ARG;
  d->H = c->num_attention_heads;
  d->hd = c->attention_head_dim;
  d->D = d->H * d->hd;
  d->F = c->ffn_inner > 0 ? c->ffn_inner : find_multiple(static_cast<int>(2.0 * (4.0 * d->D) / 3.0), 256);
  d->G = isqrt_exact(c->pos_embed_max_size);
  if (d->G <= 0) return AF_ERR_INVALID_ARG;
  return AF_OK;
}

struct TensorInfo {
  std::string name;
  int ndim;
  int64_t shape[2];
  size_t offset;  // bytes into the pack
  // FFN up-projection pairs (linear_1, linear_2) are stored interleaved in
  // 128-row groups, [W1 g | W2 g] for g = 0, 1, ..., so one 256-row tile of
  // the pair feeds both halves of the SwiGLU epilogue: 1 = W1, 2 = W2.
  int interleave = 0;
  size_t pair_base = 0;
  size_t numel() const { return ndim == 1 ? shape[0] : static_cast<size_t>(shape[0]) * shape[1]; }
};

}  // namespace

struct af_weights {
  af_config cfg;
  Derived d;
  int device;
  bool f32 = false;  // AF_DTYPE_F32 pack: fp32 tensors, fp32 forward (fp32.cu)
  size_t esz = 2;    // bytes per stored element
  uint8_t* base = nullptr;
  size_t bytes = 0;
  std::vector<TensorInfo> tensors;
  std::unordered_map<std::string, int> index;
  // adaLN region: rows of every modulation linear, contiguous, in unit order
  size_t ada_rows = 0;
  std::vector<size_t> unit_row;  // first row of unit u (joint i: 2i img, 2i+1 txt; single j: 2J + j)
  size_t pf_row = 0;             // first row of norm_out
  // 8-bit variant: e4m3 copies of every block projection's weight (fused
  // QKV, output projection, FFN up pair, FFN down) with one fp32 scale per
  // row (af_weights_quantize_fp8).  Each region's scales start at a multiple
  // of 256 rows, so every scale a 256-column tile can touch exists.
  struct Fp8Region {
    size_t code_off;   // bytes into fp8_codes
    size_t scale_off;  // entries into fp8_scales
  };
  bool fp8 = false;
  uint8_t* fp8_codes = nullptr;
  float* fp8_scales = nullptr;
  std::unordered_map<std::string, Fp8Region> fp8_region;  // region's first tensor name -> offsets

  const uint16_t* ptr(const std::string& n) const {
    auto it = index.find(n);
    return it == index.end() ? nullptr : reinterpret_cast<const uint16_t*>(base + tensors[it->second].offset);
  }
  const float* ptrf(const std::string& n) const { return reinterpret_cast<const float*>(ptr(n)); }
};

struct af_scratch {
  const af_weights* w;
  int max_b, max_ni, max_l, max_nt, max_n;
  int device;
  uint8_t* base = nullptr;
  size_t bytes = 0;
  int* err;
  float *temb, *h1, *mods, *tfeat;
  uint16_t *y, *q, *k, *v, *o, *h;
  uint8_t* y8;    // 8-bit variant: e4m3 codes of y, one fp32 scale per row in yscale
  float* yscale;
  uint16_t *img, *txt, *x;   // (fp32 pack: these activation buffers hold floats)
  float* tmp;                // fp32 pack: GEMM outputs before QK-norm / SwiGLU, [B*N, max(3D, 2F)]
  uint16_t* wfold;           // output stage: proj_out * (1 + scale_b), [B, 256, D] bf16 (rows >= p*p*C zero)
  float *obias, *oproj;      // output stage: W . shift_b [B, 64]; projected tokens [B * Ni, p*p*C] fp32
  float *lat2, *vel, *tvec;  // denoise step: CFG-duplicated latents, velocity, model times
  int sms;
  // launch accounting / profiling (kernel classes: GEMM, attention, LN, other)
  int64_t launches[AF_NUM_KERNEL_CLASSES] = {0, 0, 0, 0};
  bool profiling = false;
  std::vector<cudaEvent_t> pool;
  size_t pool_used = 0;
  struct Rec {
    int cls;
    size_t e0;
    int n;
    double work;
  };
  std::vector<Rec> recs;
};

namespace {

void add_tensor(af_weights* w, size_t& off, const std::string& name, int64_t r, int64_t c, bool align = true) {
  if (align) off = (off + 255) & ~size_t(255);
  TensorInfo t;
  t.name = name;
  t.ndim = c > 0 ? 2 : 1;
  t.shape[0] = r;
  t.shape[1] = c > 0 ? c : 0;
  t.offset = off;
  w->index[name] = static_cast<int>(w->tensors.size());
  w->tensors.push_back(t);
  off += t.numel() * w->esz;
}

void mark_pair(af_weights* w, const std::string& w1, const std::string& w2) {
  TensorInfo& a = w->tensors[w->index[w1]];
  TensorInfo& b = w->tensors[w->index[w2]];
  a.interleave = 1;
  b.interleave = 2;
  a.pair_base = b.pair_base = a.offset;
}

void build_layout(af_weights* w) {
  const af_config& c = w->cfg;
  const int D = w->d.D, F = w->d.F, p = c.patch_size;
  size_t off = 0;
  // adaLN-Zero / pre-final linears, one contiguous [rows, D] matrix
  size_t row = 0;
  w->unit_row.clear();
  for (int i = 0; i < c.num_mmdit_layers; ++i) {
    const std::string b = "joint_transformer_blocks." + std::to_string(i) + ".";
    w->unit_row.push_back(row);
    add_tensor(w, off, b + "norm1.linear.weight", 6 * D, D, row == 0);
    row += 6 * D;
    w->unit_row.push_back(row);
    add_tensor(w, off, b + "norm1_context.linear.weight", 6 * D, D, false);
    row += 6 * D;
  }
  for (int i = 0; i < c.num_single_dit_layers; ++i) {
    w->unit_row.push_back(row);
    add_tensor(w, off, "single_transformer_blocks." + std::to_string(i) + ".norm1.linear.weight", 6 * D, D,
               row == 0);
    row += 6 * D;
  }
  w->pf_row = row;
  add_tensor(w, off, "norm_out.linear.weight", 2 * D, D, row == 0);
  row += 2 * D;
  w->ada_rows = row;
  // blocks: q,k,v contiguous (fused QKV), linear_1, linear_2 contiguous (SwiGLU up)
  for (int i = 0; i < c.num_mmdit_layers; ++i) {
    const std::string b = "joint_transformer_blocks." + std::to_string(i) + ".";
    add_tensor(w, off, b + "attn.to_q.weight", D, D);
    add_tensor(w, off, b + "attn.to_k.weight", D, D, false);
    add_tensor(w, off, b + "attn.to_v.weight", D, D, false);
    add_tensor(w, off, b + "attn.add_q_proj.weight", D, D);
    add_tensor(w, off, b + "attn.add_k_proj.weight", D, D, false);
    add_tensor(w, off, b + "attn.add_v_proj.weight", D, D, false);
    add_tensor(w, off, b + "attn.to_out.0.weight", D, D);
    add_tensor(w, off, b + "attn.to_add_out.weight", D, D);
    add_tensor(w, off, b + "ff.linear_1.weight", F, D);
    add_tensor(w, off, b + "ff.linear_2.weight", F, D, false);
    add_tensor(w, off, b + "ff.out_projection.weight", D, F);
    add_tensor(w, off, b + "ff_context.linear_1.weight", F, D);
    add_tensor(w, off, b + "ff_context.linear_2.weight", F, D, false);
    add_tensor(w, off, b + "ff_context.out_projection.weight", D, F);
    if (!w->f32) {  // the fp32 forward multiplies by [linear_1; linear_2] as stored
      mark_pair(w, b + "ff.linear_1.weight", b + "ff.linear_2.weight");
      mark_pair(w, b + "ff_context.linear_1.weight", b + "ff_context.linear_2.weight");
    }
  }
  for (int i = 0; i < c.num_single_dit_layers; ++i) {
    const std::string b = "single_transformer_blocks." + std::to_string(i) + ".";
    add_tensor(w, off, b + "attn.to_q.weight", D, D);
    add_tensor(w, off, b + "attn.to_k.weight", D, D, false);
    add_tensor(w, off, b + "attn.to_v.weight", D, D, false);
    add_tensor(w, off, b + "attn.to_out.0.weight", D, D);
    add_tensor(w, off, b + "ff.linear_1.weight", F, D);
    add_tensor(w, off, b + "ff.linear_2.weight", F, D, false);
    add_tensor(w, off, b + "ff.out_projection.weight", D, F);
    if (!w->f32) mark_pair(w, b + "ff.linear_1.weight", b + "ff.linear_2.weight");
  }
  add_tensor(w, off, "pos_embed.proj.weight", D, p * p * c.in_channels);
  add_tensor(w, off, "pos_embed.pos_embed", c.pos_embed_max_size, D);
  add_tensor(w, off, "time_step_proj.linear_1.weight", D, c.timestep_channels);
  add_tensor(w, off, "time_step_proj.linear_1.bias", D, 0);
  add_tensor(w, off, "time_step_proj.linear_2.weight", D, D);
  add_tensor(w, off, "time_step_proj.linear_2.bias", D, 0);
  add_tensor(w, off, "context_embedder.weight", D, c.joint_attention_dim);
  add_tensor(w, off, "register_tokens", c.num_register_tokens, D);
  add_tensor(w, off, "proj_out.weight", p * p * c.out_channels, D);
  w->bytes = (off + 255) & ~size_t(255);
}

const uint16_t* ada_base(const af_weights* w) {
  return reinterpret_cast<const uint16_t*>(w->base + w->tensors[0].offset);
}

// Kernels launch on the current device, so it must be the pack's.
af_status check_device(const af_weights* w) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    g_last_error = cudaGetErrorString(cudaGetLastError());
    return AF_ERR_CUDA;
  }
  if (dev != w->device) {
    g_last_error = "the current device (" + std::to_string(dev) + ") is not the weight pack's device (" +
                   std::to_string(w->device) + ")";
    return AF_ERR_INVALID_ARG;
  }
  return AF_OK;
}

af_status check_scratch(const af_weights* w, af_scratch* s) {
  if (!w || !s || s->w != w) return AF_ERR_INVALID_ARG;
  return check_device(w);
}

enum { KC_GEMM = 0, KC_ATTN = 1, KC_LN = 2, KC_OTHER = 3 };

// Counts the launches made inside its scope and, while profiling, brackets
// them with a CUDA event pair on `st`.
struct LaunchScope {
  af_scratch* s;
  cudaStream_t st;
  size_t e0 = SIZE_MAX;
  LaunchScope(af_scratch* s_, int cls, double work, cudaStream_t st_, int n = 1) : s(s_), st(st_) {
    s->launches[cls] += n;
    if (!s->profiling) return;
    while (s->pool.size() < s->pool_used + 2) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return;
      s->pool.push_back(e);
    }
    e0 = s->pool_used;
    s->pool_used += 2;
    cudaEventRecord(s->pool[e0], st);
    s->recs.push_back({cls, e0, n, work});
  }
  ~LaunchScope() {
    if (e0 != SIZE_MAX) cudaEventRecord(s->pool[e0 + 1], st);
  }
};

// ---------------------------------------------------------------- GEMM helpers
GemmParams gemm_base(const af_scratch* s, int M, int N, int K, int mode, int rows_per_batch) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.K = K;
  p.mode = mode;
  p.rows_per_batch = rows_per_batch > 0 ? rows_per_batch : (M > 0 ? M : 1);
  p.out_rows_per_batch = p.rows_per_batch;
  p.out_row_off = 0;
  p.err = s->err;
  return p;
}

af_status run_gemm(af_scratch* s, const GemmParams& p, const void* A, const void* W, int W_rows,
                   cudaStream_t st) {
  const double ncols = p.mode == EPI_SWIGLU ? 2.0 * p.N : static_cast<double>(p.N);
  LaunchScope ls(s, KC_GEMM, 2.0 * p.M * ncols * p.K, st);
  cudaError_t e = launch_gemm(p, A, W, W_rows, st, s->sms);
  if (e != cudaSuccess) return cuda_fail(e);
  return AF_OK;
}

// A GEMM operand: bf16 (scale == nullptr) or e4m3 codes with one fp32 scale per row.
struct Operand {
  const void* ptr;
  const float* scale;
};

// The weight region starting at tensor `name` as the GEMM reads it.
Operand weight_op(const af_weights* w, const std::string& name) {
  if (w->fp8) {
    auto it = w->fp8_region.find(name);
    if (it != w->fp8_region.end())
      return {w->fp8_codes + it->second.code_off, w->fp8_scales + it->second.scale_off};
  }
  return {w->ptr(name), nullptr};
}

// A tensor-core GEMM call: parameters, operands and the weight rows the
// tensor map spans.
struct GemmCall {
  GemmParams p;
  const void* A;
  const void* W;
  int W_rows;
  bool ok;  // operand types agree (both bf16 or both e4m3)
};

// QKV projection of one stream with per-head LayerNorm of Q and K.
GemmCall qkv_call(const af_weights* w, af_scratch* s, Operand y, int B, int rows, Operand wqkv, int row_off,
                  int n_total) {
  const Derived& d = w->d;
  GemmParams p = gemm_base(s, B * rows, 3 * d.D, d.D, EPI_QKV, rows);
  p.q = s->q;
  p.k = s->k;
  p.v = s->v;
  p.heads = d.H;
  p.hd = d.hd;
  p.n_total = n_total;
  p.qkv_row_off = row_off;
  p.D = d.D;
  p.eps = w->cfg.ln_eps;
  p.a_scale = y.scale;
  p.w_scale = wqkv.scale;
  return {p, y.ptr, wqkv.ptr, 3 * d.D, (y.scale != nullptr) == (wqkv.scale != nullptr)};
}

// x += gate[b] * (A W^T)
GemmCall gres_call(af_scratch* s, Operand A, int B, int rows, int K, Operand W, int N, uint16_t* x,
                   const float* gate, int gate_stride) {
  GemmParams p = gemm_base(s, B * rows, N, K, EPI_GATE_RES, rows);
  p.out = x;
  p.ldo = N;
  p.gate = gate;
  p.gate_stride = gate_stride;
  p.a_scale = A.scale;
  p.w_scale = W.scale;
  return {p, A.ptr, W.ptr, N, (A.scale != nullptr) == (W.scale != nullptr)};
}

// h = silu(y W1^T) * (y W2^T), W1 and W2 interleaved in 128-row groups ([2F, D])
GemmCall swiglu_call(const af_weights* w, af_scratch* s, Operand y, int M, Operand w12, uint16_t* h) {
  const Derived& d = w->d;
  GemmParams p = gemm_base(s, M, d.F, d.D, EPI_SWIGLU, M);
  p.out = h;
  p.ldo = d.F;
  p.a_scale = y.scale;
  p.w_scale = w12.scale;
  return {p, y.ptr, w12.ptr, 2 * d.F, (y.scale != nullptr) == (w12.scale != nullptr)};
}

double gemm_flops(const GemmParams& p) {
  const double ncols = p.mode == EPI_SWIGLU ? 2.0 * p.N : static_cast<double>(p.N);
  return 2.0 * p.M * ncols * p.K;
}

af_status run_call(af_scratch* s, const GemmCall& c, cudaStream_t st) {
  if (!c.ok) return AF_ERR_UNSUPPORTED;
  return run_gemm(s, c.p, c.A, c.W, c.W_rows, st);
}

// Two independent projections (the joint block's image and text streams) in
// one persistent launch: the text tiles fill the image GEMM's last wave.
af_status run_calls_grouped(af_scratch* s, const GemmCall& a, const GemmCall& b, cudaStream_t st) {
  if (!a.ok || !b.ok) return AF_ERR_UNSUPPORTED;
  LaunchScope ls(s, KC_GEMM, gemm_flops(a.p) + gemm_flops(b.p), st);
  cudaError_t e = launch_gemm_grouped(a.p, a.A, a.W, a.W_rows, b.p, b.A, b.W, b.W_rows, st, s->sms);
  return e == cudaSuccess ? AF_OK : cuda_fail(e);
}

af_status qkv(const af_weights* w, af_scratch* s, Operand y, int B, int rows, Operand wqkv, int row_off,
              int n_total, cudaStream_t st) {
  return run_call(s, qkv_call(w, s, y, B, rows, wqkv, row_off, n_total), st);
}

af_status gated_residual(af_scratch* s, Operand A, int B, int rows, int K, Operand W, int N, uint16_t* x,
                         const float* gate, int gate_stride, cudaStream_t st) {
  return run_call(s, gres_call(s, A, B, rows, K, W, N, x, gate, gate_stride), st);
}

// The 8-bit variant's per-token quantisation of a bf16 activation [rows, K]
// (attention output, SwiGLU product) into e4m3 codes + row scales.
af_status quantize_act(af_scratch* s, const uint16_t* x, int rows, int K, uint8_t* q, float* scale, cudaStream_t st) {
  LaunchScope ls(s, KC_LN, 3.0 * rows * K, st);
  cudaError_t e = launch_quantize_rows_e4m3(x, rows, K, q, scale, st);
  return e == cudaSuccess ? AF_OK : cuda_fail(e);
}

af_status swiglu(const af_weights* w, af_scratch* s, Operand y, int M, Operand w12, uint16_t* h, cudaStream_t st) {
  return run_call(s, swiglu_call(w, s, y, M, w12, h), st);
}

// Padding of the text part: for sample b the keys [base + len[b], end) are
// masked (len == nullptr: no mask).
struct KeyMask {
  const int* len = nullptr;
  int base = 0, end = 0;
};

KeyMask text_mask(const af_weights* w, const int* text_len, int Nt) {
  KeyMask m;
  if (text_len) {
    m.len = text_len;
    m.base = w->cfg.num_register_tokens;
    m.end = Nt;
  }
  return m;
}

af_status attention(const af_weights* w, af_scratch* s, int B, int N, uint16_t* out_a, uint16_t* out_b, int split,
                    const KeyMask& km, cudaStream_t st) {
  const Derived& d = w->d;
  AttnParams p;
  p.B = B;
  p.H = d.H;
  p.N = N;
  p.hd = d.hd;
  p.out_a = out_a;
  p.out_b = out_b;
  p.split = split;
  p.ldo = d.D;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(d.hd));
  p.qk_normalized = 1;  // q and k come from the QK-norm epilogue of the QKV GEMM
  p.err = s->err;
  p.key_len = km.len;
  p.key_base = km.base;
  p.key_end = km.end;
  LaunchScope ls(s, KC_ATTN, 4.0 * B * d.H * static_cast<double>(N) * N * d.hd, st);
  p.q = s->q;
  cudaError_t e = launch_attention(p, s->q, s->k, s->v, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return AF_OK;
}

// LayerNorm + modulate of `rows` rows into y (bf16), or into e4m3 codes y8 +
// row scales ys when y8 != nullptr.
af_status ln_mod(af_scratch* s, const uint16_t* x, const float* shift, const float* scale, int mod_stride, uint16_t* y,
                 int rows, int rows_per_batch, int D, float eps, cudaStream_t st, uint8_t* y8 = nullptr,
                 float* ys = nullptr) {
  LaunchScope ls(s, KC_LN, (y8 ? 3.0 : 4.0) * rows * D, st);
  cudaError_t e = launch_ln_modulate(x, shift, scale, mod_stride, y, rows, rows_per_batch, D, eps, st, s->err, y8, ys);
  return e == cudaSuccess ? AF_OK : cuda_fail(e);
}

// The joint block's image and text LayerNorms in one launch: shift at m, scale
// at m + D of each stream's modulation rows (same layout rules as ln_mod).
af_status ln_mod2(af_scratch* s, const uint16_t* xi, const float* mi, uint16_t* yi, uint8_t* yi8, float* ysi,
                  int Ni, const uint16_t* xt, const float* mt, uint16_t* yt, uint8_t* yt8, float* yst, int Nt,
                  int B, int mod_stride, int D, float eps, cudaStream_t st) {
  LaunchScope ls(s, KC_LN, (yi8 ? 3.0 : 4.0) * B * (Ni + Nt) * D, st);
  const LnSegment g0{xi, mi, mi + D, yi, yi8, ysi, Ni, B, 0};
  const LnSegment g1{xt, mt, mt + D, yt, yt8, yst, Nt, Nt > 0 ? B : 0, 0};
  cudaError_t e = launch_ln_modulate_pair(g0, g1, mod_stride, D, eps, st, s->err);
  return e == cudaSuccess ? AF_OK : cuda_fail(e);
}

#define AF_TRY(x)                  \
  do {                             \
    af_status st_ = (x);           \
    if (st_ != AF_OK) return st_;  \
  } while (0)

// One joint block given the modulation vectors of both streams (mods rows
// [unit_row, +6D) per sample, sample stride mod_stride).
af_status joint_block_impl(const af_weights* w, af_scratch* s, int layer, uint16_t* img, uint16_t* txt,
                           const float* mi, const float* mt, int mod_stride, int B, int Ni, int Nt,
                           const KeyMask& km, cudaStream_t st) {
  const Derived& d = w->d;
  const int D = d.D;
  const float eps = w->cfg.ln_eps;
  const std::string pre = "joint_transformer_blocks." + std::to_string(layer) + ".";
  const int N = Nt + Ni;
  uint16_t* y_img = s->y;
  uint16_t* y_txt = s->y + static_cast<size_t>(B) * Ni * D;
  uint16_t* o_img = s->o;
  uint16_t* o_txt = s->o + static_cast<size_t>(B) * Ni * D;
  uint16_t* h_img = s->h;
  uint16_t* h_txt = s->h + static_cast<size_t>(B) * Ni * d.F;
  // 8-bit variant: the LayerNorm outputs feeding QKV and FFN-up become e4m3 + row scales
  const bool f8 = w->fp8;
  uint8_t* q8_img = f8 ? s->y8 : nullptr;
  uint8_t* q8_txt = f8 ? s->y8 + static_cast<size_t>(B) * Ni * D : nullptr;
  float* ys_img = f8 ? s->yscale : nullptr;
  float* ys_txt = f8 ? s->yscale + static_cast<size_t>(B) * Ni : nullptr;
  const Operand a_img = f8 ? Operand{q8_img, ys_img} : Operand{y_img, nullptr};
  const Operand a_txt = f8 ? Operand{q8_txt, ys_txt} : Operand{y_txt, nullptr};

  // shift = m + 0 D, scale = m + 1 D of each stream, both streams in one launch
  AF_TRY(ln_mod2(s, img, mi + 0 * D, y_img, q8_img, ys_img, Ni, txt, mt + 0 * D, y_txt, q8_txt, ys_txt, Nt, B,
                 mod_stride, D, eps, st));
  // each projection pair (image, text) runs as one grouped launch
  AF_TRY(run_calls_grouped(s, qkv_call(w, s, a_img, B, Ni, weight_op(w, pre + "attn.to_q.weight"), Nt, N),
                           qkv_call(w, s, a_txt, B, Nt, weight_op(w, pre + "attn.add_q_proj.weight"), 0, N), st));
  AF_TRY(attention(w, s, B, N, o_txt, o_img, Nt, km, st));
  // 8-bit variant: the attention output and the SwiGLU product are quantised
  // per token (into the same e4m3 buffer, free again once QKV / FFN-up ran)
  Operand oa_img{o_img, nullptr}, oa_txt{o_txt, nullptr}, ha_img{h_img, nullptr}, ha_txt{h_txt, nullptr};
  if (f8) {
    AF_TRY(quantize_act(s, o_img, B * Ni, D, q8_img, ys_img, st));
    AF_TRY(quantize_act(s, o_txt, B * Nt, D, q8_txt, ys_txt, st));
    oa_img = {q8_img, ys_img};
    oa_txt = {q8_txt, ys_txt};
  }
  AF_TRY(run_calls_grouped(
      s, gres_call(s, oa_img, B, Ni, D, weight_op(w, pre + "attn.to_out.0.weight"), D, img, mi + 2 * D, mod_stride),
      gres_call(s, oa_txt, B, Nt, D, weight_op(w, pre + "attn.to_add_out.weight"), D, txt, mt + 2 * D, mod_stride),
      st));
  AF_TRY(ln_mod2(s, img, mi + 3 * D, y_img, q8_img, ys_img, Ni, txt, mt + 3 * D, y_txt, q8_txt, ys_txt, Nt, B,
                 mod_stride, D, eps, st));
  AF_TRY(run_calls_grouped(s, swiglu_call(w, s, a_img, B * Ni, weight_op(w, pre + "ff.linear_1.weight"), h_img),
                           swiglu_call(w, s, a_txt, B * Nt, weight_op(w, pre + "ff_context.linear_1.weight"), h_txt),
                           st));
  if (f8) {
    uint8_t* h8_txt = s->y8 + static_cast<size_t>(B) * Ni * d.F;
    AF_TRY(quantize_act(s, h_img, B * Ni, d.F, s->y8, ys_img, st));
    AF_TRY(quantize_act(s, h_txt, B * Nt, d.F, h8_txt, ys_txt, st));
    ha_img = {s->y8, ys_img};
    ha_txt = {h8_txt, ys_txt};
  }
  AF_TRY(run_calls_grouped(
      s, gres_call(s, ha_img, B, Ni, d.F, weight_op(w, pre + "ff.out_projection.weight"), D, img, mi + 5 * D,
                   mod_stride),
      gres_call(s, ha_txt, B, Nt, d.F, weight_op(w, pre + "ff_context.out_projection.weight"), D, txt, mt + 5 * D,
                mod_stride),
      st));
  return AF_OK;
}

af_status single_block_impl(const af_weights* w, af_scratch* s, int layer, uint16_t* x, const float* m,
                            int mod_stride, int B, int N, const KeyMask& km, cudaStream_t st) {
  const Derived& d = w->d;
  const int D = d.D;
  const float eps = w->cfg.ln_eps;
  const std::string pre = "single_transformer_blocks." + std::to_string(layer) + ".";
  const bool f8 = w->fp8;
  uint8_t* q8 = f8 ? s->y8 : nullptr;
  float* ys = f8 ? s->yscale : nullptr;
  const Operand a = f8 ? Operand{q8, ys} : Operand{s->y, nullptr};
  AF_TRY(ln_mod(s, x, m + 0 * D, m + 1 * D, mod_stride, s->y, B * N, N, D, eps, st, q8, ys));
  AF_TRY(qkv(w, s, a, B, N, weight_op(w, pre + "attn.to_q.weight"), 0, N, st));
  AF_TRY(attention(w, s, B, N, s->o, s->o, 0, km, st));
  Operand oa{s->o, nullptr}, ha{s->h, nullptr};
  if (f8) {  // per-token e4m3 of the attention output (the QKV input codes are dead by now)
    AF_TRY(quantize_act(s, s->o, B * N, D, q8, ys, st));
    oa = {q8, ys};
  }
  AF_TRY(gated_residual(s, oa, B, N, D, weight_op(w, pre + "attn.to_out.0.weight"), D, x, m + 2 * D, mod_stride, st));
  AF_TRY(ln_mod(s, x, m + 3 * D, m + 4 * D, mod_stride, s->y, B * N, N, D, eps, st, q8, ys));
  AF_TRY(swiglu(w, s, a, B * N, weight_op(w, pre + "ff.linear_1.weight"), s->h, st));
  if (f8) {  // per-token e4m3 of the SwiGLU product (rows of F codes)
    AF_TRY(quantize_act(s, s->h, B * N, d.F, q8, ys, st));
    ha = {q8, ys};
  }
  AF_TRY(gated_residual(s, ha, B, N, d.F, weight_op(w, pre + "ff.out_projection.weight"), D, x, m + 5 * D, mod_stride,
                        st));
  return AF_OK;
}

af_status check_dev_ptr(const void* p) {
  if (!p) return AF_ERR_INVALID_ARG;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return AF_ERR_INVALID_ARG;
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return AF_ERR_INVALID_ARG;
  return AF_OK;
}

}  // namespace

// ------------------------------------------------------------ the fp32 forward
// Same sequence as forward_impl ([ARCH] §前向传播流程, §联合注意力块, §单 DiT 块)
// on an fp32 pack, every step in fp32 (fp32.cu).  Activation buffers of the
// scratch hold floats; s->tmp holds the [rows, 3D] QKV and [rows, 2F] FFN-up
// products before the QK-norm split and the SwiGLU.
namespace {

struct F32Step {
  af_scratch* s;
  cudaStream_t st;
};

af_status f32_done(cudaError_t e) { return e == cudaSuccess ? AF_OK : cuda_fail(e); }

af_status f32_gemm_op(F32Step& k, const float* A, const float* W, int M, int N, int K, int mode, float* out, int ldo,
                      int rows_per_batch, int out_rows_per_batch = 0, int out_row_off = 0, const float* gate = nullptr,
                      int gate_stride = 0) {
  LaunchScope ls(k.s, KC_GEMM, 2.0 * M * N * K, k.st);
  return f32_done(f32_gemm(A, W, M, N, K, mode, out, ldo, rows_per_batch,
                           out_rows_per_batch > 0 ? out_rows_per_batch : rows_per_batch, out_row_off, gate,
                           gate_stride, k.st));
}

af_status f32_ln_op(F32Step& k, const float* x, const float* shift, const float* scale, int mod_stride, float* y,
                    int rows, int rows_per_batch, int D, float eps) {
  LaunchScope ls(k.s, KC_LN, 8.0 * rows * D, k.st);
  return f32_done(f32_ln_modulate(x, shift, scale, mod_stride, y, rows, rows_per_batch, D, eps, k.st));
}

// Q/K/V of one stream: [rows, 3D] product, per-head LayerNorm of Q and K, scatter
af_status f32_qkv_op(const af_weights* w, F32Step& k, const float* y, int B, int rows, const float* wqkv, int row_off,
                     int n_total) {
  const Derived& d = w->d;
  AF_TRY(f32_gemm_op(k, y, wqkv, B * rows, 3 * d.D, d.D, EPI_STORE, k.s->tmp, 3 * d.D, B * rows));
  LaunchScope ls(k.s, KC_OTHER, 24.0 * B * rows * d.D, k.st);
  return f32_done(f32_qkv_split(k.s->tmp, B * rows, rows, d.H, d.hd, w->cfg.ln_eps, reinterpret_cast<float*>(k.s->q),
                                reinterpret_cast<float*>(k.s->k), reinterpret_cast<float*>(k.s->v), n_total, row_off,
                                k.st));
}

// x += gate * (silu(y W1^T) * (y W2^T)) W3^T, with W1 and W2 stored one after the other
af_status f32_ffn_op(const af_weights* w, F32Step& k, const float* y, int B, int rows, const float* w12,
                     const float* w3, float* h, float* x, const float* gate, int gate_stride) {
  const Derived& d = w->d;
  const int M = B * rows;
  AF_TRY(f32_gemm_op(k, y, w12, M, 2 * d.F, d.D, EPI_STORE, k.s->tmp, 2 * d.F, M));
  {
    LaunchScope ls(k.s, KC_OTHER, 12.0 * M * d.F, k.st);
    AF_TRY(f32_done(f32_swiglu(k.s->tmp, M, d.F, h, k.st)));
  }
  return f32_gemm_op(k, h, w3, M, d.D, d.F, EPI_GATE_RES, x, d.D, rows, 0, 0, gate, gate_stride);
}

af_status f32_attention_op(const af_weights* w, F32Step& k, int B, int N, float* out_a, float* out_b, int split,
                           const KeyMask& km) {
  const Derived& d = w->d;
  LaunchScope ls(k.s, KC_ATTN, 4.0 * B * d.H * static_cast<double>(N) * N * d.hd, k.st);
  return f32_done(f32_attention(reinterpret_cast<const float*>(k.s->q), reinterpret_cast<const float*>(k.s->k),
                                reinterpret_cast<const float*>(k.s->v), B, d.H, N, d.hd,
                                1.0f / sqrtf(static_cast<float>(d.hd)), out_a, out_b, split, d.D, km.len, km.base,
                                km.end, k.st));
}

af_status f32_timestep_mlp(const af_weights* w, F32Step& k, const float* t, int B, float* feat, float* h1,
                           float* temb) {
  const int C = w->cfg.timestep_channels, D = w->d.D;
  LaunchScope ls(k.s, KC_OTHER, 4.0 * D * (C + D), k.st, 3);
  AF_TRY(f32_done(launch_timestep_features(t, B, C, feat, k.st)));
  AF_TRY(f32_done(f32_gemv(feat, B, C, w->ptrf("time_step_proj.linear_1.weight"),
                           w->ptrf("time_step_proj.linear_1.bias"), D, 0, 1, h1, D, k.st)));
  return f32_done(f32_gemv(h1, B, D, w->ptrf("time_step_proj.linear_2.weight"), w->ptrf("time_step_proj.linear_2.bias"),
                           D, 0, 0, temb, D, k.st));
}

af_status f32_modulations(const af_weights* w, F32Step& k, const float* temb, int B, float* out) {
  const int rows = static_cast<int>(w->ada_rows);
  LaunchScope ls(k.s, KC_OTHER, 4.0 * rows * w->d.D, k.st);
  return f32_done(f32_gemv(temb, B, w->d.D, reinterpret_cast<const float*>(w->base + w->tensors[0].offset), nullptr,
                           rows, 1, 0, out, rows, k.st));
}

af_status f32_forward(const af_weights* w, af_scratch* s, const float* latents, const float* text_emb, const float* t,
                      int B, int H, int W, int L, const KeyMask& km, float* velocity, cudaStream_t st,
                      const float* premods, int pre_stride) {
  const af_config& c = w->cfg;
  const Derived& d = w->d;
  const int p = c.patch_size, hp = H / p, wp = W / p, Ni = hp * wp;
  const int R = c.num_register_tokens, Nt = R + L, N = Nt + Ni, D = d.D;
  const float eps = c.ln_eps;
  F32Step k{s, st};
  float* img = reinterpret_cast<float*>(s->img);
  float* txt = reinterpret_cast<float*>(s->txt);
  float* x = reinterpret_cast<float*>(s->x);
  float* y = reinterpret_cast<float*>(s->y);
  float* o = reinterpret_cast<float*>(s->o);
  float* h = reinterpret_cast<float*>(s->h);
  const float* mods = premods ? premods : s->mods;
  const int ms = premods ? pre_stride : static_cast<int>(w->ada_rows);
  if (!premods) {
    AF_TRY(f32_timestep_mlp(w, k, t, B, s->tfeat, s->h1, s->temb));
    AF_TRY(f32_modulations(w, k, s->temb, B, s->mods));
  }
  {
    LaunchScope ls(s, KC_OTHER, 8.0 * B * Ni * D, st);
    AF_TRY(f32_done(f32_patch_embed(latents, B, c.in_channels, H, W, p, w->ptrf("pos_embed.proj.weight"),
                                    w->ptrf("pos_embed.pos_embed"), d.G, D, img, st)));
  }
  for (int b = 0; b < B && R > 0; ++b)  // register tokens at the head of every sample's text stream
    AF_CUDA(cudaMemcpyAsync(txt + static_cast<size_t>(b) * Nt * D, w->ptrf("register_tokens"),
                            static_cast<size_t>(R) * D * 4, cudaMemcpyDeviceToDevice, st));
  if (L > 0)
    AF_TRY(f32_gemm_op(k, text_emb, w->ptrf("context_embedder.weight"), B * L, D, c.joint_attention_dim, EPI_STORE,
                       txt, D, L, Nt, R));
  for (int i = 0; i < c.num_mmdit_layers; ++i) {
    const std::string pre = "joint_transformer_blocks." + std::to_string(i) + ".";
    const float* mi = mods + w->unit_row[2 * i];
    const float* mt = mods + w->unit_row[2 * i + 1];
    float* yi = y;
    float* yt = y + static_cast<size_t>(B) * Ni * D;
    float* oi = o;
    float* ot = o + static_cast<size_t>(B) * Ni * D;
    float* hi = h;
    float* ht = h + static_cast<size_t>(B) * Ni * d.F;
    AF_TRY(f32_ln_op(k, img, mi + 0 * D, mi + 1 * D, ms, yi, B * Ni, Ni, D, eps));
    AF_TRY(f32_ln_op(k, txt, mt + 0 * D, mt + 1 * D, ms, yt, B * Nt, Nt, D, eps));
    AF_TRY(f32_qkv_op(w, k, yt, B, Nt, w->ptrf(pre + "attn.add_q_proj.weight"), 0, N));
    AF_TRY(f32_qkv_op(w, k, yi, B, Ni, w->ptrf(pre + "attn.to_q.weight"), Nt, N));
    AF_TRY(f32_attention_op(w, k, B, N, ot, oi, Nt, km));
    AF_TRY(f32_gemm_op(k, oi, w->ptrf(pre + "attn.to_out.0.weight"), B * Ni, D, D, EPI_GATE_RES, img, D, Ni, 0, 0,
                       mi + 2 * D, ms));
    AF_TRY(f32_gemm_op(k, ot, w->ptrf(pre + "attn.to_add_out.weight"), B * Nt, D, D, EPI_GATE_RES, txt, D, Nt, 0, 0,
                       mt + 2 * D, ms));
    AF_TRY(f32_ln_op(k, img, mi + 3 * D, mi + 4 * D, ms, yi, B * Ni, Ni, D, eps));
    AF_TRY(f32_ln_op(k, txt, mt + 3 * D, mt + 4 * D, ms, yt, B * Nt, Nt, D, eps));
    AF_TRY(f32_ffn_op(w, k, yi, B, Ni, w->ptrf(pre + "ff.linear_1.weight"), w->ptrf(pre + "ff.out_projection.weight"),
                      hi, img, mi + 5 * D, ms));
    AF_TRY(f32_ffn_op(w, k, yt, B, Nt, w->ptrf(pre + "ff_context.linear_1.weight"),
                      w->ptrf(pre + "ff_context.out_projection.weight"), ht, txt, mt + 5 * D, ms));
  }
  // x = cat(text, image) per sample
  AF_CUDA(cudaMemcpy2DAsync(x, static_cast<size_t>(N) * D * 4, txt, static_cast<size_t>(Nt) * D * 4,
                            static_cast<size_t>(Nt) * D * 4, B, cudaMemcpyDeviceToDevice, st));
  AF_CUDA(cudaMemcpy2DAsync(x + static_cast<size_t>(Nt) * D, static_cast<size_t>(N) * D * 4, img,
                            static_cast<size_t>(Ni) * D * 4, static_cast<size_t>(Ni) * D * 4, B,
                            cudaMemcpyDeviceToDevice, st));
  for (int i = 0; i < c.num_single_dit_layers; ++i) {
    const std::string pre = "single_transformer_blocks." + std::to_string(i) + ".";
    const float* m = mods + w->unit_row[2 * c.num_mmdit_layers + i];
    AF_TRY(f32_ln_op(k, x, m + 0 * D, m + 1 * D, ms, y, B * N, N, D, eps));
    AF_TRY(f32_qkv_op(w, k, y, B, N, w->ptrf(pre + "attn.to_q.weight"), 0, N));
    AF_TRY(f32_attention_op(w, k, B, N, o, o, 0, km));
    AF_TRY(f32_gemm_op(k, o, w->ptrf(pre + "attn.to_out.0.weight"), B * N, D, D, EPI_GATE_RES, x, D, N, 0, 0,
                       m + 2 * D, ms));
    AF_TRY(f32_ln_op(k, x, m + 3 * D, m + 4 * D, ms, y, B * N, N, D, eps));
    AF_TRY(f32_ffn_op(w, k, y, B, N, w->ptrf(pre + "ff.linear_1.weight"), w->ptrf(pre + "ff.out_projection.weight"),
                      h, x, m + 5 * D, ms));
  }
  const float* pf = mods + w->pf_row;  // pre-final: scale first, then shift
  LaunchScope ls(s, KC_OTHER, 8.0 * B * Ni * D, st);
  return f32_done(f32_output_stage(x, N, Nt, B, hp, wp, D, pf, pf + D, ms, w->ptrf("proj_out.weight"), p,
                                   c.out_channels, velocity, st));
}

}  // namespace

namespace af {
const uint16_t* weights_tensor(const af_weights* w, const char* name) { return w->ptr(name); }
int weights_device(const af_weights* w) { return w->device; }
int weights_inner_dim(const af_weights* w) { return w->d.D; }
int weights_timestep_channels(const af_weights* w) { return w->cfg.timestep_channels; }
bool weights_is_f32(const af_weights* w) { return w->f32; }
void set_last_error(const std::string& msg) { g_last_error = msg; }
}  // namespace af

// =========================================================================== C ABI

extern "C" {

const char* af_status_string(af_status st) {
  switch (st) {
    case AF_OK: return "ok";
    case AF_ERR_INVALID_ARG: return "invalid argument";
    case AF_ERR_SHAPE: return "shape error";
    case AF_ERR_UNSUPPORTED: return "unsupported configuration";
    case AF_ERR_OOM: return "out of device memory";
    case AF_ERR_CUDA: return "CUDA error";
    case AF_ERR_TIMEOUT: return "device wait timed out";
    case AF_ERR_NOT_FOUND: return "tensor not found";
  }
  return "unknown status";
}

const char* af_last_error(void) { return g_last_error.c_str(); }

af_status af_config_default(af_config* c) {
  if (!c) return AF_ERR_INVALID_ARG;
  c->patch_size = 2;
  c->in_channels = 4;
  c->out_channels = 4;
  c->num_mmdit_layers = 4;
  c->num_single_dit_layers = 32;
  c->attention_head_dim = 256;
  c->num_attention_heads = 12;
  c->joint_attention_dim = 2048;
  c->pos_embed_max_size = 1024;
  c->num_register_tokens = 8;
  c->timestep_channels = 256;
  c->ffn_inner = 0;
  c->ln_eps = 1e-6f;
  c->dtype = AF_DTYPE_BF16;
  return AF_OK;
}

af_status af_config_derive(const af_config* c, int* inner_dim, int* ffn_inner, int* grid_side) {
  Derived d;
  AF_TRY(derive(c, &d));
  if (inner_dim) *inner_dim = d.D;
  if (ffn_inner) *ffn_inner = d.F;
  if (grid_side) *grid_side = d.G;
  return AF_OK;
}

af_status af_weights_create(const af_config* cfg, int device, af_weights** out) {
  if (!out) return AF_ERR_INVALID_ARG;
  *out = nullptr;
  Derived d;
  AF_TRY(derive(cfg, &d));
  if (cfg->dtype != AF_DTYPE_BF16 && cfg->dtype != AF_DTYPE_F32) return AF_ERR_INVALID_ARG;
  // shapes the kernels cover
  if (cfg->dtype == AF_DTYPE_F32) {
    if (!(d.hd == 8 || d.hd == 16 || d.hd == 32 || d.hd == 64)) return AF_ERR_UNSUPPORTED;
  } else {
    if (d.D % 32 != 0 || d.F % 128 != 0 || cfg->joint_attention_dim % 8 != 0) return AF_ERR_UNSUPPORTED;
    if (!(d.hd == 256 || d.hd == 8 || d.hd == 16 || d.hd == 32 || d.hd == 64)) return AF_ERR_UNSUPPORTED;
    if (cfg->patch_size * cfg->patch_size * cfg->in_channels > 64) return AF_ERR_UNSUPPORTED;
    // the output projection's folded weights fill rows of a 256-row GEMM tile
    if (cfg->patch_size * cfg->patch_size * cfg->out_channels > 256) return AF_ERR_UNSUPPORTED;
    // the timestep / modulation GEMV reads rows of 16-byte vectors, at most 4096 wide
    if (cfg->timestep_channels % 8 != 0 || cfg->timestep_channels > 4096 || d.D > 4096) return AF_ERR_UNSUPPORTED;
  }
  af_weights* w = new af_weights();
  w->cfg = *cfg;
  w->d = d;
  w->device = device;
  w->f32 = cfg->dtype == AF_DTYPE_F32;
  w->esz = w->f32 ? 4 : 2;
  build_layout(w);
  int prev = 0;
  cudaGetDevice(&prev);
  if (cudaSetDevice(device) != cudaSuccess) {
    delete w;
    return AF_ERR_INVALID_ARG;
  }
  cudaError_t e = cudaMalloc(&w->base, w->bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    cudaSetDevice(prev);
    delete w;
    return AF_ERR_OOM;
  }
  e = cudaMemset(w->base, 0, w->bytes);
  cudaSetDevice(prev);
  if (e != cudaSuccess) {
    cudaFree(w->base);
    delete w;
    return cuda_fail(e);
  }
  *out = w;
  return AF_OK;
}

void af_weights_destroy(af_weights* w) {
  if (!w) return;
  if (w->base) cudaFree(w->base);
  if (w->fp8_codes) cudaFree(w->fp8_codes);
  if (w->fp8_scales) cudaFree(w->fp8_scales);
  delete w;
}

af_status af_weights_num_tensors(const af_weights* w, int* n) {
  if (!w || !n) return AF_ERR_INVALID_ARG;
  *n = static_cast<int>(w->tensors.size());
  return AF_OK;
}

af_status af_weights_tensor_info(const af_weights* w, int id, char* name, size_t name_cap, int* ndim,
                                 int64_t shape[2]) {
  if (!w || id < 0 || id >= static_cast<int>(w->tensors.size())) return AF_ERR_INVALID_ARG;
  const TensorInfo& t = w->tensors[id];
  if (name && name_cap > 0) {
    strncpy(name, t.name.c_str(), name_cap - 1);
    name[name_cap - 1] = '\0';
  }
  if (ndim) *ndim = t.ndim;
  if (shape) {
    shape[0] = t.shape[0];
    shape[1] = t.shape[1];
  }
  return AF_OK;
}

af_status af_weights_find(const af_weights* w, const char* name, int* id) {
  if (!w || !name || !id) return AF_ERR_INVALID_ARG;
  auto it = w->index.find(name);
  if (it == w->index.end()) return AF_ERR_NOT_FOUND;
  *id = it->second;
  return AF_OK;
}

af_status af_weights_set(af_weights* w, int id, const void* src, int src_is_device, int src_dtype, void* stream) {
  if (!w || !src || id < 0 || id >= static_cast<int>(w->tensors.size())) return AF_ERR_INVALID_ARG;
  if (src_dtype != AF_DTYPE_BF16 && src_dtype != AF_DTYPE_F32) return AF_ERR_INVALID_ARG;
  AF_TRY(check_device(w));
  const TensorInfo& t = w->tensors[id];
  const bool src_f32 = src_dtype == AF_DTYPE_F32;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (src_is_device) AF_TRY(check_dev_ptr(src));
  uint8_t* dst = w->base + (t.interleave ? t.pair_base : t.offset);
  const int cols = t.ndim == 2 ? static_cast<int>(t.shape[1]) : 1;
  if (src_is_device && src_f32 != w->f32) {  // convert on the device, in the pack's layout
    AF_CUDA(launch_convert_copy(src, src_f32, dst, w->f32, t.numel(), cols, t.interleave, st));
    return AF_OK;
  }
  std::vector<uint8_t> conv;
  if (!src_is_device && src_f32 != w->f32) {  // convert on the host, then copy
    conv.resize(t.numel() * w->esz);
    for (size_t i = 0; i < t.numel(); ++i) {
      if (w->f32) {
        const uint32_t u = static_cast<uint32_t>(static_cast<const uint16_t*>(src)[i]) << 16;
        memcpy(conv.data() + 4 * i, &u, 4);
      } else {
        uint32_t u;
        memcpy(&u, static_cast<const float*>(src) + i, 4);
        const uint16_t b = static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);  // nearest even
        memcpy(conv.data() + 2 * i, &b, 2);
      }
    }
    src = conv.data();
  }
  const size_t bytes = t.numel() * w->esz;
  if (t.interleave) {
    // 128-row groups of this half go to every other 128-row slot of the pair
    const size_t group = static_cast<size_t>(128) * t.shape[1] * w->esz;
    uint8_t* d0 = dst + (t.interleave == 2 ? group : 0);
    const size_t groups = static_cast<size_t>(t.shape[0]) / 128;
    if (src_is_device)
      AF_CUDA(cudaMemcpy2DAsync(d0, 2 * group, src, group, group, groups, cudaMemcpyDeviceToDevice, st));
    else
      AF_CUDA(cudaMemcpy2D(d0, 2 * group, src, group, group, groups, cudaMemcpyHostToDevice));
    return AF_OK;
  }
  if (src_is_device) {
    AF_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st));
  } else {
    AF_CUDA(cudaMemcpy(dst, src, bytes, cudaMemcpyHostToDevice));
  }
  return AF_OK;
}

af_status af_weights_get(const af_weights* w, int id, void* dst, int dst_is_device, void* stream) {
  if (!w || !dst || id < 0 || id >= static_cast<int>(w->tensors.size())) return AF_ERR_INVALID_ARG;
  AF_TRY(check_device(w));
  if (dst_is_device) AF_TRY(check_dev_ptr(dst));
  const TensorInfo& t = w->tensors[id];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaMemcpyKind kind = dst_is_device ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost;
  if (t.interleave) {
    const size_t group = static_cast<size_t>(128) * t.shape[1] * w->esz;
    const uint8_t* s0 = w->base + t.pair_base + (t.interleave == 2 ? group : 0);
    const size_t groups = static_cast<size_t>(t.shape[0]) / 128;
    if (dst_is_device)
      AF_CUDA(cudaMemcpy2DAsync(dst, group, s0, 2 * group, group, groups, kind, st));
    else
      AF_CUDA(cudaMemcpy2D(dst, group, s0, 2 * group, group, groups, kind));
    return AF_OK;
  }
  if (dst_is_device)
    AF_CUDA(cudaMemcpyAsync(dst, w->base + t.offset, t.numel() * w->esz, kind, st));
  else
    AF_CUDA(cudaMemcpy(dst, w->base + t.offset, t.numel() * w->esz, kind));
  return AF_OK;
}

af_status af_weights_init_random(af_weights* w, uint64_t seed, float std, void* stream) {
  if (!w || !(std >= 0.f)) return AF_ERR_INVALID_ARG;
  AF_TRY(check_device(w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (const TensorInfo& t : w->tensors) {
    // [ARCH] §Patch Embedding: positions ~N(0, 0.1^2); §Register Tokens: ~N(0, 0.02^2)
    const bool pos = t.name == "pos_embed.pos_embed";
    const float sd = pos ? 0.1f : (t.name == "register_tokens" ? 0.02f : std);
    uint8_t* dst = w->base + (t.interleave ? t.pair_base : t.offset);
    const int cols = t.ndim == 2 ? static_cast<int>(t.shape[1]) : 1;
    AF_CUDA(launch_init_normal(dst, w->f32, t.numel(), cols, t.interleave, crc32_ieee(t.name.c_str()), seed, sd, st));
  }
  return AF_OK;
}

af_status af_weights_quantize_fp8(af_weights* w, int enable, void* stream) {
  if (!w) return AF_ERR_INVALID_ARG;
  if (w->f32) return AF_ERR_UNSUPPORTED;
  AF_TRY(check_device(w));
  if (!enable) {
    if (w->fp8_codes) cudaFree(w->fp8_codes);
    if (w->fp8_scales) cudaFree(w->fp8_scales);
    w->fp8_codes = nullptr;
    w->fp8_scales = nullptr;
    w->fp8_region.clear();
    w->fp8 = false;
    return AF_OK;
  }
  const af_config& c = w->cfg;
  const size_t D = w->d.D, F = w->d.F;
  struct Region {
    std::string name;
    size_t rows, cols;
  };
  std::vector<Region> regions;
  for (int i = 0; i < c.num_mmdit_layers; ++i) {
    const std::string b = "joint_transformer_blocks." + std::to_string(i) + ".";
    regions.push_back({b + "attn.to_q.weight", 3 * D, D});
    regions.push_back({b + "attn.add_q_proj.weight", 3 * D, D});
    regions.push_back({b + "attn.to_out.0.weight", D, D});
    regions.push_back({b + "attn.to_add_out.weight", D, D});
    regions.push_back({b + "ff.linear_1.weight", 2 * F, D});
    regions.push_back({b + "ff_context.linear_1.weight", 2 * F, D});
    regions.push_back({b + "ff.out_projection.weight", D, F});
    regions.push_back({b + "ff_context.out_projection.weight", D, F});
  }
  for (int i = 0; i < c.num_single_dit_layers; ++i) {
    const std::string b = "single_transformer_blocks." + std::to_string(i) + ".";
    regions.push_back({b + "attn.to_q.weight", 3 * D, D});
    regions.push_back({b + "attn.to_out.0.weight", D, D});
    regions.push_back({b + "ff.linear_1.weight", 2 * F, D});
    regions.push_back({b + "ff.out_projection.weight", D, F});
  }
  std::unordered_map<std::string, af_weights::Fp8Region> where;
  size_t code_bytes = 0, scale_rows = 0;
  for (auto& r : regions) {
    where[r.name] = {code_bytes, scale_rows};
    code_bytes = (code_bytes + r.rows * r.cols + 255) & ~size_t(255);
    scale_rows += (r.rows + 255) / 256 * 256;
  }
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(w->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (!w->fp8_codes) {
    e = cudaMalloc(&w->fp8_codes, code_bytes);
    if (e == cudaSuccess) e = cudaMalloc(&w->fp8_scales, scale_rows * sizeof(float));
    if (e != cudaSuccess) {
      cudaGetLastError();
      if (w->fp8_codes) cudaFree(w->fp8_codes);
      w->fp8_codes = nullptr;
      w->fp8_scales = nullptr;
      cudaSetDevice(prev);
      return AF_ERR_OOM;
    }
    e = cudaMemsetAsync(w->fp8_scales, 0, scale_rows * sizeof(float), st);  // padding rows
  }
  for (size_t i = 0; i < regions.size() && e == cudaSuccess; ++i) {
    const auto& r = regions[i];
    const auto& at = where[r.name];
    e = launch_quantize_rows_e4m3(w->ptr(r.name), static_cast<int>(r.rows), static_cast<int>(r.cols),
                                  w->fp8_codes + at.code_off, w->fp8_scales + at.scale_off, st);
  }
  cudaSetDevice(prev);
  if (e != cudaSuccess) return cuda_fail(e);
  w->fp8_region = where;
  w->fp8 = true;
  return AF_OK;
}

af_status af_weights_bytes(const af_weights* w, size_t* bytes) {
  if (!w || !bytes) return AF_ERR_INVALID_ARG;
  *bytes = w->bytes;
  return AF_OK;
}

af_status af_scratch_create(const af_weights* w, int max_batch, int max_img_tokens, int max_text_len,
                            af_scratch** out) {
  if (!w || !out || max_batch <= 0 || max_img_tokens <= 0 || max_text_len < 0) return AF_ERR_INVALID_ARG;
  *out = nullptr;
  AF_TRY(check_device(w));
  const Derived& d = w->d;
  af_scratch* s = new af_scratch();
  s->w = w;
  s->max_b = max_batch;
  s->max_ni = max_img_tokens;
  s->max_l = max_text_len;
  s->max_nt = max_text_len + w->cfg.num_register_tokens;
  s->max_n = s->max_nt + max_img_tokens;
  s->device = w->device;
  const size_t B = max_batch, N = s->max_n, D = d.D, F = d.F;
  const size_t rowsN = B * N;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t o_err = take(256);
  const size_t o_temb = take(B * D * 4);
  const size_t o_h1 = take(B * D * 4);
  const size_t o_tfeat = take(B * w->cfg.timestep_channels * 4);
  const size_t o_mods = take(B * w->ada_rows * 4);
  const size_t es = w->esz;  // activations are stored like the weights: bf16, or fp32 for an fp32 pack
  const size_t o_y = take(rowsN * D * es);
  const size_t o_q = take(rowsN * D * es);
  const size_t o_k = take(rowsN * D * es);
  const size_t o_v = take(rowsN * D * es);
  const size_t o_o = take(rowsN * D * es);
  const size_t o_h = take(rowsN * F * es);
  const size_t o_img = take(B * s->max_ni * D * es);
  const size_t o_txt = take(B * s->max_nt * D * es);
  const size_t o_x = take(rowsN * D * es);
  const size_t o_y8 = take(w->f32 ? 0 : rowsN * (D > F ? D : F));  // e4m3 codes of y, O or h (8-bit variant)
  const size_t o_ys = take(w->f32 ? 0 : rowsN * 4);
  const size_t o_tmp = take(w->f32 ? rowsN * (3 * D > 2 * F ? 3 * D : 2 * F) * 4 : 0);
  const int cmax = w->cfg.in_channels > w->cfg.out_channels ? w->cfg.in_channels : w->cfg.out_channels;
  const size_t lat_elems = B * static_cast<size_t>(cmax) * s->max_ni * w->cfg.patch_size * w->cfg.patch_size;
  const size_t o_lat2 = take(lat_elems * 4);
  const size_t o_vel = take(lat_elems * 4);
  const size_t o_tvec = take(B * 4);
  const int kpo = w->cfg.patch_size * w->cfg.patch_size * w->cfg.out_channels;
  const size_t o_wfold = take(w->f32 ? 0 : B * 256 * D * 2);
  const size_t o_obias = take(B * 256 * 4);
  const size_t o_oproj = take(w->f32 ? 0 : B * static_cast<size_t>(s->max_ni) * kpo * 4);
  s->bytes = off;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(w->device);
  cudaError_t e = cudaMalloc(&s->base, s->bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    cudaSetDevice(prev);
    delete s;
    return AF_ERR_OOM;
  }
  e = cudaMemset(s->base, 0, s->bytes);
  s->sms = device_sm_count();
  cudaSetDevice(prev);
  if (e != cudaSuccess) {
    cudaFree(s->base);
    delete s;
    return cuda_fail(e);
  }
  s->err = reinterpret_cast<int*>(s->base + o_err);
  s->temb = reinterpret_cast<float*>(s->base + o_temb);
  s->h1 = reinterpret_cast<float*>(s->base + o_h1);
  s->tfeat = reinterpret_cast<float*>(s->base + o_tfeat);
  s->mods = reinterpret_cast<float*>(s->base + o_mods);
  s->y = reinterpret_cast<uint16_t*>(s->base + o_y);
  s->q = reinterpret_cast<uint16_t*>(s->base + o_q);
  s->k = reinterpret_cast<uint16_t*>(s->base + o_k);
  s->v = reinterpret_cast<uint16_t*>(s->base + o_v);
  s->o = reinterpret_cast<uint16_t*>(s->base + o_o);
  s->h = reinterpret_cast<uint16_t*>(s->base + o_h);
  s->img = reinterpret_cast<uint16_t*>(s->base + o_img);
  s->txt = reinterpret_cast<uint16_t*>(s->base + o_txt);
  s->x = reinterpret_cast<uint16_t*>(s->base + o_x);
  s->y8 = s->base + o_y8;
  s->tmp = reinterpret_cast<float*>(s->base + o_tmp);
  s->yscale = reinterpret_cast<float*>(s->base + o_ys);
  s->lat2 = reinterpret_cast<float*>(s->base + o_lat2);
  s->vel = reinterpret_cast<float*>(s->base + o_vel);
  s->tvec = reinterpret_cast<float*>(s->base + o_tvec);
  s->wfold = reinterpret_cast<uint16_t*>(s->base + o_wfold);
  s->obias = reinterpret_cast<float*>(s->base + o_obias);
  s->oproj = reinterpret_cast<float*>(s->base + o_oproj);
  *out = s;
  return AF_OK;
}

void af_scratch_destroy(af_scratch* s) {
  if (!s) return;
  for (cudaEvent_t e : s->pool) cudaEventDestroy(e);
  if (s->base) cudaFree(s->base);
  delete s;
}

af_status af_sync(af_scratch* s, void* stream) {
  if (!s) return AF_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AF_CUDA(cudaStreamSynchronize(st));
  int h = 0;
  AF_CUDA(cudaMemcpy(&h, s->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (h != 0) {
    AF_CUDA(cudaMemset(s->err, 0, sizeof(int)));
    return AF_ERR_TIMEOUT;
  }
  return AF_OK;
}

af_status af_check_wait_timeout(af_scratch* s, int64_t limit_ns, void* stream) {
  if (!s) return AF_ERR_INVALID_ARG;
  const int64_t lim = limit_ns < 1000000 ? 1000000 : (limit_ns > 1000000000 ? 1000000000 : limit_ns);
  LaunchScope ls(s, KC_OTHER, 0.0, static_cast<cudaStream_t>(stream));
  cudaError_t e = launch_wait_timeout_check(s->err, static_cast<uint64_t>(lim), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return AF_OK;
}

af_status af_timestep_embed(const af_weights* w, af_scratch* s, const float* t, int B, float* temb, void* stream) {
  AF_TRY(check_scratch(w, s));
  if (!t || !temb || B <= 0) return AF_ERR_INVALID_ARG;
  if (B > s->max_b) return AF_ERR_SHAPE;
  const Derived& d = w->d;
  if (w->f32) {
    F32Step k{s, static_cast<cudaStream_t>(stream)};
    return f32_timestep_mlp(w, k, t, B, s->tfeat, s->h1, temb);
  }
  LaunchScope ls(s, KC_OTHER, 2.0 * d.D * (w->cfg.timestep_channels + d.D), static_cast<cudaStream_t>(stream), 3);
  AF_CUDA(launch_timestep_mlp(t, B, w->ptr("time_step_proj.linear_1.weight"), w->ptr("time_step_proj.linear_1.bias"),
                              w->ptr("time_step_proj.linear_2.weight"), w->ptr("time_step_proj.linear_2.bias"),
                              w->cfg.timestep_channels, d.D, s->tfeat, s->h1, temb, static_cast<cudaStream_t>(stream)));
  return AF_OK;
}

af_status af_patch_embed(const af_weights* w, af_scratch* s, const float* latents, int B, int H, int W,
                         uint16_t* img_tokens, void* stream) {
  AF_TRY(check_scratch(w, s));
  if (!latents || !img_tokens || B <= 0 || H <= 0 || W <= 0) return AF_ERR_INVALID_ARG;
  if (w->f32) return AF_ERR_UNSUPPORTED;
  const int p = w->cfg.patch_size;
  if (H % p || W % p || H / p > w->d.G || W / p > w->d.G) return AF_ERR_SHAPE;
  const int Ni = (H / p) * (W / p);
  LaunchScope ls(s, KC_OTHER, 4.0 * B * Ni * w->d.D + 4.0 * B * w->cfg.in_channels * H * W,
                 static_cast<cudaStream_t>(stream));
  AF_CUDA(launch_patch_embed(latents, B, w->cfg.in_channels, H, W, p, w->ptr("pos_embed.proj.weight"),
                             w->ptr("pos_embed.pos_embed"), w->d.G, w->d.D, img_tokens, Ni, 0,
                             static_cast<cudaStream_t>(stream)));
  return AF_OK;
}

af_status af_joint_block(const af_weights* w, af_scratch* s, int layer, uint16_t* img, uint16_t* txt,
                         const float* temb, int B, int Ni, int Nt, const int* text_len, void* stream) {
  AF_TRY(check_scratch(w, s));
  if (!img || !txt || !temb || B <= 0 || Ni <= 0 || Nt <= 0) return AF_ERR_INVALID_ARG;
  if (w->f32) return AF_ERR_UNSUPPORTED;
  if (text_len && Nt < w->cfg.num_register_tokens) return AF_ERR_SHAPE;
  if (layer < 0 || layer >= w->cfg.num_mmdit_layers) return AF_ERR_INVALID_ARG;
  if (B > s->max_b || Ni + Nt > s->max_n || Ni > s->max_n) return AF_ERR_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = w->d.D;
  // modulation of this block's two streams only
  const size_t r_img = w->unit_row[2 * layer];
  const uint16_t* ada = ada_base(w);
  {
    LaunchScope ls(s, KC_OTHER, 2.0 * 12 * D * D, st, (B + 7) / 8);
    AF_CUDA(launch_modulation(temb, B, D, ada + r_img * D, 12 * D, s->mods, st));
  }
  const float* mi = s->mods;
  const float* mt = s->mods + 6 * D;
  return joint_block_impl(w, s, layer, img, txt, mi, mt, 12 * D, B, Ni, Nt, text_mask(w, text_len, Nt), st);
}

af_status af_single_block(const af_weights* w, af_scratch* s, int layer, uint16_t* x, const float* temb, int B,
                          int N, int Nt, const int* text_len, void* stream) {
  AF_TRY(check_scratch(w, s));
  if (!x || !temb || B <= 0 || N <= 0) return AF_ERR_INVALID_ARG;
  if (w->f32) return AF_ERR_UNSUPPORTED;
  if (text_len && (Nt < w->cfg.num_register_tokens || Nt > N)) return AF_ERR_SHAPE;
  if (layer < 0 || layer >= w->cfg.num_single_dit_layers) return AF_ERR_INVALID_ARG;
  if (B > s->max_b || N > s->max_n) return AF_ERR_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = w->d.D;
  const size_t r = w->unit_row[2 * w->cfg.num_mmdit_layers + layer];
  {
    LaunchScope ls(s, KC_OTHER, 2.0 * 6 * D * D, st, (B + 7) / 8);
    AF_CUDA(launch_modulation(temb, B, D, ada_base(w) + r * D, 6 * D, s->mods, st));
  }
  return single_block_impl(w, s, layer, x, s->mods, 6 * D, B, N, text_mask(w, text_len, Nt), st);
}

// The output stage ([ARCH] §调制与归一化, §前向传播流程): z = x (1 + scale) + shift
// on the image rows, o = z proj_out^T, unpatchify.  The modulation folds into a
// per-sample bf16 copy of proj_out (and a bias W . shift), so the projection of
// all image rows is one tensor-core GEMM with an fp32 store (the samples as
// the two problems of a grouped launch), then a scatter adds the bias and
// unpatchifies.  Accounted as an HBM-bound step (bytes), not as a GEMM.
static af_status output_stage(const af_weights* w, af_scratch* s, int B, int N, int Nt, int hp, int wp,
                              const float* pf, int mstride, float* velocity, cudaStream_t st) {
  const af_config& c = w->cfg;
  const int p = c.patch_size, D = w->d.D, Ni = hp * wp;
  const int kpo = p * p * c.out_channels;
  {
    LaunchScope ls(s, KC_OTHER, 2.0 * B * kpo * D * 2 + 4.0 * B * kpo, st);
    AF_CUDA(launch_output_fold(w->ptr("proj_out.weight"), kpo, D, pf, pf + D, mstride, B, s->wfold, s->obias, st));
  }
  for (int b0 = 0; b0 < B; b0 += 2) {
    GemmCall g[2];
    const int nb = B - b0 < 2 ? B - b0 : 2;
    for (int j = 0; j < nb; ++j) {
      const int b = b0 + j;
      GemmParams gp = gemm_base(s, Ni, kpo, D, EPI_STORE_F32, Ni);
      gp.out_f32 = s->oproj + static_cast<size_t>(b) * Ni * kpo;
      gp.ldo = kpo;
      g[j] = {gp, s->x + (static_cast<size_t>(b) * N + Nt) * D, s->wfold + static_cast<size_t>(b) * 256 * D, 256, true};
    }
    LaunchScope ls(s, KC_OTHER, 2.0 * nb * Ni * D + 4.0 * nb * Ni * kpo, st);
    const cudaError_t e = nb == 2 ? launch_gemm_grouped(g[0].p, g[0].A, g[0].W, g[0].W_rows, g[1].p, g[1].A, g[1].W,
                                                        g[1].W_rows, st, s->sms)
                                  : launch_gemm(g[0].p, g[0].A, g[0].W, g[0].W_rows, st, s->sms);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  LaunchScope ls(s, KC_OTHER, 4.0 * B * Ni * kpo * 2, st);
  AF_CUDA(launch_output_scatter(s->oproj, s->obias, B, hp, wp, p, c.out_channels, velocity, st));
  return AF_OK;
}

// premods != nullptr: every adaLN / pre-final modulation of this step was
// precomputed (rows in the adaLN unit order, element (b, r) at
// premods[b * pre_stride + r]); the timestep MLP and the modulation GEMV are
// skipped and `t` is not read.
static af_status forward_impl(const af_weights* w, af_scratch* s, const float* latents, const void* text_emb,
                              const float* t, int B, int H, int W, int L, const int* text_len, float* velocity,
                              cudaStream_t st, const float* premods = nullptr, int pre_stride = 0) {
  AF_TRY(check_scratch(w, s));
  if (!latents || !text_emb || !t || !velocity || B <= 0 || H <= 0 || W <= 0 || L < 0) return AF_ERR_INVALID_ARG;
  const af_config& c = w->cfg;
  const Derived& d = w->d;
  const int p = c.patch_size;
  if (H % p || W % p || H / p > d.G || W / p > d.G) return AF_ERR_SHAPE;
  const int hp = H / p, wp = W / p, Ni = hp * wp;
  const int R = c.num_register_tokens, Nt = R + L, N = Nt + Ni;
  if (B > s->max_b || Ni > s->max_ni || L > s->max_l) return AF_ERR_SHAPE;
  if (Nt <= 0) return AF_ERR_SHAPE;
  const int D = d.D;
  const size_t R_ada = w->ada_rows;
  const float* mods = premods ? premods : s->mods;
  const int mstride = premods ? pre_stride : static_cast<int>(R_ada);
  const KeyMask km = text_mask(w, text_len, Nt);
  if (w->f32)
    return f32_forward(w, s, latents, static_cast<const float*>(text_emb), t, B, H, W, L, km, velocity, st, premods,
                       pre_stride);

  // embedding stage
  if (!premods) {
    LaunchScope ls(s, KC_OTHER, 2.0 * D * (c.timestep_channels + D), st, 3);
    AF_CUDA(launch_timestep_mlp(t, B, w->ptr("time_step_proj.linear_1.weight"),
                                w->ptr("time_step_proj.linear_1.bias"), w->ptr("time_step_proj.linear_2.weight"),
                                w->ptr("time_step_proj.linear_2.bias"), c.timestep_channels, D, s->tfeat, s->h1,
                                s->temb, st));
  }
  if (!premods) {
    // every modulation of the step in one tensor-core GEMM over the adaLN
    // rows (mods[b, r] = W_ada[r] . silu(temb_b)), silu(temb) rounded to bf16
    // as in the sampler plan: the 4.6 GB of modulation weights stream once at
    // HBM rate, where the per-row GEMV ran at about a third of it.  Accounted
    // by its bytes: the weight stream, not the tensor core, bounds it.
    uint16_t* silu = reinterpret_cast<uint16_t*>(s->h1);  // h1 is free once temb is formed
    {
      LaunchScope ls(s, KC_OTHER, 6.0 * B * D, st);
      AF_CUDA(launch_silu_bf16(s->temb, B * D, silu, st));
    }
    GemmParams gp = gemm_base(s, B, static_cast<int>(R_ada), D, EPI_STORE_F32, B);
    gp.out_f32 = s->mods;
    gp.ldo = static_cast<int>(R_ada);
    LaunchScope ls(s, KC_OTHER, 2.0 * R_ada * D, st);
    AF_CUDA(launch_gemm(gp, silu, ada_base(w), static_cast<int>(R_ada), st, s->sms));
  }
  {
    LaunchScope ls(s, KC_OTHER, 4.0 * B * Ni * D + 4.0 * B * c.in_channels * H * W, st);
    AF_CUDA(launch_patch_embed(latents, B, c.in_channels, H, W, p, w->ptr("pos_embed.proj.weight"),
                               w->ptr("pos_embed.pos_embed"), d.G, D, s->img, Ni, 0, st));
  }
  for (int b = 0; b < B && R > 0; ++b)  // register tokens at the head of every sample's text stream
    AF_CUDA(cudaMemcpyAsync(s->txt + static_cast<size_t>(b) * Nt * D, w->ptr("register_tokens"),
                            static_cast<size_t>(R) * D * 2, cudaMemcpyDeviceToDevice, st));
  if (L > 0) {
    GemmParams gp = gemm_base(s, B * L, D, c.joint_attention_dim, EPI_STORE, L);
    gp.out = s->txt;
    gp.ldo = D;
    gp.out_rows_per_batch = Nt;
    gp.out_row_off = R;
    AF_TRY(run_gemm(s, gp, static_cast<const uint16_t*>(text_emb), w->ptr("context_embedder.weight"), D, st));
  }
  // joint blocks
  for (int i = 0; i < c.num_mmdit_layers; ++i) {
    const float* mi = mods + w->unit_row[2 * i];
    const float* mt = mods + w->unit_row[2 * i + 1];
    AF_TRY(joint_block_impl(w, s, i, s->img, s->txt, mi, mt, mstride, B, Ni, Nt, km, st));
  }
  // x = cat(text, image) per sample
  AF_CUDA(cudaMemcpy2DAsync(s->x, static_cast<size_t>(N) * D * 2, s->txt, static_cast<size_t>(Nt) * D * 2,
                            static_cast<size_t>(Nt) * D * 2, B, cudaMemcpyDeviceToDevice, st));
  AF_CUDA(cudaMemcpy2DAsync(s->x + static_cast<size_t>(Nt) * D, static_cast<size_t>(N) * D * 2, s->img,
                            static_cast<size_t>(Ni) * D * 2, static_cast<size_t>(Ni) * D * 2, B,
                            cudaMemcpyDeviceToDevice, st));
  for (int i = 0; i < c.num_single_dit_layers; ++i) {
    const float* m = mods + w->unit_row[2 * c.num_mmdit_layers + i];
    AF_TRY(single_block_impl(w, s, i, s->x, m, mstride, B, N, km, st));
  }
  // pre-final (scale first, then shift), proj_out, unpatchify on the image rows
  const float* pf = mods + w->pf_row;
  return output_stage(w, s, B, N, Nt, hp, wp, pf, mstride, velocity, st);
}

af_status af_transformer_forward(const af_weights* w, af_scratch* s, const float* latents, const void* text_emb,
                                 const float* t, int B, int H, int W, int L, const int* text_len, float* velocity,
                                 void* stream) {
  return forward_impl(w, s, latents, text_emb, t, B, H, W, L, text_len, velocity, static_cast<cudaStream_t>(stream));
}

static af_status denoise_step_impl(const af_weights* w, af_scratch* s, float* latents, const void* text_emb,
                                   int Bi, int H, int W, int L, const int* text_len, float guidance, float sigma,
                                   float sigma_next, cudaStream_t st, const float* premods = nullptr) {
  const int B = 2 * Bi;
  const size_t per = static_cast<size_t>(w->cfg.in_channels) * H * W;
  // CFG batch [uncond; text] shares the latents
  AF_CUDA(cudaMemcpyAsync(s->lat2, latents, per * Bi * 4, cudaMemcpyDeviceToDevice, st));
  AF_CUDA(cudaMemcpyAsync(s->lat2 + per * Bi, latents, per * Bi * 4, cudaMemcpyDeviceToDevice, st));
  if (!premods) {
    LaunchScope ls(s, KC_OTHER, 4.0 * B, st);
    AF_CUDA(launch_fill(s->tvec, B, sigma, st));
  }
  AF_TRY(forward_impl(w, s, s->lat2, text_emb, s->tvec, B, H, W, L, text_len, s->vel, st, premods, 0));
  LaunchScope ls(s, KC_OTHER, 16.0 * per * Bi, st);
  AF_CUDA(launch_euler_cfg(latents, s->vel, Bi, static_cast<int64_t>(per), guidance, sigma, sigma_next, st));
  return AF_OK;
}

static af_status check_step_args(const af_weights* w, af_scratch* s, const float* latents, const void* text_emb,
                                 int Bi, int H, int W, int L) {
  AF_TRY(check_scratch(w, s));
  if (!latents || !text_emb || Bi <= 0 || H <= 0 || W <= 0 || L < 0) return AF_ERR_INVALID_ARG;
  const int p = w->cfg.patch_size;
  if (H % p || W % p || H / p > w->d.G || W / p > w->d.G) return AF_ERR_SHAPE;
  if (2 * Bi > s->max_b || (H / p) * (W / p) > s->max_ni || L > s->max_l) return AF_ERR_SHAPE;
  if (w->cfg.in_channels != w->cfg.out_channels) return AF_ERR_UNSUPPORTED;
  return AF_OK;
}

af_status af_denoise_step(const af_weights* w, af_scratch* s, float* latents, const void* text_emb, int Bi, int H,
                          int W, int L, const int* text_len, float guidance, float sigma, float sigma_next,
                          void* stream) {
  AF_TRY(check_step_args(w, s, latents, text_emb, Bi, H, W, L));
  return denoise_step_impl(w, s, latents, text_emb, Bi, H, W, L, text_len, guidance, sigma, sigma_next,
                           static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------- sampler
struct af_sampler {
  const af_weights* w = nullptr;
  af_scratch* s = nullptr;
  float* latents = nullptr;
  const void* text = nullptr;
  const int* text_len = nullptr;
  int Bi = 0, H = 0, W = 0, L = 0, n_steps = 0;
  float guidance = 1.f;
  bool use_graphs = false;
  std::vector<float> sigmas;  // n_steps + 1
  uint8_t* base = nullptr;
  float *t_dev = nullptr, *feat = nullptr, *h1 = nullptr, *temb = nullptr, *mods = nullptr;
  uint16_t* silu = nullptr;
  std::vector<cudaGraphExec_t> graphs;
  std::vector<std::array<int64_t, AF_NUM_KERNEL_CLASSES>> graph_launches;
};

extern "C" {

af_status af_sampler_create(const af_weights* w, af_scratch* s, float* latents, const void* text_emb, int Bi,
                            int H, int W, int L, const int* text_len, int n_steps, const float* sigmas,
                            float guidance, int use_graphs, af_sampler** out) {
  if (!out) return AF_ERR_INVALID_ARG;
  *out = nullptr;
  AF_TRY(check_step_args(w, s, latents, text_emb, Bi, H, W, L));
  if (n_steps <= 0 || !sigmas) return AF_ERR_INVALID_ARG;
  af_sampler* m = new af_sampler();
  m->w = w;
  m->s = s;
  m->latents = latents;
  m->text = text_emb;
  m->text_len = text_len;
  m->Bi = Bi;
  m->H = H;
  m->W = W;
  m->L = L;
  m->n_steps = n_steps;
  m->guidance = guidance;
  m->use_graphs = use_graphs != 0;
  m->sigmas.assign(sigmas, sigmas + n_steps + 1);
  const size_t n = n_steps, D = w->d.D, C = w->cfg.timestep_channels;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t o_t = take(n * 4), o_f = take(n * C * 4), o_h = take(n * D * 4), o_e = take(n * D * 4);
  const size_t o_s = take(n * D * 2), o_m = take(n * w->ada_rows * 4);
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(w->device);
  cudaError_t e = cudaMalloc(&m->base, off);
  if (e == cudaSuccess) e = cudaMemcpy(m->base + o_t, sigmas, n * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = gemm_set_attributes();
  if (e == cudaSuccess) e = attention_set_attributes();
  if (e == cudaSuccess) e = small_kernels_set_attributes();
  cudaSetDevice(prev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    if (m->base) cudaFree(m->base);
    delete m;
    return e == cudaErrorMemoryAllocation ? AF_ERR_OOM : cuda_fail(e);
  }
  m->t_dev = reinterpret_cast<float*>(m->base + o_t);
  m->feat = reinterpret_cast<float*>(m->base + o_f);
  m->h1 = reinterpret_cast<float*>(m->base + o_h);
  m->temb = reinterpret_cast<float*>(m->base + o_e);
  m->silu = reinterpret_cast<uint16_t*>(m->base + o_s);
  m->mods = reinterpret_cast<float*>(m->base + o_m);
  m->graphs.assign(n, nullptr);
  m->graph_launches.assign(n, std::array<int64_t, AF_NUM_KERNEL_CLASSES>{0, 0, 0, 0});
  *out = m;
  return AF_OK;
}

void af_sampler_destroy(af_sampler* m) {
  if (!m) return;
  for (cudaGraphExec_t g : m->graphs)
    if (g) cudaGraphExecDestroy(g);
  if (m->base) cudaFree(m->base);
  delete m;
}

af_status af_sampler_prepare(af_sampler* m, void* stream) {
  if (!m) return AF_ERR_INVALID_ARG;
  const af_weights* w = m->w;
  af_scratch* s = m->s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int n = m->n_steps, D = w->d.D, C = w->cfg.timestep_channels;
  AF_TRY(check_device(w));
  if (w->f32) {  // every step's modulations by the fp32 GEMV, silu(temb) kept in fp32
    F32Step k{s, st};
    AF_TRY(f32_timestep_mlp(w, k, m->t_dev, n, m->feat, m->h1, m->temb));
    return f32_modulations(w, k, m->temb, n, m->mods);
  }
  {
    LaunchScope ls(s, KC_OTHER, 2.0 * D * (C + D), st, 2 * ((n + 7) / 8) + 1);
    AF_CUDA(launch_timestep_mlp(m->t_dev, n, w->ptr("time_step_proj.linear_1.weight"),
                                w->ptr("time_step_proj.linear_1.bias"), w->ptr("time_step_proj.linear_2.weight"),
                                w->ptr("time_step_proj.linear_2.bias"), C, D, m->feat, m->h1, m->temb, st));
  }
  {
    LaunchScope ls(s, KC_OTHER, 6.0 * n * D, st);
    AF_CUDA(launch_silu_bf16(m->temb, n * D, m->silu, st));
  }
  // every modulation of every step: mods[i, r] = W_ada[r] . silu(temb_i), one weight pass
  GemmParams gp = gemm_base(s, n, static_cast<int>(w->ada_rows), D, EPI_STORE_F32, n);
  gp.out_f32 = m->mods;
  gp.ldo = static_cast<int>(w->ada_rows);
  return run_gemm(s, gp, m->silu, ada_base(w), static_cast<int>(w->ada_rows), st);
}

af_status af_sampler_step(af_sampler* m, int step, void* stream) {
  if (!m || step < 0 || step >= m->n_steps) return AF_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float* premods = m->mods + static_cast<size_t>(step) * m->w->ada_rows;
  auto enqueue = [&]() {
    return denoise_step_impl(m->w, m->s, m->latents, m->text, m->Bi, m->H, m->W, m->L, m->text_len, m->guidance,
                             m->sigmas[step], m->sigmas[step + 1], st, premods);
  };
  if (!m->use_graphs) return enqueue();
  if (!st) return AF_ERR_INVALID_ARG;  // the legacy default stream cannot be captured
  if (!m->graphs[step]) {
    int64_t before[AF_NUM_KERNEL_CLASSES];
    for (int i = 0; i < AF_NUM_KERNEL_CLASSES; ++i) before[i] = m->s->launches[i];
    const bool prof = m->s->profiling;
    m->s->profiling = false;  // no event records inside a graph
    AF_CUDA(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
    const af_status qs = enqueue();
    cudaGraph_t g = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(st, &g);
    m->s->profiling = prof;
    for (int i = 0; i < AF_NUM_KERNEL_CLASSES; ++i) {
      m->graph_launches[step][i] = m->s->launches[i] - before[i];
      m->s->launches[i] = before[i];
    }
    if (qs != AF_OK) {
      if (g) cudaGraphDestroy(g);
      return qs;
    }
    AF_CUDA(ce);
    cudaGraphExec_t exec = nullptr;
    const cudaError_t ie = cudaGraphInstantiate(&exec, g, 0);
    cudaGraphDestroy(g);
    AF_CUDA(ie);
    m->graphs[step] = exec;
  }
  AF_CUDA(cudaGraphLaunch(m->graphs[step], st));
  for (int i = 0; i < AF_NUM_KERNEL_CLASSES; ++i) m->s->launches[i] += m->graph_launches[step][i];
  return AF_OK;
}

af_status af_sigma_schedule(int n_steps, float shift, int num_train_timesteps, float* out) {
  if (!out || n_steps <= 0 || num_train_timesteps <= 0 || !(shift > 0.f)) return AF_ERR_INVALID_ARG;
  const double lo = 1.0 / num_train_timesteps;
  for (int i = 0; i < n_steps; ++i) {
    const double s = n_steps == 1 ? 1.0 : 1.0 + (lo - 1.0) * i / (n_steps - 1);
    out[i] = static_cast<float>(shift * s / (1.0 + (shift - 1.0) * s));
  }
  out[n_steps] = 0.f;
  return AF_OK;
}

af_status af_launch_counts(const af_scratch* s, int64_t counts[AF_NUM_KERNEL_CLASSES]) {
  if (!s || !counts) return AF_ERR_INVALID_ARG;
  for (int i = 0; i < AF_NUM_KERNEL_CLASSES; ++i) counts[i] = s->launches[i];
  return AF_OK;
}

af_status af_profile_begin(af_scratch* s) {
  if (!s) return AF_ERR_INVALID_ARG;
  s->profiling = true;
  s->pool_used = 0;
  s->recs.clear();
  return AF_OK;
}

af_status af_profile_end(af_scratch* s, void* stream, double ms[AF_NUM_KERNEL_CLASSES],
                         int64_t launches[AF_NUM_KERNEL_CLASSES], double work[AF_NUM_KERNEL_CLASSES]) {
  if (!s) return AF_ERR_INVALID_ARG;
  s->profiling = false;
  AF_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  double t[AF_NUM_KERNEL_CLASSES] = {0, 0, 0, 0}, wk[AF_NUM_KERNEL_CLASSES] = {0, 0, 0, 0};
  int64_t n[AF_NUM_KERNEL_CLASSES] = {0, 0, 0, 0};
  for (const auto& r : s->recs) {
    float e = 0.f;
    AF_CUDA(cudaEventElapsedTime(&e, s->pool[r.e0], s->pool[r.e0 + 1]));
    t[r.cls] += e;
    n[r.cls] += r.n;
    wk[r.cls] += r.work;
  }
  s->recs.clear();
  s->pool_used = 0;
  for (int i = 0; i < AF_NUM_KERNEL_CLASSES; ++i) {
    if (ms) ms[i] = t[i];
    if (launches) launches[i] = n[i];
    if (work) work[i] = wk[i];
  }
  return AF_OK;
}

af_status af_euler_cfg_step(float* latents, const float* velocity, int Bi, int C, int H, int W, float guidance,
                            float sigma, float sigma_next, void* stream) {
  if (!latents || !velocity || Bi <= 0 || C <= 0 || H <= 0 || W <= 0) return AF_ERR_INVALID_ARG;
  AF_CUDA(launch_euler_cfg(latents, velocity, Bi, static_cast<int64_t>(C) * H * W, guidance, sigma, sigma_next,
                           static_cast<cudaStream_t>(stream)));
  return AF_OK;
}

af_status af_ln_modulate(const uint16_t* x, const float* shift, const float* scale, int mod_stride, uint16_t* y,
                         int B, int N, int D, float eps, void* stream) {
  if (!x || !shift || !scale || !y || B <= 0 || N <= 0 || D <= 0 || mod_stride < 0) return AF_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > 4096) return AF_ERR_UNSUPPORTED;
  AF_CUDA(launch_ln_modulate(x, shift, scale, mod_stride, y, B * N, N, D, eps, static_cast<cudaStream_t>(stream)));
  return AF_OK;
}

af_status af_ln_modulate_e4m3(const uint16_t* x, const float* shift, const float* scale, int mod_stride, uint8_t* y8,
                              float* yscale, int B, int N, int D, float eps, void* stream) {
  if (!x || !shift || !scale || !y8 || !yscale || B <= 0 || N <= 0 || D <= 0 || mod_stride < 0)
    return AF_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > 4096) return AF_ERR_UNSUPPORTED;
  AF_CUDA(launch_ln_modulate(x, shift, scale, mod_stride, nullptr, B * N, N, D, eps, static_cast<cudaStream_t>(stream),
                             nullptr, y8, yscale));
  return AF_OK;
}

af_status af_quantize_rows_e4m3(const uint16_t* x, int rows, int cols, uint8_t* q, float* scale, void* stream) {
  if (!x || !q || !scale || rows <= 0 || cols <= 0) return AF_ERR_INVALID_ARG;
  if (cols % 8 != 0) return AF_ERR_UNSUPPORTED;
  AF_CUDA(launch_quantize_rows_e4m3(x, rows, cols, q, scale, static_cast<cudaStream_t>(stream)));
  return AF_OK;
}

af_status af_linear_fp8(const uint8_t* A, const float* a_scale, const uint8_t* W, const float* w_scale, uint16_t* C,
                        int M, int N, int K, void* stream) {
  if (!A || !a_scale || !W || !w_scale || !C || M <= 0 || N <= 0 || K <= 0) return AF_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % 8 != 0) return AF_ERR_UNSUPPORTED;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.K = K;
  p.mode = EPI_STORE;
  p.rows_per_batch = M;
  p.out_rows_per_batch = M;
  p.out = C;
  p.ldo = N;
  p.err = nullptr;
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  static int sms = 0;
  if (!sms) sms = device_sm_count();
  AF_CUDA(launch_gemm(p, A, W, N, static_cast<cudaStream_t>(stream), sms));
  return AF_OK;
}

// A plain bf16 product C[M, N] = A W^T as GEMM parameters.
static GemmParams plain_gemm(uint16_t* C, int M, int N, int K) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.K = K;
  p.mode = EPI_STORE;
  p.rows_per_batch = M;
  p.out_rows_per_batch = M;
  p.out = C;
  p.ldo = N;
  p.err = nullptr;
  return p;
}

af_status af_linear(const uint16_t* A, const uint16_t* W, uint16_t* C, int M, int N, int K, void* stream) {
  if (!A || !W || !C || M <= 0 || N <= 0 || K <= 0) return AF_ERR_INVALID_ARG;
  if (K % 8 != 0 || N % 8 != 0) return AF_ERR_UNSUPPORTED;
  static int sms = 0;
  if (!sms) sms = device_sm_count();
  AF_CUDA(launch_gemm(plain_gemm(C, M, N, K), A, W, N, static_cast<cudaStream_t>(stream), sms));
  return AF_OK;
}

af_status af_linear_grouped(const uint16_t* A0, const uint16_t* W0, uint16_t* C0, int M0, int N0, int K0,
                            const uint16_t* A1, const uint16_t* W1, uint16_t* C1, int M1, int N1, int K1,
                            void* stream) {
  if (!A0 || !W0 || !C0 || M0 <= 0 || N0 <= 0 || K0 <= 0) return AF_ERR_INVALID_ARG;
  if (!A1 || !W1 || !C1 || M1 <= 0 || N1 <= 0 || K1 <= 0) return AF_ERR_INVALID_ARG;
  if (K0 % 8 != 0 || N0 % 8 != 0 || K1 % 8 != 0 || N1 % 8 != 0) return AF_ERR_UNSUPPORTED;
  static int sms = 0;
  if (!sms) sms = device_sm_count();
  AF_CUDA(launch_gemm_grouped(plain_gemm(C0, M0, N0, K0), A0, W0, N0, plain_gemm(C1, M1, N1, K1), A1, W1, N1,
                              static_cast<cudaStream_t>(stream), sms));
  return AF_OK;
}

af_status af_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o, int B, int H, int N,
                       int hd, int qk_normalized, const int* key_len, int key_base, int key_end, void* stream) {
  if (!q || !k || !v || !o || B <= 0 || H <= 0 || N <= 0) return AF_ERR_INVALID_ARG;
  if (key_len && (key_base < 1 || key_end < key_base || key_end > N)) return AF_ERR_INVALID_ARG;
  if (!(hd == 256 || hd == 8 || hd == 16 || hd == 32 || hd == 64)) return AF_ERR_UNSUPPORTED;
  AttnParams p;
  p.B = B;
  p.H = H;
  p.N = N;
  p.hd = hd;
  p.out_a = o;
  p.out_b = o;
  p.split = 0;
  p.ldo = H * hd;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(hd));
  p.qk_normalized = qk_normalized ? 1 : 0;
  p.q = q;
  p.err = nullptr;
  p.key_len = key_len;
  p.key_base = key_base;
  p.key_end = key_end;
  AF_CUDA(launch_attention(p, q, k, v, static_cast<cudaStream_t>(stream)));
  return AF_OK;
}

}  // extern "C"
