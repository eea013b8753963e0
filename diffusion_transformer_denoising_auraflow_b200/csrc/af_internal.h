// af_internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <string>

namespace af {

// Epilogues fused into the tensor-core GEMM.
enum GemmMode : int {
  EPI_STORE = 0,     // C = acc (bf16), optional output row remap
  EPI_GATE_RES = 1,  // x += gate[b] * acc   (adaLN-Zero gated residual)
  EPI_SWIGLU = 2,    // h = silu(acc[W1 half]) * acc[W2 half]
  EPI_QKV = 3,       // per-head LayerNorm of Q and K, scatter to [B, H, N, hd]
  EPI_STORE_F32 = 4, // C = acc (fp32) into out_f32
};

struct GemmParams {
  int M, N, K;        // acc[M, N] = A[M, K] * W[N, K]^T  (EPI_SWIGLU: N = output width F)
  int mode;
  int rows_per_batch;      // sample index of GEMM row r is r / rows_per_batch
  int out_rows_per_batch;  // output rows per sample
  int out_row_off;         // first output row of each sample
  uint16_t* out;           // STORE / SWIGLU output, GATE_RES residual (in/out)
  float* out_f32;          // STORE_F32 output
  int ldo;                 // row stride of `out` in elements
  const float* gate;       // GATE_RES: gate of sample b at gate[b * gate_stride + col]
  int gate_stride;
  uint16_t* q;             // QKV: destinations [B, heads, n_total, hd]
  uint16_t* k;
  uint16_t* v;
  int heads, hd, n_total, qkv_row_off, D;
  float eps;
  int num_m_tiles, num_n_tiles, num_tiles, group_n;
  int* err;                // device error word
  // 8-bit GEMM (A and W in e4m3) when w_scale != nullptr: acc[m, n] is
  // rescaled by a_scale[m] * w_scale[weight row of n]; w_scale must be
  // readable 32 rows past every weight row the GEMM touches (pad to 256)
  const float* a_scale = nullptr;
  const float* w_scale = nullptr;
  // nonzero when the epilogue's output tiles move by TMA through shared
  // memory (set by the launcher): GATE_RES (residual in and out) and SWIGLU
  // when `out` is 16-byte aligned, ldo * 2 a multiple of 16 and the output
  // rows are the GEMM rows; QKV when q, k and v are equally spaced buffers
  // (one 3-D tensor map over the three)
  int res_tma = 0;
};

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_THREADS = 192;
// per epilogue warp, two 32 x 32 bf16 residual boxes (gated-residual epilogue)
constexpr int GEMM_RES_BYTES = 4 * 2 * 32 * 32 * 2;
constexpr int GEMM_SMEM_BYTES =
    GEMM_STAGES * (GEMM_BM + GEMM_BN) * GEMM_BK * 2 + GEMM_RES_BYTES + 1024 /*barriers*/ + 1024 /*align*/;

// Host helpers (gemm.cu)
bool encode_tmap_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer, bool bytes = false, int swizzle_bytes = 128);
bool encode_tmap_3d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                    uint64_t s2_bytes, uint32_t b0, uint32_t b1, uint32_t b2, int swizzle_bytes = 128);
cudaError_t launch_gemm(const GemmParams& p_in, const void* A, const void* W, int W_rows, cudaStream_t stream,
                        int num_sms);
// Two problems (same operand type) in one persistent CTA-pair launch, the
// second's tiles after the first's; falls back to two launches when the
// problems are too small for CTA pairs.
cudaError_t launch_gemm_grouped(const GemmParams& p0, const void* A0, const void* W0, int W0_rows,
                                const GemmParams& p1, const void* A1, const void* W1, int W1_rows,
                                cudaStream_t stream, int num_sms);
int device_sm_count();

// Attention (attention.cu)
struct AttnParams {
  int B, H, N, hd;
  // output row r (< N) of sample b goes to
  //   r <  split: out_a + (b * split + r) * ldo + h * hd
  //   r >= split: out_b + (b * (N - split) + r - split) * ldo + h * hd
  uint16_t* out_a;
  uint16_t* out_b;
  int split;
  int ldo;
  float scale_log2;  // softmax scale * log2(e)
  int qk_normalized; // nonzero: every q, k row has L2 norm <= sqrt(hd) (per-head LayerNorm output)
  const uint16_t* q; // [B, H, N, hd] (read directly by the QK-normalised kernel)
  int* err;
  // optional key mask: for sample b the keys [key_base + key_len[b], key_end)
  // take no part in the softmax (key_len == nullptr: none); key_len[b] is
  // clamped to [0, key_end - key_base]
  const int* key_len = nullptr;
  int key_base = 0, key_end = 0;
};
cudaError_t launch_attention(const AttnParams& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             cudaStream_t stream);

// Small kernels (kernels.cu)
cudaError_t launch_ln_modulate(const uint16_t* x, const float* shift, const float* scale, int mod_stride,
                               uint16_t* y, int rows, int rows_per_batch, int D, float eps, cudaStream_t s,
                               int* err = nullptr, uint8_t* y8 = nullptr, float* yscale = nullptr);
// y8 != nullptr: write e4m3 codes + per-row scales (y8 [rows, D], yscale [rows]) instead of bf16 y
// One LayerNorm + modulate problem of nb samples x rows_per_batch rows (D = 3072):
// scale / shift of sample b at + b * mod_stride; per = CTAs per sample (set by the launcher).
struct LnSegment {
  const uint16_t* x;
  const float* shift;
  const float* scale;
  uint16_t* y;
  uint8_t* y8;
  float* ys;
  int rows_per_batch;
  int nb;
  int per;
};
// Both segments in one launch (the joint block's image and text streams); g1.nb = 0 for one.
cudaError_t launch_ln_modulate_pair(LnSegment g0, LnSegment g1, int mod_stride, int D, float eps, cudaStream_t s,
                                    int* err);
cudaError_t launch_quantize_rows_e4m3(const uint16_t* x, int rows, int K, uint8_t* q, float* scale, cudaStream_t s);
// The bounded-wait check: one CTA waits on an mbarrier phase nothing completes
// for limit_ns, records the timeout in *err and returns (kernels.cu).
cudaError_t launch_wait_timeout_check(int* err, uint64_t limit_ns, cudaStream_t s);
cudaError_t launch_timestep_mlp(const float* t, int B, const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                                const uint16_t* b2, int C, int D, float* feat, float* h1, float* temb, cudaStream_t s);
cudaError_t launch_modulation(const float* temb, int B, int D, const uint16_t* w, int rows, float* out,
                              cudaStream_t s);
cudaError_t launch_patch_embed(const float* lat, int B, int C, int H, int W, int p, const uint16_t* w_pe,
                               const uint16_t* pos, int G, int D, uint16_t* out, int out_rows_per_batch,
                               int out_row_off, cudaStream_t s);
// The output stage on the tensor cores: fold (1 + scale) into a bf16 copy of
// proj_out per sample (256-row blocks, rows >= KP zero) and shift into a
// bias; after the fp32-output GEMM, add the bias and unpatchify.
cudaError_t launch_output_fold(const uint16_t* w_out, int KP, int D, const float* scale, const float* shift,
                               int mod_stride, int B, uint16_t* wfold, float* bias, cudaStream_t s);
cudaError_t launch_output_scatter(const float* o, const float* bias, int B, int hp, int wp, int p, int C, float* vel,
                                  cudaStream_t s);
cudaError_t launch_fill(float* dst, int n, float value, cudaStream_t s);
cudaError_t launch_silu_bf16(const float* x, int n, uint16_t* y, cudaStream_t s);
cudaError_t gemm_set_attributes();
cudaError_t attention_set_attributes();
cudaError_t small_kernels_set_attributes();
cudaError_t launch_euler_cfg(float* lat, const float* v, int Bi, int64_t per_sample, float g, float sigma,
                             float sigma_next, cudaStream_t s);
cudaError_t launch_timestep_features(const float* t, int B, int C, float* feat, cudaStream_t s);
// x += (sigma' - sigma) (vu + g (vc - vu)) over n elements, the halves given apart
cudaError_t launch_euler_cfg2(float* lat, const float* v_uncond, const float* v_text, int64_t n, float g, float sigma,
                              float sigma_next, cudaStream_t s);

// Weight-pack filling (init.cu).  interleave: 0 plain, 1 / 2 = linear_1 /
// linear_2 rows of an FFN up pair stored in alternating 128-row groups.
uint32_t crc32_ieee(const char* s);
cudaError_t launch_init_normal(void* dst, bool f32, size_t numel, int cols, int interleave, uint32_t key,
                               uint64_t seed, float stdv, cudaStream_t s);
cudaError_t launch_convert_copy(const void* src, bool src_f32, void* dst, bool dst_f32, size_t numel, int cols,
                                int interleave, cudaStream_t s);

// The fp32 forward's kernels (fp32.cu).  mode: EPI_STORE (rows remapped per
// sample) or EPI_GATE_RES (out[m, n] += gate[b, n] * acc).
cudaError_t f32_gemm(const float* A, const float* W, int M, int N, int K, int mode, float* out, int ldo,
                     int rows_per_batch, int out_rows_per_batch, int out_row_off, const float* gate, int gate_stride,
                     cudaStream_t s);
cudaError_t f32_ln_modulate(const float* x, const float* shift, const float* scale, int mod_stride, float* y,
                            int rows, int rows_per_batch, int D, float eps, cudaStream_t s);
cudaError_t f32_qkv_split(const float* t, int M, int rows_per_batch, int heads, int hd, float eps, float* q, float* k,
                          float* v, int n_total, int row_off, cudaStream_t s);
cudaError_t f32_swiglu(const float* t, int M, int F, float* h, cudaStream_t s);
cudaError_t f32_attention(const float* q, const float* k, const float* v, int B, int H, int N, int hd, float scale,
                          float* out_a, float* out_b, int split, int ldo, const int* key_len, int key_base,
                          int key_end, cudaStream_t s);
cudaError_t f32_gemv(const float* x, int B, int K, const float* W, const float* bias, int rows, int pre, int post,
                     float* out, int out_stride, cudaStream_t s);
cudaError_t f32_patch_embed(const float* lat, int B, int C, int H, int W, int p, const float* w_pe, const float* pos,
                            int G, int D, float* out, cudaStream_t s);
cudaError_t f32_output_stage(const float* x, int rows_per_batch, int row_off, int B, int hp, int wp, int D,
                             const float* scale, const float* shift, int mod_stride, const float* w_out, int p, int C,
                             float* vel, cudaStream_t s);

}  // namespace af

// Read-only accessors of the weight pack and the thread's last-error text,
// for entry points defined outside api.cu.
struct af_weights;
namespace af {
const uint16_t* weights_tensor(const af_weights* w, const char* name);
int weights_device(const af_weights* w);
int weights_inner_dim(const af_weights* w);
int weights_timestep_channels(const af_weights* w);
bool weights_is_f32(const af_weights* w);
void set_last_error(const std::string& msg);
}  // namespace af
