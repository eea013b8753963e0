// fp32.cu -- the forward in fp32 arithmetic end to end (weight pack dtype
// AF_DTYPE_F32), for small configurations such as the 1 + 1-block,
// D = 32 model, where the tensor-core bf16 path would narrow the arithmetic
// the configuration states.  Plain SIMT kernels; every one follows the same
// step of "Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南"
// as its bf16 counterpart:
//
//   f32_gemm_kernel        C = A W^T (64 x 64 tiles, 4 x 4 outputs per
//                          thread) with a plain store (output rows remapped
//                          per sample) or the adaLN-Zero gated residual
//                          x += gate[b] * acc (§联合注意力块, §单 DiT 块)
//   f32_ln_modulate_kernel LayerNorm without affine weights, then
//                          (1 + scale) and + shift (§调制与归一化)
//   f32_qkv_split_kernel   per-head LayerNorm of Q and K, V as is, scattered
//                          to [B, H, n_total, hd] (§注意力处理器与 QKV 融合)
//   f32_swiglu_kernel      silu(y W1^T) * (y W2^T) (§FeedForward)
//   f32_attn_kernel        softmax(q k^T * scale) v per query row, two passes
//                          (row maximum, then the weighted sum), with the
//                          optional text-padding key mask
//   f32_gemv_kernel        timestep MLP and every modulation (§前向传播流程)
//   f32_patch_embed_kernel patch projection + centre-cropped position row
//                          (§Patch Embedding)
//   f32_output_stage_kernel pre-final modulation, proj_out, unpatchify
//                          (§调制与归一化, §前向传播流程)
#include <cmath>

#include "af_internal.h"

namespace af {

namespace {

constexpr int FT = 64;  // output tile side
constexpr int FK = 16;  // k-slice per shared-memory stage

__device__ __forceinline__ float silu_f(float a) { return a / (1.0f + expf(-a)); }

__global__ void __launch_bounds__(256) f32_gemm_kernel(const float* __restrict__ A, const float* __restrict__ W,
                                                       int M, int N, int K, int mode, float* __restrict__ out,
                                                       int ldo, int rows_per_batch, int out_rows_per_batch,
                                                       int out_row_off, const float* __restrict__ gate,
                                                       int gate_stride) {
  __shared__ float As[FK][FT + 1];
  __shared__ float Ws[FK][FT + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * FT, n0 = blockIdx.x * FT;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += FK) {
    for (int e = threadIdx.x; e < FT * FK; e += blockDim.x) {
      const int r = e / FK, c = e - r * FK;
      const int gk = k0 + c;
      const int gm = m0 + r, gn = n0 + r;
      As[c][r] = (gm < M && gk < K) ? A[static_cast<size_t>(gm) * K + gk] : 0.f;
      Ws[c][r] = (gn < N && gk < K) ? W[static_cast<size_t>(gn) * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < FK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= M) continue;
    const int b = m / rows_per_batch, r = m - b * rows_per_batch;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= N) continue;
      if (mode == EPI_GATE_RES) {
        float* x = out + static_cast<size_t>(m) * ldo + n;
        *x = *x + gate[static_cast<size_t>(b) * gate_stride + n] * acc[i][j];
      } else {
        const size_t orow = static_cast<size_t>(b) * out_rows_per_batch + out_row_off + r;
        out[orow * ldo + n] = acc[i][j];
      }
    }
  }
}

__global__ void __launch_bounds__(256) f32_ln_modulate_kernel(const float* __restrict__ x,
                                                              const float* __restrict__ shift,
                                                              const float* __restrict__ scale, int mod_stride,
                                                              float* __restrict__ y, int rows, int rows_per_batch,
                                                              int D, float eps) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* xr = x + static_cast<size_t>(row) * D;
  float s = 0.f;
  for (int d = lane; d < D; d += 32) s += xr[d];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mu = s / static_cast<float>(D);
  float v = 0.f;
  for (int d = lane; d < D; d += 32) {
    const float c = xr[d] - mu;
    v += c * c;
  }
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const float rstd = 1.0f / sqrtf(v / static_cast<float>(D) + eps);
  const int b = row / rows_per_batch;
  const float* sh = shift + static_cast<size_t>(b) * mod_stride;
  const float* sc = scale + static_cast<size_t>(b) * mod_stride;
  float* yr = y + static_cast<size_t>(row) * D;
  for (int d = lane; d < D; d += 32) yr[d] = (xr[d] - mu) * rstd * (1.0f + sc[d]) + sh[d];
}

// t: [M, 3D] rows (Q | K | V); one thread per (row, head, part)
__global__ void f32_qkv_split_kernel(const float* __restrict__ t, int M, int rows_per_batch, int heads, int hd,
                                     float eps, float* __restrict__ q, float* __restrict__ k, float* __restrict__ v,
                                     int n_total, int row_off) {
  const int D = heads * hd;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= M * heads * 3) return;
  const int part = idx % 3;
  const int h = (idx / 3) % heads;
  const int m = idx / (3 * heads);
  const int b = m / rows_per_batch, r = m - b * rows_per_batch;
  const float* src = t + static_cast<size_t>(m) * 3 * D + part * D + h * hd;
  float* dst = (part == 0 ? q : (part == 1 ? k : v)) +
               ((static_cast<size_t>(b) * heads + h) * n_total + row_off + r) * hd;
  if (part == 2) {
    for (int d = 0; d < hd; ++d) dst[d] = src[d];
    return;
  }
  float mu = 0.f;
  for (int d = 0; d < hd; ++d) mu += src[d];
  mu /= static_cast<float>(hd);
  float var = 0.f;
  for (int d = 0; d < hd; ++d) var += (src[d] - mu) * (src[d] - mu);
  const float rstd = 1.0f / sqrtf(var / static_cast<float>(hd) + eps);
  for (int d = 0; d < hd; ++d) dst[d] = (src[d] - mu) * rstd;
}

__global__ void f32_swiglu_kernel(const float* __restrict__ t, int M, int F, float* __restrict__ h) {
  const size_t n = static_cast<size_t>(M) * F;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t m = i / F, f = i - m * F;
    const float a = t[m * 2 * F + f], g = t[m * 2 * F + F + f];
    h[i] = silu_f(a) * g;
  }
}

template <int HD>
__global__ void f32_attn_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                const float* __restrict__ v, int B, int H, int N, float scale,
                                float* __restrict__ out_a, float* __restrict__ out_b, int split, int ldo,
                                const int* __restrict__ key_len, int key_base, int key_end) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * H * N) return;
  const int i = idx % N, bh = idx / N, h = bh % H, b = bh / H;
  int lo = N, hi = N;  // masked keys [lo, hi)
  if (key_len) {
    int len = key_len[b];
    const int cap = key_end - key_base;
    len = len < 0 ? 0 : (len > cap ? cap : len);
    lo = key_base + len;
    hi = key_end;
  }
  const float* kb = k + static_cast<size_t>(bh) * N * HD;
  const float* vb = v + static_cast<size_t>(bh) * N * HD;
  float qv[HD];
#pragma unroll
  for (int d = 0; d < HD; ++d) qv[d] = q[(static_cast<size_t>(bh) * N + i) * HD + d];
  float mx = -INFINITY;
  for (int j = 0; j < N; ++j) {
    if (j >= lo && j < hi) continue;
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < HD; ++d) s = fmaf(qv[d], kb[static_cast<size_t>(j) * HD + d], s);
    mx = fmaxf(mx, s * scale);
  }
  float l = 0.f, o[HD];
#pragma unroll
  for (int d = 0; d < HD; ++d) o[d] = 0.f;
  for (int j = 0; j < N; ++j) {
    if (j >= lo && j < hi) continue;
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < HD; ++d) s = fmaf(qv[d], kb[static_cast<size_t>(j) * HD + d], s);
    const float p = expf(s * scale - mx);
    l += p;
#pragma unroll
    for (int d = 0; d < HD; ++d) o[d] = fmaf(p, vb[static_cast<size_t>(j) * HD + d], o[d]);
  }
  float* dst = i < split ? out_a + (static_cast<size_t>(b) * split + i) * ldo
                         : out_b + (static_cast<size_t>(b) * (N - split) + (i - split)) * ldo;
  dst += h * HD;
  const float inv = 1.0f / l;
#pragma unroll
  for (int d = 0; d < HD; ++d) dst[d] = o[d] * inv;
}

// out[b * out_stride + j] = post(sum_k W[j, k] pre(x[b, k]) + bias[j]); one warp per row j
__global__ void __launch_bounds__(256) f32_gemv_kernel(const float* __restrict__ x, int B, int K,
                                                       const float* __restrict__ W, const float* __restrict__ bias,
                                                       int rows, int pre, int post, float* __restrict__ out,
                                                       int out_stride) {
  const int lane = threadIdx.x & 31;
  const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (j >= rows) return;
  const float* wr = W + static_cast<size_t>(j) * K;
  for (int b = 0; b < B; ++b) {
    const float* xb = x + static_cast<size_t>(b) * K;
    float s = 0.f;
    for (int kk = lane; kk < K; kk += 32) {
      const float a = pre == 1 ? silu_f(xb[kk]) : xb[kk];
      s = fmaf(wr[kk], a, s);
    }
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      if (bias) s += bias[j];
      if (post == 1) s = silu_f(s);
      out[static_cast<size_t>(b) * out_stride + j] = s;
    }
  }
}

// one thread per (b, token, d)
__global__ void f32_patch_embed_kernel(const float* __restrict__ lat, int B, int C, int H, int W, int p,
                                       const float* __restrict__ wpe, const float* __restrict__ pos, int G, int D,
                                       float* __restrict__ out) {
  const int hp = H / p, wp = W / p, Ni = hp * wp, KP = p * p * C;
  const size_t total = static_cast<size_t>(B) * Ni * D;
  const int r0 = (G - hp) / 2, c0 = (G - wp) / 2;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int d = static_cast<int>(i % D);
    const size_t bn = i / D;
    const int n = static_cast<int>(bn % Ni), b = static_cast<int>(bn / Ni);
    const int ph = n / wp, pw = n - ph * wp;
    float s = 0.f;
    for (int kk = 0; kk < KP; ++kk) {
      const int c = kk % C, pxy = kk / C, py = pxy / p, px = pxy - py * p;
      const float xv = lat[((static_cast<size_t>(b) * C + c) * H + ph * p + py) * W + pw * p + px];
      s = fmaf(wpe[static_cast<size_t>(d) * KP + kk], xv, s);
    }
    out[i] = s + pos[static_cast<size_t>((r0 + ph) * G + c0 + pw) * D + d];
  }
}

// one thread per (b, token, output column oc = (py * p + px) * C + c)
__global__ void f32_output_stage_kernel(const float* __restrict__ x, int rows_per_batch, int row_off, int B, int hp,
                                        int wp, int D, const float* __restrict__ scale,
                                        const float* __restrict__ shift, int mod_stride,
                                        const float* __restrict__ wout, int p, int C, float* __restrict__ vel) {
  const int Ni = hp * wp, OC = p * p * C;
  const int total = B * Ni * OC;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int oc = idx % OC, n = (idx / OC) % Ni, b = idx / (OC * Ni);
  const float* xr = x + (static_cast<size_t>(b) * rows_per_batch + row_off + n) * D;
  const float* sc = scale + static_cast<size_t>(b) * mod_stride;
  const float* sh = shift + static_cast<size_t>(b) * mod_stride;
  const float* wr = wout + static_cast<size_t>(oc) * D;
  float s = 0.f;
  for (int d = 0; d < D; ++d) s = fmaf(xr[d] * (1.0f + sc[d]) + sh[d], wr[d], s);
  const int c = oc % C, pxy = oc / C, py = pxy / p, px = pxy - py * p;
  const int ph = n / wp, pw = n - ph * wp;
  const int Himg = hp * p, Wimg = wp * p;
  vel[((static_cast<size_t>(b) * C + c) * Himg + ph * p + py) * Wimg + pw * p + px] = s;
}

int blocks_for(size_t n, int threads) {
  const size_t b = (n + threads - 1) / threads;
  return static_cast<int>(b < 1 ? 1 : (b > (1u << 20) ? (1u << 20) : b));
}

}  // namespace

cudaError_t f32_gemm(const float* A, const float* W, int M, int N, int K, int mode, float* out, int ldo,
                     int rows_per_batch, int out_rows_per_batch, int out_row_off, const float* gate, int gate_stride,
                     cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const dim3 grid((N + FT - 1) / FT, (M + FT - 1) / FT);
  f32_gemm_kernel<<<grid, 256, 0, s>>>(A, W, M, N, K, mode, out, ldo, rows_per_batch, out_rows_per_batch,
                                       out_row_off, gate, gate_stride);
  return cudaGetLastError();
}

cudaError_t f32_ln_modulate(const float* x, const float* shift, const float* scale, int mod_stride, float* y,
                            int rows, int rows_per_batch, int D, float eps, cudaStream_t s) {
  f32_ln_modulate_kernel<<<(rows + 7) / 8, 256, 0, s>>>(x, shift, scale, mod_stride, y, rows, rows_per_batch, D, eps);
  return cudaGetLastError();
}

cudaError_t f32_qkv_split(const float* t, int M, int rows_per_batch, int heads, int hd, float eps, float* q, float* k,
                          float* v, int n_total, int row_off, cudaStream_t s) {
  const int n = M * heads * 3;
  f32_qkv_split_kernel<<<(n + 127) / 128, 128, 0, s>>>(t, M, rows_per_batch, heads, hd, eps, q, k, v, n_total,
                                                       row_off);
  return cudaGetLastError();
}

cudaError_t f32_swiglu(const float* t, int M, int F, float* h, cudaStream_t s) {
  f32_swiglu_kernel<<<blocks_for(static_cast<size_t>(M) * F, 256), 256, 0, s>>>(t, M, F, h);
  return cudaGetLastError();
}

cudaError_t f32_attention(const float* q, const float* k, const float* v, int B, int H, int N, int hd, float scale,
                          float* out_a, float* out_b, int split, int ldo, const int* key_len, int key_base,
                          int key_end, cudaStream_t s) {
  const int n = B * H * N, blocks = (n + 127) / 128;
  switch (hd) {
    case 8: f32_attn_kernel<8><<<blocks, 128, 0, s>>>(q, k, v, B, H, N, scale, out_a, out_b, split, ldo, key_len,
                                                      key_base, key_end); break;
    case 16: f32_attn_kernel<16><<<blocks, 128, 0, s>>>(q, k, v, B, H, N, scale, out_a, out_b, split, ldo, key_len,
                                                        key_base, key_end); break;
    case 32: f32_attn_kernel<32><<<blocks, 128, 0, s>>>(q, k, v, B, H, N, scale, out_a, out_b, split, ldo, key_len,
                                                        key_base, key_end); break;
    case 64: f32_attn_kernel<64><<<blocks, 128, 0, s>>>(q, k, v, B, H, N, scale, out_a, out_b, split, ldo, key_len,
                                                        key_base, key_end); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t f32_gemv(const float* x, int B, int K, const float* W, const float* bias, int rows, int pre, int post,
                     float* out, int out_stride, cudaStream_t s) {
  f32_gemv_kernel<<<(rows + 7) / 8, 256, 0, s>>>(x, B, K, W, bias, rows, pre, post, out, out_stride);
  return cudaGetLastError();
}

cudaError_t f32_patch_embed(const float* lat, int B, int C, int H, int W, int p, const float* w_pe, const float* pos,
                            int G, int D, float* out, cudaStream_t s) {
  const size_t n = static_cast<size_t>(B) * (H / p) * (W / p) * D;
  f32_patch_embed_kernel<<<blocks_for(n, 256), 256, 0, s>>>(lat, B, C, H, W, p, w_pe, pos, G, D, out);
  return cudaGetLastError();
}

cudaError_t f32_output_stage(const float* x, int rows_per_batch, int row_off, int B, int hp, int wp, int D,
                             const float* scale, const float* shift, int mod_stride, const float* w_out, int p, int C,
                             float* vel, cudaStream_t s) {
  const int n = B * hp * wp * p * p * C;
  f32_output_stage_kernel<<<(n + 127) / 128, 128, 0, s>>>(x, rows_per_batch, row_off, B, hp, wp, D, scale, shift,
                                                         mod_stride, w_out, p, C, vel);
  return cudaGetLastError();
}

}  // namespace af
