// kernels.cu -- the HBM-bound kernels of the AuraFlow forward on sm_100a.
//
// Page cited: "Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南"
// (sections named per kernel) and "Diffusers 中 AuraFlow 管线实战" (CFG).
//
//   ln_modulate      FP32 LayerNorm (no affine) + adaLN (1 + scale), + shift
//                    (§调制与归一化).  One warp per row, 16-byte loads, the
//                    row kept in registers, two-pass mean / variance with
//                    warp shuffles.
//   gemv_rows        out[b, j] = act(W[j] . in(x[b]) + bias[j]) for the
//                    timestep MLP and every adaLN-Zero / pre-final linear
//                    (§前向传播流程, §联合注意力块): one warp per weight row,
//                    weights streamed once for the whole batch.
//   patch_embed      patch gather + Linear(p*p*C -> D) + centre-cropped
//                    learned position row (§Patch Embedding).
//   output_fold /    the output stage around one tensor-core GEMM: the
//   output_scatter   pre-final x * (1 + scale) + shift folded into a per-sample
//                    copy of proj_out plus a bias, and after the GEMM the
//                    bias added and the unpatchify scatter (§调制与归一化,
//                    §前向传播流程).
//   euler_cfg        v = v_u + g (v_c - v_u); x += (sigma' - sigma) v.
#include "af_internal.h"
#include "ptx.cuh"

namespace af {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Per-row e4m3 scaling (the 8-bit GEMM inputs): a = max |row|, codes
// e4m3(x * (448 / a)), scale a / 448 (1 and zeros for an all-zero row).
__device__ __forceinline__ float e4m3_inv_scale(float amax) { return amax > 0.f ? 448.0f / amax : 1.0f; }
__device__ __forceinline__ float e4m3_scale(float amax) { return amax > 0.f ? amax / 448.0f : 1.0f; }

// max |v| over the full warp in one instruction (sm_100a f32 redux; NaN
// inputs are ignored, as fmaxf does)
__device__ __forceinline__ float redux_max_abs(float v) {
  float r;
  asm volatile("redux.sync.max.abs.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// ------------------------------------------------------------------ LN + modulate
template <int VPL, bool OUT8>  // 8-element vectors per lane; OUT8: e4m3 codes + row scale
__global__ void __launch_bounds__(256) ln_modulate_kernel(const uint16_t* __restrict__ x,
                                                          const float* __restrict__ shift,
                                                          const float* __restrict__ scale, int mod_stride,
                                                          uint16_t* __restrict__ y, uint8_t* __restrict__ y8,
                                                          float* __restrict__ yscale, int rows, int rows_per_batch,
                                                          int D, float eps) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const int nvec = D >> 3;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(warp) * D);
  float v[VPL][8];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = i * 32 + lane;
    if (vi < nvec) {
      const uint4 u = xr[vi];
      v[i][0] = bf16_lo(u.x); v[i][1] = bf16_hi(u.x); v[i][2] = bf16_lo(u.y); v[i][3] = bf16_hi(u.y);
      v[i][4] = bf16_lo(u.z); v[i][5] = bf16_hi(u.z); v[i][6] = bf16_lo(u.w); v[i][7] = bf16_hi(u.w);
#pragma unroll
      for (int e = 0; e < 8; ++e) s += v[i][e];
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
    }
  }
  const float mean = warp_sum(s) / D;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    if (i * 32 + lane < nvec) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = v[i][e] - mean;
        ss += d * d;
      }
    }
  }
  const float rstd = rsqrtf(warp_sum(ss) / D + eps);
  const int b = warp / rows_per_batch;
  const float* sh = shift + static_cast<size_t>(b) * mod_stride;
  const float* sc = scale + static_cast<size_t>(b) * mod_stride;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = i * 32 + lane;
    if (vi < nvec) {
      const float4 s0 = *reinterpret_cast<const float4*>(sc + vi * 8);
      const float4 s1 = *reinterpret_cast<const float4*>(sc + vi * 8 + 4);
      const float4 h0 = *reinterpret_cast<const float4*>(sh + vi * 8);
      const float4 h1 = *reinterpret_cast<const float4*>(sh + vi * 8 + 4);
      const float scv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      const float shv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        v[i][e] = (v[i][e] - mean) * rstd * (1.0f + scv[e]) + shv[e];  // the row's output, in place
        amax = fmaxf(amax, fabsf(v[i][e]));
      }
    }
  }
  if constexpr (OUT8) {
    amax = redux_max_abs(amax);
    const float inv = e4m3_inv_scale(amax);
    uint2* yr = reinterpret_cast<uint2*>(y8 + static_cast<size_t>(warp) * D);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = i * 32 + lane;
      if (vi < nvec)
        yr[vi] = make_uint2(pack_e4m3x4(v[i][0] * inv, v[i][1] * inv, v[i][2] * inv, v[i][3] * inv),
                            pack_e4m3x4(v[i][4] * inv, v[i][5] * inv, v[i][6] * inv, v[i][7] * inv));
    }
    if (lane == 0) yscale[warp] = e4m3_scale(amax);
  } else {
    uint4* yr = reinterpret_cast<uint4*>(y + static_cast<size_t>(warp) * D);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = i * 32 + lane;
      if (vi < nvec) {
        uint4 u;
        u.x = pack_bf16(v[i][0], v[i][1]);
        u.y = pack_bf16(v[i][2], v[i][3]);
        u.z = pack_bf16(v[i][4], v[i][5]);
        u.w = pack_bf16(v[i][6], v[i][7]);
        yr[vi] = u;
      }
    }
  }
}

// Wide rows (D = 3072), HBM-bound: rows stream into shared memory by bulk
// copies, stages of LNB_ROWS rows (LNB_STAGES stages) per CTA, LNB_PER_SM
// CTAs per SM.  The producer warp first bulk-copies the CTA's sample's scale
// and shift, then streams rows.  The LNB_CW consumer warps split the columns,
// not the rows: each owns a fixed set of 16-byte column vectors of every row,
// so its (1 + scale) and shift stay in registers for the CTA's lifetime; a
// warp loads its part of the stage's rows into registers and hands the stage
// back at once, and the row statistics (two-pass mean and variance, then the
// e4m3 row maximum for 8-bit output) are combined across the consumer warps
// through shared memory at named barrier 1.  Arithmetic on packed fp32 pairs
// (sm_100 f32x2).  One launch serves up to two problems (the joint block's
// image and text streams), CTAs split between them in proportion to their
// rows; 1-D grid: segment 0's samples x CTAs per sample, then segment 1's.
constexpr int LNB_D = 3072;
constexpr int LNB_ROWS = 2;     // rows per stage
constexpr int LNB_STAGES = 4;
constexpr int LNB_CW = 4;       // consumer warps
constexpr int LNB_PER_SM = 2;
constexpr uint32_t LNB_ROW_BYTES = LNB_D * 2;
constexpr int LNB_THREADS = 32 * (LNB_CW + 1);
constexpr int LNB_SMEM = LNB_STAGES * LNB_ROWS * LNB_ROW_BYTES + 2 * LNB_D * 4;

// packed fp32 pairs
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// the two bf16 halves of w as a packed fp32 pair, kept opaque to
// common-subexpression elimination: a row held as bf16 pairs is expanded
// again in each pass instead of being cached as fp32 (twice the registers)
__device__ __forceinline__ uint64_t f2_from_bf16x2_each(uint32_t w) {
  uint64_t r;
  asm volatile(
      "{\n\t.reg .b32 lo, hi;\n\t"
      "shl.b32 lo, %1, 16;\n\t"
      "and.b32 hi, %1, 0xFFFF0000;\n\t"
      "mov.b64 %0, {lo, hi};\n\t}"
      : "=l"(r)
      : "r"(w));
  return r;
}

template <bool OUT8>
__global__ void __launch_bounds__(LNB_THREADS, LNB_PER_SM) ln_modulate_bulk_kernel(LnSegment g0, LnSegment g1,
                                                                                   int mod_stride, float eps,
                                                                                   int* err) {
  extern __shared__ __align__(128) uint8_t lnb_raw[];  // [stage][row] x 6 KB, then (1 + scale) | shift
  uint8_t* rowbuf = lnb_raw;
  float* mod_s = reinterpret_cast<float*>(lnb_raw + LNB_STAGES * LNB_ROWS * LNB_ROW_BYTES);
  __shared__ uint64_t full[LNB_STAGES], empty[LNB_STAGES], mod_full;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the first g0.nb * g0.per CTAs serve segment 0, the rest segment 1
  const int n0 = g0.nb * g0.per;
  const bool sec = static_cast<int>(blockIdx.x) >= n0;
  const int id = sec ? static_cast<int>(blockIdx.x) - n0 : static_cast<int>(blockIdx.x);
  const int per = sec ? g1.per : g0.per;
  const int rows_per_batch = sec ? g1.rows_per_batch : g0.rows_per_batch;
  const int b = id / per, cx = id - b * per;
  const uint16_t* __restrict__ x = sec ? g1.x : g0.x;
  const int nchunks = (rows_per_batch + LNB_ROWS - 1) / LNB_ROWS;
  const size_t row0 = static_cast<size_t>(b) * rows_per_batch;
  if (threadIdx.x == 0) {
    for (int i = 0; i < LNB_STAGES; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), LNB_CW);
    }
    mbar_init(smem_u32(&mod_full), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == LNB_CW) {
    // producer: one elected thread copies this sample's scale and shift, then
    // streams chunks of LNB_ROWS rows
    if (lane == 0) {
      const size_t mo = static_cast<size_t>(b) * mod_stride;
      mbar_arrive_expect_tx(smem_u32(&mod_full), 2 * LNB_D * 4);
      bulk_load(smem_u32(mod_s), (sec ? g1.scale : g0.scale) + mo, LNB_D * 4, smem_u32(&mod_full));
      bulk_load(smem_u32(mod_s + LNB_D), (sec ? g1.shift : g0.shift) + mo, LNB_D * 4, smem_u32(&mod_full));
      bool ok = true;
      int k = 0;
      for (int c = cx; c < nchunks; c += per, ++k) {
        const int st = k % LNB_STAGES;
        const uint32_t ph = (k / LNB_STAGES) & 1;
        if (!mbar_wait(smem_u32(&empty[st]), ph ^ 1u, err, &abort_flag)) { ok = false; break; }
        const int n = min(LNB_ROWS, rows_per_batch - c * LNB_ROWS);
        mbar_arrive_expect_tx(smem_u32(&full[st]), n * LNB_ROW_BYTES);
        for (int r = 0; r < n; ++r)
          bulk_load(smem_u32(rowbuf + (st * LNB_ROWS + r) * LNB_ROW_BYTES),
                    x + (row0 + static_cast<size_t>(c) * LNB_ROWS + r) * LNB_D, LNB_ROW_BYTES,
                    smem_u32(&full[st]));
      }
      if (!ok) {  // let copies already in flight land before the CTA exits
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 200000ull) {
        }
      }
    }
    return;
  }
  // consumers: warp w owns 16-byte column vectors [32 VPW w, 32 VPW (w + 1))
  // of both rows of a stage (lane l: vectors 32 VPW w + 32 i + l, i < VPW),
  // so its (1 + scale) and shift stay in registers; the row statistics are
  // summed across the LNB_CW warps through shared memory at the consumers'
  // named barrier 1.  Every barrier is a bar.red.or of "this thread
  // gave up", so all consumer threads leave the loop together.
  auto any_failed = [](bool failed) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(failed)), "r"(32 * LNB_CW)
        : "memory");
    return r != 0;
  };
  __shared__ __align__(16) float red[3][LNB_ROWS][LNB_CW];  // [statistic][row][warp]
  constexpr int VPW = LNB_D / 8 / LNB_CW / 32;               // 16-byte vectors per lane
  static_assert(VPW * 32 * LNB_CW * 8 == LNB_D, "columns split evenly over the consumer warps");
  auto total = [&](const float* t) {
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < LNB_CW; ++i) v += t[i];
    return v;
  };
  auto largest = [&](const float* t) {
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < LNB_CW; ++i) v = fmaxf(v, t[i]);
    return v;
  };
  uint64_t av[VPW][4], hv[VPW][4];                           // (1 + scale), shift as packed pairs
  {
    const bool got = mbar_wait(smem_u32(&mod_full), 0, err, &abort_flag);
    if (any_failed(!got)) return;
#pragma unroll
    for (int i = 0; i < VPW; ++i) {
      const int c0 = 8 * (warp * 32 * VPW + i * 32 + lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        av[i][e] = f2_pack(1.0f + mod_s[c0 + 2 * e], 1.0f + mod_s[c0 + 2 * e + 1]);
        hv[i][e] = f2_pack(mod_s[LNB_D + c0 + 2 * e], mod_s[LNB_D + c0 + 2 * e + 1]);
      }
    }
  }
  // this sample's first output row
  uint16_t* __restrict__ y = OUT8 ? nullptr : (sec ? g1.y : g0.y) + row0 * LNB_D;
  uint8_t* __restrict__ y8 = OUT8 ? (sec ? g1.y8 : g0.y8) + row0 * LNB_D : nullptr;
  float* __restrict__ yscale = OUT8 ? (sec ? g1.ys : g0.ys) + row0 : nullptr;
  const int v0 = warp * 32 * VPW + lane;  // this lane's first vector; then every 32th
  int k = 0;
  for (int c = cx; c < nchunks; c += per, ++k) {
    const int st = k % LNB_STAGES;
    const uint32_t ph = (k / LNB_STAGES) & 1;
    const bool got = mbar_wait(smem_u32(&full[st]), ph, err, &abort_flag);
    uint4 u[LNB_ROWS][VPW];
    if (got) {
#pragma unroll
      for (int rr = 0; rr < LNB_ROWS; ++rr) {
        const uint4* xr = reinterpret_cast<const uint4*>(rowbuf + (st * LNB_ROWS + rr) * LNB_ROW_BYTES);
#pragma unroll
        for (int i = 0; i < VPW; ++i) u[rr][i] = xr[v0 + 32 * i];
      }
    }
    // the rows are in registers: the stage goes back to the producer
    __syncwarp();
    if (got && lane == 0) mbar_arrive(smem_u32(&empty[st]));
    // pass 1: row sums
#pragma unroll
    for (int rr = 0; rr < LNB_ROWS; ++rr) {
      uint64_t s2 = f2_pack(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < VPW; ++i) {
        const uint32_t w[4] = {u[rr][i].x, u[rr][i].y, u[rr][i].z, u[rr][i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) s2 = f2_add(s2, f2_from_bf16x2_each(w[e]));
      }
      const float2 sv = f2_unpack(s2);
      const float t = warp_sum(sv.x + sv.y);
      if (lane == 0) red[0][rr][warp] = t;
    }
    if (any_failed(!got)) break;
    uint64_t nm[LNB_ROWS];
#pragma unroll
    for (int rr = 0; rr < LNB_ROWS; ++rr) {
      const float mean = total(red[0][rr]) * (1.0f / LNB_D);
      nm[rr] = f2_pack(-mean, -mean);
    }
    // pass 2: centred squares
#pragma unroll
    for (int rr = 0; rr < LNB_ROWS; ++rr) {
      uint64_t q2 = f2_pack(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < VPW; ++i) {
        const uint32_t w[4] = {u[rr][i].x, u[rr][i].y, u[rr][i].z, u[rr][i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint64_t d = f2_add(f2_from_bf16x2_each(w[e]), nm[rr]);
          q2 = f2_fma(d, d, q2);
        }
      }
      const float2 qv = f2_unpack(q2);
      const float t = warp_sum(qv.x + qv.y);
      if (lane == 0) red[1][rr][warp] = t;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(32 * LNB_CW) : "memory");
    const int nrows = min(LNB_ROWS, rows_per_batch - c * LNB_ROWS);
    uint64_t q[LNB_ROWS][VPW][4];  // 8-bit output: the rows' outputs, kept until the row maxima are known
#pragma unroll
    for (int rr = 0; rr < LNB_ROWS; ++rr) {
      const float rstd = rsqrtf(total(red[1][rr]) * (1.0f / LNB_D) + eps);
      const uint64_t rs2 = f2_pack(rstd, rstd);
      // (x - mean) rstd (1 + scale) + shift for vector i, pairs 0..3
      auto outv = [&](int i, uint64_t (&o)[4]) {
        const uint32_t w[4] = {u[rr][i].x, u[rr][i].y, u[rr][i].z, u[rr][i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = f2_fma(f2_mul(f2_add(f2_from_bf16x2_each(w[e]), nm[rr]), rs2), av[i][e], hv[i][e]);
      };
      const int r = c * LNB_ROWS + rr;
      if constexpr (OUT8) {
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < VPW; ++i) {
          outv(i, q[rr][i]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 v = f2_unpack(q[rr][i][e]);
            amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
          }
        }
        amax = redux_max_abs(amax);
        if (lane == 0) red[2][rr][warp] = amax;
      } else if (rr < nrows) {
        uint4* yr = reinterpret_cast<uint4*>(y + static_cast<size_t>(r) * LNB_D);
#pragma unroll
        for (int i = 0; i < VPW; ++i) {
          uint64_t o[4];
          outv(i, o);
          const float2 a0 = f2_unpack(o[0]), a1 = f2_unpack(o[1]), a2 = f2_unpack(o[2]), a3 = f2_unpack(o[3]);
          yr[v0 + 32 * i] = make_uint4(pack_bf16(a0.x, a0.y), pack_bf16(a1.x, a1.y), pack_bf16(a2.x, a2.y),
                                       pack_bf16(a3.x, a3.y));
        }
      }
    }
    if constexpr (OUT8) {
      // the row's e4m3 scale needs the maximum over all four warps' columns
      asm volatile("bar.sync 1, %0;" ::"r"(32 * LNB_CW) : "memory");
#pragma unroll
      for (int rr = 0; rr < LNB_ROWS; ++rr) {
        if (rr >= nrows) continue;
        const float amax = largest(red[2][rr]);
        const float inv = e4m3_inv_scale(amax);
        const int r = c * LNB_ROWS + rr;
        uint2* yr = reinterpret_cast<uint2*>(y8 + static_cast<size_t>(r) * LNB_D);
#pragma unroll
        for (int i = 0; i < VPW; ++i) {
          float2 v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) v[e] = f2_unpack(q[rr][i][e]);
          yr[v0 + 32 * i] = make_uint2(pack_e4m3x4(v[0].x * inv, v[0].y * inv, v[1].x * inv, v[1].y * inv),
                                       pack_e4m3x4(v[2].x * inv, v[2].y * inv, v[3].x * inv, v[3].y * inv));
        }
        if (threadIdx.x == 0) yscale[r] = e4m3_scale(amax);
      }
    }
  }
}

// Segment sizes: CTAs per sample in proportion to the segment's rows, about
// LNB_PER_SM CTAs per SM over the whole launch.
static void ln_plan(LnSegment& g, int total_rows, int sms) {
  if (g.nb <= 0) { g.nb = 0; g.per = 0; return; }
  const int nchunks = (g.rows_per_batch + LNB_ROWS - 1) / LNB_ROWS;
  const double share = static_cast<double>(g.rows_per_batch) * g.nb / total_rows;
  const int want = static_cast<int>(LNB_PER_SM * sms * share / g.nb + 0.5);
  g.per = max(1, min(nchunks, want));
}

static bool ln_bulk_ok(const LnSegment& g, int mod_stride) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return al(g.x) && al(g.shift) && al(g.scale) && (mod_stride % 4) == 0;
}

cudaError_t launch_ln_modulate_pair(LnSegment g0, LnSegment g1, int mod_stride, int D, float eps, cudaStream_t s,
                                    int* err) {
  if (g1.nb > 0 && ((g0.y8 == nullptr) != (g1.y8 == nullptr))) return cudaErrorInvalidValue;
  if (D != LNB_D || !ln_bulk_ok(g0, mod_stride) || (g1.nb > 0 && !ln_bulk_ok(g1, mod_stride))) {
    // the generic row kernel, one launch per segment
    cudaError_t e = launch_ln_modulate(g0.x, g0.shift, g0.scale, mod_stride, g0.y, g0.nb * g0.rows_per_batch,
                                       g0.rows_per_batch, D, eps, s, err, g0.y8, g0.ys);
    if (e != cudaSuccess || g1.nb <= 0) return e;
    return launch_ln_modulate(g1.x, g1.shift, g1.scale, mod_stride, g1.y, g1.nb * g1.rows_per_batch,
                              g1.rows_per_batch, D, eps, s, err, g1.y8, g1.ys);
  }
  if (g0.nb <= 0 || g0.rows_per_batch <= 0) return cudaErrorInvalidValue;
  if (g1.nb > 0 && g1.rows_per_batch <= 0) g1.nb = 0;
  cudaError_t e = small_kernels_set_attributes();
  if (e != cudaSuccess) return e;
  static int sms = 0;
  if (!sms) sms = device_sm_count();
  const int total = g0.nb * g0.rows_per_batch + max(g1.nb, 0) * g1.rows_per_batch;
  ln_plan(g0, total, sms);
  ln_plan(g1, total, sms);
  const int grid = g0.nb * g0.per + g1.nb * g1.per;
  if (g0.y8)
    ln_modulate_bulk_kernel<true><<<grid, LNB_THREADS, LNB_SMEM, s>>>(g0, g1, mod_stride, eps, err);
  else
    ln_modulate_bulk_kernel<false><<<grid, LNB_THREADS, LNB_SMEM, s>>>(g0, g1, mod_stride, eps, err);
  return cudaGetLastError();
}

cudaError_t launch_ln_modulate(const uint16_t* x, const float* shift, const float* scale, int mod_stride,
                               uint16_t* y, int rows, int rows_per_batch, int D, float eps, cudaStream_t s,
                               int* err, uint8_t* y8, float* yscale) {
  if (rows <= 0) return cudaSuccess;
  if (D % 8 != 0) return cudaErrorInvalidValue;
  const bool out8 = y8 != nullptr;
  if (out8 && !yscale) return cudaErrorInvalidValue;
  if (rows_per_batch <= 0) return cudaErrorInvalidValue;
  if (D == LNB_D && rows % rows_per_batch == 0) {
    const LnSegment g0{x, shift, scale, y, y8, yscale, rows_per_batch, rows / rows_per_batch, 0};
    if (ln_bulk_ok(g0, mod_stride)) return launch_ln_modulate_pair(g0, LnSegment{}, mod_stride, D, eps, s, err);
  }
  const int nvec = D / 8;
  const int vpl = (nvec + 31) / 32;
  const int blocks = (rows + 7) / 8;
#define AF_LN_CASE(N)                                                                                        \
  if (vpl <= N) {                                                                                            \
    if (out8)                                                                                                \
      ln_modulate_kernel<N, true><<<blocks, 256, 0, s>>>(x, shift, scale, mod_stride, y, y8, yscale, rows,    \
                                                         rows_per_batch, D, eps);                            \
    else                                                                                                     \
      ln_modulate_kernel<N, false><<<blocks, 256, 0, s>>>(x, shift, scale, mod_stride, y, y8, yscale, rows,   \
                                                          rows_per_batch, D, eps);                           \
    return cudaGetLastError();                                                                               \
  }
  AF_LN_CASE(1)
  AF_LN_CASE(2)
  AF_LN_CASE(4)
  AF_LN_CASE(8)
  AF_LN_CASE(12)
  AF_LN_CASE(16)
#undef AF_LN_CASE
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ per-row e4m3 quantisation
// One warp per row of a bf16 [rows, K] matrix (K a multiple of 8): codes
// e4m3(x * 448 / amax) into q [rows, K] and the row scale amax / 448.
__global__ void __launch_bounds__(256) quantize_rows_e4m3_kernel(const uint16_t* __restrict__ x, int rows, int K,
                                                                 uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row) * K);
  const int nvec = K >> 3;
  float amax = 0.f;
  for (int vi = lane; vi < nvec; vi += 32) {
    const uint4 u = xr[vi];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
  }
  amax = redux_max_abs(amax);
  const float inv = e4m3_inv_scale(amax);
  uint2* qr = reinterpret_cast<uint2*>(q + static_cast<size_t>(row) * K);
  for (int vi = lane; vi < nvec; vi += 32) {
    const uint4 u = xr[vi];
    qr[vi] = make_uint2(pack_e4m3x4(bf16_lo(u.x) * inv, bf16_hi(u.x) * inv, bf16_lo(u.y) * inv, bf16_hi(u.y) * inv),
                        pack_e4m3x4(bf16_lo(u.z) * inv, bf16_hi(u.z) * inv, bf16_lo(u.w) * inv, bf16_hi(u.w) * inv));
  }
  if (lane == 0) scale[row] = e4m3_scale(amax);
}

// Wide rows (K a multiple of 1024, up to 8192: the attention output and the
// SwiGLU product): one CTA per row, each thread keeps 32 consecutive values
// in registers, so the row is read from HBM once; the row maximum is reduced
// across the CTA's warps through shared memory.
__global__ void __launch_bounds__(256) quantize_wide_rows_e4m3_kernel(const uint16_t* __restrict__ x, int K,
                                                                      uint8_t* __restrict__ q,
                                                                      float* __restrict__ scale) {
  __shared__ float wmax[8];
  const size_t row = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * K) + 4 * t;
  uint4 u[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) u[i] = xr[i];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
  }
  amax = redux_max_abs(amax);
  if (lane == 0) wmax[warp] = amax;
  __syncthreads();
  amax = wmax[0];
  for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) amax = fmaxf(amax, wmax[i]);
  const float inv = e4m3_inv_scale(amax);
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    c[2 * i] = pack_e4m3x4(bf16_lo(u[i].x) * inv, bf16_hi(u[i].x) * inv, bf16_lo(u[i].y) * inv, bf16_hi(u[i].y) * inv);
    c[2 * i + 1] =
        pack_e4m3x4(bf16_lo(u[i].z) * inv, bf16_hi(u[i].z) * inv, bf16_lo(u[i].w) * inv, bf16_hi(u[i].w) * inv);
  }
  uint4* qr = reinterpret_cast<uint4*>(q + row * K) + 2 * t;
  qr[0] = make_uint4(c[0], c[1], c[2], c[3]);
  qr[1] = make_uint4(c[4], c[5], c[6], c[7]);
  if (t == 0) scale[row] = e4m3_scale(amax);
}

cudaError_t launch_quantize_rows_e4m3(const uint16_t* x, int rows, int K, uint8_t* q, float* scale, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (K <= 0 || K % 8 != 0) return cudaErrorInvalidValue;
  const bool aligned = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(q)) & 15) == 0;
  if (K % 1024 == 0 && K <= 8192 && aligned) {  // 32 values per thread, 1 to 8 warps
    quantize_wide_rows_e4m3_kernel<<<rows, K / 32, 0, s>>>(x, K, q, scale);
    return cudaGetLastError();
  }
  quantize_rows_e4m3_kernel<<<(rows + 7) / 8, 256, 0, s>>>(x, rows, K, q, scale);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ batched GEMV
// out[b * out_stride + j] = post(sum_k W[j, k] * pre(x[b, k]) + bias[j]),  j < rows
// pre/post: 0 = identity, 1 = SiLU.  x is staged once per CTA in shared memory.
constexpr int GEMV_MAX_B = 8;

template <int VPL>  // 16-byte weight vectors per lane (K = VPL * 256), all issued before use
__global__ void __launch_bounds__(256) gemv_rows_kernel(const float* __restrict__ x, int B, int K,
                                                        const uint16_t* __restrict__ W,
                                                        const uint16_t* __restrict__ bias, int rows, int pre,
                                                        int post, float* __restrict__ out, int out_stride) {
  extern __shared__ float xs[];  // [B, K]
  for (int i = threadIdx.x; i < B * K; i += blockDim.x) {
    float a = x[i];
    if (pre == 1) a = a / (1.0f + __expf(-a));
    xs[i] = a;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int j = blockIdx.x * wpb + (threadIdx.x >> 5); j < rows; j += gridDim.x * wpb) {
    const uint4* wr = reinterpret_cast<const uint4*>(W + static_cast<size_t>(j) * K);
    const int nvec = K >> 3;
    uint4 u[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) u[i] = (i * 32 + lane < nvec) ? __ldg(wr + i * 32 + lane) : make_uint4(0, 0, 0, 0);
    float acc[GEMV_MAX_B];
#pragma unroll
    for (int bb = 0; bb < GEMV_MAX_B; ++bb) acc[bb] = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const float w[8] = {bf16_lo(u[i].x), bf16_hi(u[i].x), bf16_lo(u[i].y), bf16_hi(u[i].y),
                          bf16_lo(u[i].z), bf16_hi(u[i].z), bf16_lo(u[i].w), bf16_hi(u[i].w)};
#pragma unroll
      for (int bb = 0; bb < GEMV_MAX_B; ++bb) {
        if (bb < B && i * 32 + lane < nvec) {
          const float4* xb = reinterpret_cast<const float4*>(xs + bb * K + (i * 32 + lane) * 8);
          const float4 x0 = xb[0], x1 = xb[1];
          acc[bb] += w[0] * x0.x + w[1] * x0.y + w[2] * x0.z + w[3] * x0.w + w[4] * x1.x + w[5] * x1.y +
                     w[6] * x1.z + w[7] * x1.w;
        }
      }
    }
#pragma unroll
    for (int bb = 0; bb < GEMV_MAX_B; ++bb) {
      if (bb < B) {
        float r = warp_sum(acc[bb]);
        if (lane == 0) {
          if (bias) r += __uint_as_float(static_cast<uint32_t>(bias[j]) << 16);
          if (post == 1) r = r / (1.0f + __expf(-r));
          out[static_cast<size_t>(bb) * out_stride + j] = r;
        }
      }
    }
  }
}

template <int VPL>
static cudaError_t gemv_attr() {
  return cudaFuncSetAttribute(gemv_rows_kernel<VPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              GEMV_MAX_B * VPL * 256 * static_cast<int>(sizeof(float)));
}

// ------------------------------------------------------------------ bounded-wait check
// The timeout path of every pipeline wait, run on purpose and without any
// fault: the warp takes 32 TMEM columns as the tensor-core kernels do, waits
// on an mbarrier phase that no thread completes, gives up after limit_ns
// (recording the timeout in *err, as mbar_wait does for any expired wait),
// and frees the columns before it exits.
__global__ void __launch_bounds__(32) wait_timeout_check_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t slot;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  tmem_alloc(smem_u32(&slot), 32);
  tmem_relinquish();
  tc_fence_before();
  __syncwarp();
  tc_fence_after();
  const uint32_t tmem = slot;
  mbar_wait(smem_u32(&bar), 0, err, &abort_flag, limit_ns);  // nothing arrives: runs out
  tc_fence_before();
  __syncwarp();
  tc_fence_after();
  tmem_dealloc(tmem, 32);
}

cudaError_t launch_wait_timeout_check(int* err, uint64_t limit_ns, cudaStream_t s) {
  if (!err) return cudaErrorInvalidValue;
  wait_timeout_check_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

// Shared-memory opt-ins of this file's kernels, once per device.
cudaError_t small_kernels_set_attributes() {
  static uint64_t done = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if ((done >> dev) & 1u) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(ln_modulate_bulk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, LNB_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(ln_modulate_bulk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, LNB_SMEM);
  if (e == cudaSuccess) e = gemv_attr<1>();
  if (e == cudaSuccess) e = gemv_attr<2>();
  if (e == cudaSuccess) e = gemv_attr<4>();
  if (e == cudaSuccess) e = gemv_attr<8>();
  if (e == cudaSuccess) e = gemv_attr<12>();
  if (e == cudaSuccess) e = gemv_attr<16>();
  if (e != cudaSuccess) return e;
  done |= uint64_t(1) << dev;
  return cudaSuccess;
}

template <int VPL>
static cudaError_t gemv_launch(const float* x, int nb, int K, const uint16_t* W, const uint16_t* bias, int rows,
                               int pre, int post, float* out, int out_stride, cudaStream_t s, int blocks) {
  const size_t smem = static_cast<size_t>(nb) * K * sizeof(float);
  cudaError_t e = small_kernels_set_attributes();
  if (e != cudaSuccess) return e;
  gemv_rows_kernel<VPL><<<blocks, 256, smem, s>>>(x, nb, K, W, bias, rows, pre, post, out, out_stride);
  return cudaGetLastError();
}

static cudaError_t gemv(const float* x, int B, int K, const uint16_t* W, const uint16_t* bias, int rows, int pre,
                        int post, float* out, int out_stride, cudaStream_t s) {
  if (K % 8 != 0) return cudaErrorInvalidValue;
  static int sms = 0;
  if (!sms) sms = device_sm_count();
  for (int b0 = 0; b0 < B; b0 += GEMV_MAX_B) {
    const int nb = B - b0 < GEMV_MAX_B ? B - b0 : GEMV_MAX_B;
    int blocks = (rows + 7) / 8;
    const int cap = sms * 8;
    if (blocks > cap) blocks = cap;
    const float* xb = x + static_cast<size_t>(b0) * K;
    float* ob = out + static_cast<size_t>(b0) * out_stride;
    cudaError_t e;
    const int vpl = (K / 8 + 31) / 32;
    switch (vpl <= 2 ? vpl : (vpl <= 4 ? 4 : (vpl <= 8 ? 8 : (vpl <= 12 ? 12 : (vpl <= 16 ? 16 : -1))))) {
      case 1: e = gemv_launch<1>(xb, nb, K, W, bias, rows, pre, post, ob, out_stride, s, blocks); break;
      case 2: e = gemv_launch<2>(xb, nb, K, W, bias, rows, pre, post, ob, out_stride, s, blocks); break;
      case 4: e = gemv_launch<4>(xb, nb, K, W, bias, rows, pre, post, ob, out_stride, s, blocks); break;
      case 8: e = gemv_launch<8>(xb, nb, K, W, bias, rows, pre, post, ob, out_stride, s, blocks); break;
      case 12: e = gemv_launch<12>(xb, nb, K, W, bias, rows, pre, post, ob, out_stride, s, blocks); break;
      case 16: e = gemv_launch<16>(xb, nb, K, W, bias, rows, pre, post, ob, out_stride, s, blocks); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ------------------------------------------------------------------ timestep embedding
// e = [cos(1000 t w_j), sin(1000 t w_j)], w_j = exp(-ln(10000) j / half)   (§前向传播流程)
__global__ void timestep_features_kernel(const float* __restrict__ t, int B, int C, float* __restrict__ e) {
  const int half = C / 2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B * half; i += gridDim.x * blockDim.x) {
    const int b = i / half, j = i - b * half;
    const float w = expf(-9.210340371976184f * static_cast<float>(j) / static_cast<float>(half));
    const float a = 1000.0f * t[b] * w;
    e[b * C + j] = cosf(a);
    e[b * C + half + j] = sinf(a);
  }
}

cudaError_t launch_timestep_features(const float* t, int B, int C, float* feat, cudaStream_t s) {
  timestep_features_kernel<<<(B * C / 2 + 255) / 256, 256, 0, s>>>(t, B, C, feat);
  return cudaGetLastError();
}

cudaError_t launch_timestep_mlp(const float* t, int B, const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                                const uint16_t* b2, int C, int D, float* feat, float* h1, float* temb, cudaStream_t s) {
  timestep_features_kernel<<<(B * C / 2 + 255) / 256, 256, 0, s>>>(t, B, C, feat);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = gemv(feat, B, C, w1, b1, D, 0, 1, h1, D, s);  // h1 = silu(W1 e + b1)
  if (e != cudaSuccess) return e;
  return gemv(h1, B, D, w2, b2, D, 0, 0, temb, D, s);  // temb = W2 h1 + b2
}

cudaError_t launch_modulation(const float* temb, int B, int D, const uint16_t* w, int rows, float* out,
                              cudaStream_t s) {
  return gemv(temb, B, D, w, nullptr, rows, 1, 0, out, rows, s);  // out[b, r] = W[r] . silu(temb[b])
}

// ------------------------------------------------------------------ patch embedding
// img[b, n, d] = sum_k W[d, k] patch(b, n)[k] + PE[(r0 + n / wp) * G + c0 + n % wp, d]
// patch vector index k = (py * p + px) * C + c  <->  latent[b, c, hp * p + py, wp * p + px]
__global__ void __launch_bounds__(128) patch_embed_kernel(const float* __restrict__ lat, int C, int H, int W, int p,
                                                          const uint16_t* __restrict__ wpe,
                                                          const uint16_t* __restrict__ pos, int G, int D,
                                                          uint16_t* __restrict__ out, int out_rows_per_batch,
                                                          int out_row_off) {
  __shared__ float patch[64];
  const int n = blockIdx.x, b = blockIdx.y;
  const int hpn = H / p, wpn = W / p;
  const int hp = n / wpn, wp = n - hp * wpn;
  const int KP = p * p * C;
  for (int k = threadIdx.x; k < KP; k += blockDim.x) {
    const int c = k % C, pq = k / C;
    const int py = pq / p, px = pq - py * p;
    patch[k] = lat[((static_cast<size_t>(b) * C + c) * H + hp * p + py) * W + wp * p + px];
  }
  __syncthreads();
  const int r0 = (G - hpn) / 2, c0 = (G - wpn) / 2;
  const size_t prow = static_cast<size_t>(r0 + hp) * G + c0 + wp;
  uint16_t* orow = out + (static_cast<size_t>(b) * out_rows_per_batch + out_row_off + n) * D;
  const int nvec = D / 8;
  for (int vi = threadIdx.x; vi < nvec; vi += blockDim.x) {
    const uint4 pu = *reinterpret_cast<const uint4*>(pos + prow * D + vi * 8);
    float acc[8] = {bf16_lo(pu.x), bf16_hi(pu.x), bf16_lo(pu.y), bf16_hi(pu.y),
                    bf16_lo(pu.z), bf16_hi(pu.z), bf16_lo(pu.w), bf16_hi(pu.w)};
    float mm[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int e = 0; e < 8; ++e) {
      const uint16_t* wr = wpe + static_cast<size_t>(vi * 8 + e) * KP;
      float a = 0.f;
      for (int k = 0; k < KP; ++k) a += __uint_as_float(static_cast<uint32_t>(wr[k]) << 16) * patch[k];
      mm[e] = a;
    }
    uint4 u;
    u.x = pack_bf16(mm[0] + acc[0], mm[1] + acc[1]);
    u.y = pack_bf16(mm[2] + acc[2], mm[3] + acc[3]);
    u.z = pack_bf16(mm[4] + acc[4], mm[5] + acc[5]);
    u.w = pack_bf16(mm[6] + acc[6], mm[7] + acc[7]);
    *reinterpret_cast<uint4*>(orow + vi * 8) = u;
  }
}

// Fast path for p*p*C = 16 (patch 2, 4 channels): a thread owns 8 output
// columns and keeps their 8 x 16 projection weights in registers; the block
// walks PE_TOK tokens whose patch vectors are staged in shared memory.
constexpr int PE_TOK = 32;
constexpr int PE_KP = 16;

__global__ void __launch_bounds__(128) patch_embed16_kernel(const float* __restrict__ lat, int C, int H, int W,
                                                            int p, const uint16_t* __restrict__ wpe,
                                                            const uint16_t* __restrict__ pos, int G, int D,
                                                            uint16_t* __restrict__ out, int out_rows_per_batch,
                                                            int out_row_off) {
  __shared__ float patch[PE_TOK][PE_KP];
  const int b = blockIdx.z;
  const int hpn = H / p, wpn = W / p, ntok = hpn * wpn;
  const int t0 = blockIdx.x * PE_TOK;
  for (int i = threadIdx.x; i < PE_TOK * PE_KP; i += blockDim.x) {
    const int tt = i / PE_KP, k = i - tt * PE_KP;
    const int n = t0 + tt;
    float v = 0.f;
    if (n < ntok) {
      const int hp = n / wpn, wp = n - hp * wpn;
      const int c = k % C, pq = k / C;
      const int py = pq / p, px = pq - py * p;
      v = lat[((static_cast<size_t>(b) * C + c) * H + hp * p + py) * W + wp * p + px];
    }
    patch[tt][k] = v;
  }
  __syncthreads();
  const int vi = blockIdx.y * blockDim.x + threadIdx.x;
  if (vi >= D / 8) return;
  float wv[8][PE_KP];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint4* wr = reinterpret_cast<const uint4*>(wpe + static_cast<size_t>(vi * 8 + e) * PE_KP);
    const uint4 a = wr[0], c = wr[1];
    const uint32_t q[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      wv[e][2 * k] = bf16_lo(q[k]);
      wv[e][2 * k + 1] = bf16_hi(q[k]);
    }
  }
  const int r0 = (G - hpn) / 2, c0 = (G - wpn) / 2;
  for (int tt = 0; tt < PE_TOK; ++tt) {
    const int n = t0 + tt;
    if (n >= ntok) break;
    const int hp = n / wpn, wp = n - hp * wpn;
    const size_t prow = static_cast<size_t>(r0 + hp) * G + c0 + wp;
    const uint4 pu = *reinterpret_cast<const uint4*>(pos + prow * D + vi * 8);
    const float pe[8] = {bf16_lo(pu.x), bf16_hi(pu.x), bf16_lo(pu.y), bf16_hi(pu.y),
                         bf16_lo(pu.z), bf16_hi(pu.z), bf16_lo(pu.w), bf16_hi(pu.w)};
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < PE_KP; ++k) a += wv[e][k] * patch[tt][k];
      o[e] = a + pe[e];
    }
    uint4 u;
    u.x = pack_bf16(o[0], o[1]);
    u.y = pack_bf16(o[2], o[3]);
    u.z = pack_bf16(o[4], o[5]);
    u.w = pack_bf16(o[6], o[7]);
    *reinterpret_cast<uint4*>(out + (static_cast<size_t>(b) * out_rows_per_batch + out_row_off + n) * D + vi * 8) = u;
  }
}

cudaError_t launch_patch_embed(const float* lat, int B, int C, int H, int W, int p, const uint16_t* w_pe,
                               const uint16_t* pos, int G, int D, uint16_t* out, int out_rows_per_batch,
                               int out_row_off, cudaStream_t s) {
  if (p * p * C > 64 || D % 8 != 0) return cudaErrorInvalidValue;
  if (p * p * C == PE_KP) {
    const int ntok = (H / p) * (W / p);
    dim3 grid((ntok + PE_TOK - 1) / PE_TOK, (D / 8 + 127) / 128, B);
    patch_embed16_kernel<<<grid, 128, 0, s>>>(lat, C, H, W, p, w_pe, pos, G, D, out, out_rows_per_batch,
                                              out_row_off);
    return cudaGetLastError();
  }
  dim3 grid((H / p) * (W / p), B);
  patch_embed_kernel<<<grid, 128, 0, s>>>(lat, C, H, W, p, w_pe, pos, G, D, out, out_rows_per_batch, out_row_off);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ output stage on the tensor cores
// The pre-final modulation folds into the projection: with z = x (1 + sc) + sh,
// o[k] = W[k] . z = (W[k] * (1 + sc)) . x + W[k] . sh.  output_fold_kernel
// writes, per sample b, W'_b = bf16(W * (1 + sc_b)) into rows [0, KP) of a
// 256-row block (the rest stays zero, so a 256-wide GEMM tile reads only
// zeros there) and bias_b[k] = W[k] . sh_b (fp32); one CTA per (b, k).
__global__ void __launch_bounds__(256) output_fold_kernel(const uint16_t* __restrict__ wout, int KP, int D,
                                                          const float* __restrict__ scale,
                                                          const float* __restrict__ shift, int mod_stride, int B,
                                                          uint16_t* __restrict__ wfold, float* __restrict__ bias) {
  __shared__ float part[8];
  const int b = blockIdx.x / KP, k = blockIdx.x - b * KP;
  const float* sc = scale + static_cast<size_t>(b) * mod_stride;
  const float* sh = shift + static_cast<size_t>(b) * mod_stride;
  const uint16_t* wr = wout + static_cast<size_t>(k) * D;
  uint16_t* dr = wfold + (static_cast<size_t>(b) * 256 + k) * D;
  float acc = 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const float w = __uint_as_float(static_cast<uint32_t>(wr[d]) << 16);
    dr[d] = static_cast<uint16_t>(pack_bf16(w * (1.0f + sc[d]), 0.f) & 0xFFFFu);
    acc = fmaf(w, sh[d], acc);
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += part[i];
    bias[b * KP + k] = t;
  }
}

// velocity[b, c, hp p + py, wp p + px] = o[b, n, (py p + px) C + c] + bias_b[...]
// (the unpatchify of the model's output stage), o the fp32 GEMM output [B * Ni, KP]
__global__ void output_scatter_kernel(const float* __restrict__ o, const float* __restrict__ bias, int B, int hp,
                                      int wp, int p, int C, float* __restrict__ vel) {
  const int KP = p * p * C, Ni = hp * wp;
  const int total = B * Ni * KP;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int k = i % KP, n = (i / KP) % Ni, b = i / (KP * Ni);
  const int c = k % C, pq = k / C, py = pq / p, px = pq - py * p;
  const int ph = n / wp, pw = n - ph * wp;
  const int H = hp * p, W = wp * p;
  vel[((static_cast<size_t>(b) * C + c) * H + ph * p + py) * W + pw * p + px] = o[i] + bias[b * KP + k];
}

cudaError_t launch_output_fold(const uint16_t* w_out, int KP, int D, const float* scale, const float* shift,
                               int mod_stride, int B, uint16_t* wfold, float* bias, cudaStream_t s) {
  output_fold_kernel<<<B * KP, 256, 0, s>>>(w_out, KP, D, scale, shift, mod_stride, B, wfold, bias);
  return cudaGetLastError();
}

cudaError_t launch_output_scatter(const float* o, const float* bias, int B, int hp, int wp, int p, int C, float* vel,
                                  cudaStream_t s) {
  const int total = B * hp * wp * p * p * C;
  output_scatter_kernel<<<(total + 255) / 256, 256, 0, s>>>(o, bias, B, hp, wp, p, C, vel);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ fill (model time of a CFG batch)
__global__ void fill_kernel(float* __restrict__ dst, int n, float value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = value;
}

cudaError_t launch_fill(float* dst, int n, float value, cudaStream_t s) {
  fill_kernel<<<(n + 255) / 256, 256, 0, s>>>(dst, n, value);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ SiLU, fp32 -> bf16 (GEMM operand)
__global__ void silu_bf16_kernel(const float* __restrict__ x, int n, uint16_t* __restrict__ y) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = x[i];
    y[i] = static_cast<uint16_t>(pack_bf16(a / (1.0f + __expf(-a)), 0.f) & 0xFFFFu);
  }
}

cudaError_t launch_silu_bf16(const float* x, int n, uint16_t* y, cudaStream_t s) {
  silu_bf16_kernel<<<(n + 255) / 256, 256, 0, s>>>(x, n, y);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ Euler + CFG
// The two halves of the velocity come as separate pointers, so the uncond
// or the text half may live in another GPU's memory (the two-GPU CFG split
// reads its peer's half here over NVLink, no separate exchange copy).
__global__ void euler_cfg_kernel(float* __restrict__ x, const float* __restrict__ vu_p,
                                 const float* __restrict__ vc_p, int64_t n_total, float g, float dt) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n_total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float vu = vu_p[i];
    const float vc = vc_p[i];
    x[i] = x[i] + dt * (vu + g * (vc - vu));
  }
}

cudaError_t launch_euler_cfg2(float* lat, const float* v_uncond, const float* v_text, int64_t n, float g, float sigma,
                              float sigma_next, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int blocks = static_cast<int>((n + 255) / 256);
  if (blocks > 4096) blocks = 4096;
  euler_cfg_kernel<<<blocks, 256, 0, s>>>(lat, v_uncond, v_text, n, g, sigma_next - sigma);
  return cudaGetLastError();
}

cudaError_t launch_euler_cfg(float* lat, const float* v, int Bi, int64_t per_sample, float g, float sigma,
                             float sigma_next, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(Bi) * per_sample;
  return launch_euler_cfg2(lat, v, v + n, n, g, sigma, sigma_next, s);
}

}  // namespace af
