// gemm.cu -- persistent tcgen05 GEMM for sm_100a with fused epilogues.
//
//   acc[M, N] = A[M, K] * W[N, K]^T      (bf16 operands, fp32 accumulation in TMEM)
//
// These are the bias-free projections of the AuraFlow blocks: fused QKV and
// added-KV ("Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南",
// §模型概述 and §注意力处理器与 QKV 融合), the output projections and the
// SiLU-gated FFN (§FeedForward), gated by adaLN-Zero (§联合注意力块).
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: A tile 128x64 and W tile 256x64 per k-block
//               (one box each: the TMA engine's cost is per box, so the W
//               tile is never split), 128-byte swizzled, into a 4-stage
//               shared-memory ring.
//   warp 1      allocates 512 TMEM columns; one thread issues
//               tcgen05.mma (M=128, N=256, K=16) into one of two 256-column
//               fp32 accumulators, committing each stage back to the producer.
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane quarter (one thread =
//               one output row), fused epilogue; the outputs (and the gated
//               residual) move through the warp's shared-memory boxes by TMA
//               in 32 x 32 chunks where the layout allows, else by per-thread
//               stores; the other accumulator is being filled meanwhile.
// The large projections (M >= 1024) run the CTA-pair form below
// (gemm_tcgen05_pair: 256 x 256 tiles, cta_group::2) with the same epilogues.
// Every wait is bounded (ptx.cuh); a timeout sets the error word and the CTA
// drains its outstanding copies and MMAs before releasing TMEM.
#include <cstdio>
#include <mutex>

#include <cudaTypedefs.h>

#include "af_internal.h"
#include "ptx.cuh"

namespace af {

// ----------------------------------------------------------------- host: TMA descriptors

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_tmap_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer, bool bytes, int swizzle_bytes) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = enc(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_3d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                    uint64_t s2_bytes, uint32_t b0, uint32_t b1, uint32_t b2, int swizzle_bytes) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// ----------------------------------------------------------------- device: tiles

constexpr uint32_t A_STAGE_BYTES = GEMM_BM * GEMM_BK * 2;  // 16 KB
constexpr uint32_t B_STAGE_BYTES = GEMM_BN * GEMM_BK * 2;  // 32 KB
// Tile order: n-tiles are taken in groups of `group_n`; inside a group the
// tiles run m-major, so the CTAs in flight share a few A panels and the
// group's weight panels stay resident in L2.
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int group_n, int& mb, int& nb) {
  const int per_group = group_n * num_m;
  const int g = t / per_group;
  const int r = t - g * per_group;
  const int n_first = g * group_n;
  const int gw = min(group_n, num_n - n_first);
  mb = r / gw;
  nb = n_first + (r - mb * gw);
}

// silu(a) = a * sigmoid(a); the fast division (2 ulp) is far below the bf16 output rounding
__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u;
    u.x = pack_bf16(v[8 * i + 0], v[8 * i + 1]);
    u.y = pack_bf16(v[8 * i + 2], v[8 * i + 3]);
    u.z = pack_bf16(v[8 * i + 4], v[8 * i + 5]);
    u.w = pack_bf16(v[8 * i + 6], v[8 * i + 7]);
    d[i] = u;
  }
}

// Store `n` (< 32 allowed at a ragged right edge) bf16 values.
__device__ __forceinline__ void store_bf16_n(uint16_t* dst, const float* v, int n) {
  if (n >= 32 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
    store_bf16x32(dst, v);
    return;
  }
  for (int i = 0; i < n && i < 32; ++i) {
    uint32_t p = pack_bf16(v[i], 0.f);
    dst[i] = static_cast<uint16_t>(p & 0xFFFFu);
  }
}

// 32 accumulator columns of this thread's row as floats.  For the 8-bit
// GEMM (p.w_scale set) the fp32 sums of e4m3 products are rescaled by the
// row's activation scale a_s and the scales of weight rows [wrow, wrow + 32).
__device__ __forceinline__ void acc_load32(const GemmParams& p, uint32_t taddr, float a_s, int wrow, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_wait_ld();
  if (p.w_scale) {
    const float4* ws = reinterpret_cast<const float4*>(p.w_scale + wrow);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 w4 = ws[i];
      v[4 * i + 0] = __uint_as_float(r[4 * i + 0]) * (a_s * w4.x);
      v[4 * i + 1] = __uint_as_float(r[4 * i + 1]) * (a_s * w4.y);
      v[4 * i + 2] = __uint_as_float(r[4 * i + 2]) * (a_s * w4.z);
      v[4 * i + 3] = __uint_as_float(r[4 * i + 3]) * (a_s * w4.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  }
}

// Gated-residual epilogue with TMA-staged residual tiles.  Each epilogue warp
// owns 32 output rows of a tile and walks them in 32-column chunks; the
// residual box of a chunk (32 x 32 bf16, 64-byte swizzle) is loaded by TMA
// into one of the warp's two shared-memory buffers one chunk ahead (the first
// before the accumulator is ready), updated in place (thread = row, so the
// reads follow the TMEM lane layout without bank conflicts) and written back
// by a TMA store: coalesced global traffic instead of every thread walking
// its own row.
struct ResStage {
  uint32_t buf;            // this warp's two 2 KB boxes (1024-byte aligned)
  uint32_t bar;            // their two mbarriers (8 bytes apart)
  uint32_t issued, used;   // loads issued / consumed: buffer = n & 1, parity = (n >> 1) & 1
  volatile int* abort;
  bool failed;
};
constexpr uint32_t RES_BOX_BYTES = 32 * 32 * 2;

// Load the residual box at (col, row) into the next buffer (lane 0 issues).
__device__ __forceinline__ void res_issue(ResStage& rs, const CUtensorMap* tm, int col, int row, bool lane0) {
  const uint32_t k = rs.issued & 1u;
  if (lane0) {
    bulk_wait_group_read0();  // the store that last read this buffer has read it
    mbar_arrive_expect_tx(rs.bar + 8 * k, RES_BOX_BYTES);
    tma_load_2d(rs.buf + k * RES_BOX_BYTES, tm, rs.bar + 8 * k, col, row);
  }
  ++rs.issued;
}

// Wait for the oldest issued box; its shared-memory address (0 on a timeout).
__device__ __forceinline__ uint32_t res_take(ResStage& rs, int* err) {
  const uint32_t n = rs.used++;
  const uint32_t k = n & 1u;
  const bool got = mbar_wait(rs.bar + 8 * k, (n >> 1) & 1u, err, rs.abort);
  if (!__all_sync(0xffffffffu, got)) {
    rs.failed = true;
    return 0;
  }
  return rs.buf + k * RES_BOX_BYTES;
}

// Before the warp leaves: its stores have completed and no box load is still
// in flight (an abandoned prefetch lands first; bounded waits).
__device__ __forceinline__ void res_drain(ResStage& rs, bool lane0) {
  if (lane0) bulk_wait_group0();
  volatile int never = 0;
  while (rs.used < rs.issued) {
    const uint32_t n = rs.used++;
    mbar_wait(rs.bar + 8 * (n & 1u), (n >> 1) & 1u, nullptr, &never, 100000000ull);
  }
  __syncwarp();
}

// Outputs through shared memory: a warp writes one 32 x 32 bf16 chunk of its
// rows (thread = row, as read from TMEM) into the next of its two boxes and
// lane 0 stores the box with one TMA store, so the global writes are whole
// 64-byte row segments instead of every thread writing its own row; the
// store that last read the box (two chunks earlier) has read it first.
__device__ __forceinline__ uint32_t box_put(ResStage& rs, int lane, const float (&v)[32]) {
  const uint32_t box = rs.buf + (rs.issued & 1u) * RES_BOX_BYTES;
  if (lane == 0) bulk_wait_group_read1();
  __syncwarp();
  const uint32_t rowa = box + static_cast<uint32_t>(lane) * 64;
  const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = make_uint4(pack_bf16(v[8 * q + 0], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                               pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
    sts128(rowa + ((static_cast<uint32_t>(q) ^ swz) << 4), u);
  }
  fence_proxy_async_smem();
  __syncwarp();
  ++rs.issued;  // no load uses the box: issued and used advance together
  ++rs.used;
  return box;
}

// QK-norm epilogue for one output row: the tile's columns hold (256 / hd)
// heads of Q, K or V.  Q and K are LayerNorm-ed over each head's hd values,
// V is stored as is.  With rs set (hd >= 32 and the warp's 32 rows valid
// rows of sample b0, from token tok0 on) the normalised heads leave through
// shared memory by TMA (tensor map tmo over q, k, v: [3][B H n_total][hd]).
__device__ __forceinline__ void epilogue_qkv(const GemmParams& p, uint32_t tbase, int n0, bool row_ok, int b,
                                             int n_in, float a_s, ResStage* rs = nullptr,
                                             const CUtensorMap* tmo = nullptr, int lane = 0, int b0 = 0,
                                             int tok0 = 0) {
  const int hd = p.hd;
  const int tok = p.qkv_row_off + n_in;
  if (hd >= 32) {
    const int chunks = hd >> 5;
    for (int h0 = 0; h0 < GEMM_BN; h0 += hd) {
      const int col = n0 + h0;
      if (col >= p.N) break;                       // uniform across the warp
      const int which = col / p.D;
      const int head = (col - which * p.D) / hd;
      uint16_t* base = which == 0 ? p.q : (which == 1 ? p.k : p.v);
      uint16_t* dst = base + ((static_cast<size_t>(b) * p.heads + head) * p.n_total + tok) * hd;
      float mean = 0.f, rstd = 1.f;
      float v[32];
      if (which < 2) {
        // one pass over TMEM: sums of (x - k) and (x - k)^2 with the shift k =
        // the head's first value, so E[x^2] - mean^2 does not cancel when the
        // mean is large against the spread
        float k = 0.f, s1 = 0.f, s2 = 0.f;
        for (int c = 0; c < chunks; ++c) {
          acc_load32(p, tbase + h0 + c * 32, a_s, col + c * 32, v);
          if (c == 0) k = v[0];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float d = v[j] - k;
            s1 += d;
            s2 += d * d;
          }
        }
        const float m1 = s1 / hd;
        mean = k + m1;
        rstd = rsqrtf(fmaxf(s2 / hd - m1 * m1, 0.f) + p.eps);
      }
      const int drow0 = (b0 * p.heads + head) * p.n_total + tok0;  // the warp's first destination row
      for (int c = 0; c < chunks; ++c) {
        acc_load32(p, tbase + h0 + c * 32, a_s, col + c * 32, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (v[j] - mean) * rstd;
        if (rs) {
          const uint32_t box = box_put(*rs, lane, v);
          if (lane == 0) {
            tma_store_3d(tmo, box, c * 32, drow0, which);
            bulk_commit_group();
          }
        } else if (row_ok) {
          store_bf16x32(dst + c * 32, v);
        }
      }
    }
  } else {
    // small heads (hd in {8, 16}): each 32-column chunk holds 32 / hd heads
    for (int c = 0; c < GEMM_BN / 32; ++c) {
      if (n0 + c * 32 >= p.N) break;
      float r[32];
      acc_load32(p, tbase + c * 32, a_s, n0 + c * 32, r);
      for (int s0 = 0; s0 < 32; s0 += hd) {
        const int col = n0 + c * 32 + s0;
        if (col >= p.N) break;
        const int which = col / p.D;
        const int head = (col - which * p.D) / hd;
        uint16_t* base = which == 0 ? p.q : (which == 1 ? p.k : p.v);
        uint16_t* dst = base + ((static_cast<size_t>(b) * p.heads + head) * p.n_total + tok) * hd;
        float v[32];
        float mean = 0.f, rstd = 1.f;
        if (which < 2) {
          float s = 0.f;
          for (int j = 0; j < hd; ++j) s += r[s0 + j];
          mean = s / hd;
          float ss = 0.f;
          for (int j = 0; j < hd; ++j) {
            const float d = r[s0 + j] - mean;
            ss += d * d;
          }
          rstd = rsqrtf(ss / hd + p.eps);
        }
        for (int j = 0; j < hd; ++j) v[j] = (r[s0 + j] - mean) * rstd;
        if (row_ok)
          for (int j = 0; j < hd; ++j) dst[j] = static_cast<uint16_t>(pack_bf16(v[j], 0.f) & 0xFFFFu);
      }
    }
  }
}

// Epilogue of one accumulator tile for one output row (thread = TMEM lane):
// tbase addresses this warp's 32-lane quarter of the accumulator, m0 is the
// first GEMM row of the tile half held in this CTA's TMEM, nb the n-tile.
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, uint32_t tbase, int m0, int nb, int row_in_tile,
                                              ResStage* rs = nullptr, const CUtensorMap* tmo = nullptr) {
  const int r = m0 + row_in_tile;
  const bool row_ok = r < p.M;
  const int b = r / p.rows_per_batch;
  const int n_in = r - b * p.rows_per_batch;
  const size_t orow = static_cast<size_t>(b) * p.out_rows_per_batch + p.out_row_off + n_in;
  const float a_s = (p.a_scale && row_ok) ? p.a_scale[r] : 1.0f;

  const int lane = row_in_tile & 31;
  const int r0 = m0 + (row_in_tile & ~31);  // the warp's first row
  if (p.mode == EPI_QKV) {
    // by TMA when the warp's 32 rows are valid rows of one sample
    const int b0 = r0 / p.rows_per_batch;
    const bool tma = p.res_tma && p.hd >= 32 && r0 + 31 < p.M && (r0 + 31) / p.rows_per_batch == b0;
    epilogue_qkv(p, tbase, nb * GEMM_BN, row_ok, b, n_in, a_s, tma ? rs : nullptr, tmo, lane, b0,
                 p.qkv_row_off + (r0 - b0 * p.rows_per_batch));
  } else if (p.mode == EPI_GATE_RES && p.res_tma) {
    // chunk 0's box was issued by the caller before the accumulator was ready
    const int col0 = nb * GEMM_BN;
    const int wrow0 = r0;
    const int nch = min(GEMM_BN / 32, (p.N - col0 + 31) / 32);
    const float* gb = row_ok ? p.gate + static_cast<size_t>(b) * p.gate_stride : nullptr;
    const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      if (c + 1 < nch) res_issue(*rs, tmo, col0 + 32 * (c + 1), wrow0, lane == 0);
      float v[32];
      acc_load32(p, tbase + c * 32, a_s, col0 + c * 32, v);
      const uint32_t box = res_take(*rs, p.err);
      if (!box) return;
      const uint32_t rowa = box + static_cast<uint32_t>(lane) * 64;
      uint4 xv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) xv[q] = lds128(rowa + ((static_cast<uint32_t>(q) ^ swz) << 4));
      if (gb) {
        const float* g = gb + col0 + c * 32;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 g0 = *reinterpret_cast<const float4*>(g + 8 * i);
          const float4 g1 = *reinterpret_cast<const float4*>(g + 8 * i + 4);
          v[8 * i + 0] = bf16_lo(xv[i].x) + g0.x * v[8 * i + 0];
          v[8 * i + 1] = bf16_hi(xv[i].x) + g0.y * v[8 * i + 1];
          v[8 * i + 2] = bf16_lo(xv[i].y) + g0.z * v[8 * i + 2];
          v[8 * i + 3] = bf16_hi(xv[i].y) + g0.w * v[8 * i + 3];
          v[8 * i + 4] = bf16_lo(xv[i].z) + g1.x * v[8 * i + 4];
          v[8 * i + 5] = bf16_hi(xv[i].z) + g1.y * v[8 * i + 5];
          v[8 * i + 6] = bf16_lo(xv[i].w) + g1.z * v[8 * i + 6];
          v[8 * i + 7] = bf16_hi(xv[i].w) + g1.w * v[8 * i + 7];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 u = make_uint4(pack_bf16(v[8 * q + 0], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                     pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
          sts128(rowa + ((static_cast<uint32_t>(q) ^ swz) << 4), u);
        }
      }
      // rows past M (no gate) keep the loaded fill; the store clips them
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tmo, box, col0 + 32 * c, wrow0);
        bulk_commit_group();
      }
    }
  } else if (p.mode == EPI_SWIGLU) {
    const int col0 = nb * 128;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      // weight rows of the interleaved pair: W1 at nb*256 + [0, 128), W2 at nb*256 + 128 + [0, 128)
      float va[32], v[32];
      acc_load32(p, tbase + c * 32, a_s, nb * 256 + c * 32, va);
      acc_load32(p, tbase + 128 + c * 32, a_s, nb * 256 + 128 + c * 32, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = silu_f(va[j]) * v[j];
      const int col = col0 + c * 32;
      if (p.res_tma) {  // rows past M and columns past N are clipped by the tensor map
        if (col < p.N) {
          const uint32_t box = box_put(*rs, lane, v);
          if (lane == 0) {
            tma_store_2d(tmo, box, col, r0);
            bulk_commit_group();
          }
        }
      } else if (row_ok && col < p.N) {
        store_bf16_n(p.out + orow * p.ldo + col, v, p.N - col);
      }
    }
  } else {
    const int col0 = nb * GEMM_BN;
#pragma unroll 1
    for (int c = 0; c < GEMM_BN / 32; ++c) {
      const int col = col0 + c * 32;
      if (col >= p.N) break;  // uniform across the warp
      float v[32];
      acc_load32(p, tbase + c * 32, a_s, col, v);
      if (!row_ok) continue;
      const int n = min(32, p.N - col);
      if (p.mode == EPI_STORE_F32) {
        float* df = p.out_f32 + orow * p.ldo + col;
        if (n == 32) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(df)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
          for (int j = 0; j < n; ++j) df[j] = v[j];
        }
        continue;
      }
      uint16_t* dst = p.out + orow * p.ldo + col;
      if (p.mode == EPI_GATE_RES) {
        const float* g = p.gate + static_cast<size_t>(b) * p.gate_stride + col;
        if (n == 32) {
          const uint4* xs = reinterpret_cast<const uint4*>(dst);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 xv = xs[i];
            const float4 g0 = *reinterpret_cast<const float4*>(g + 8 * i);
            const float4 g1 = *reinterpret_cast<const float4*>(g + 8 * i + 4);
            v[8 * i + 0] = bf16_lo(xv.x) + g0.x * v[8 * i + 0];
            v[8 * i + 1] = bf16_hi(xv.x) + g0.y * v[8 * i + 1];
            v[8 * i + 2] = bf16_lo(xv.y) + g0.z * v[8 * i + 2];
            v[8 * i + 3] = bf16_hi(xv.y) + g0.w * v[8 * i + 3];
            v[8 * i + 4] = bf16_lo(xv.z) + g1.x * v[8 * i + 4];
            v[8 * i + 5] = bf16_hi(xv.z) + g1.y * v[8 * i + 5];
            v[8 * i + 6] = bf16_lo(xv.w) + g1.z * v[8 * i + 6];
            v[8 * i + 7] = bf16_hi(xv.w) + g1.w * v[8 * i + 7];
          }
        } else {
          for (int j = 0; j < n; ++j) v[j] = __uint_as_float(static_cast<uint32_t>(dst[j]) << 16) + g[j] * v[j];
        }
      }
      store_bf16_n(dst, v, n);
    }
  }
}


// FP8 = false: bf16 operands, 64 K elements (128 bytes) per stage, kind::f16.
// FP8 = true:  e4m3 operands, 128 K elements (128 bytes) per stage,
//              kind::f8f6f4; the epilogue applies the row / column scales.
template <bool FP8>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmO, const GemmParams p) {
  constexpr int KB = FP8 ? 2 * GEMM_BK : GEMM_BK;  // K elements per stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + GEMM_STAGES * A_STAGE_BYTES;
  uint8_t* sR = sB + GEMM_STAGES * B_STAGE_BYTES;  // residual boxes, 2 per epilogue warp
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + GEMM_RES_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + GEMM_STAGES;
  uint64_t* acc_full = bars + 2 * GEMM_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint64_t* res_bar = mma_done + 1;  // [epilogue warp][2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_bar + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GEMM_STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 128);
    }
    mbar_init(smem_u32(mma_done), 1);
    for (int i = 0; i < 8; ++i) mbar_init(smem_u32(&res_bar[i]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int num_k = (p.K + KB - 1) / KB;
  volatile int never = 0;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p.num_m_tiles, p.num_n_tiles, p.group_n, mb, nb);
        const int wrow = nb * GEMM_BN;  // SwiGLU: W1/W2 are interleaved per 128 rows in the pack
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.err, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, A_STAGE_BYTES + B_STAGE_BYTES);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          const uint32_t a_dst = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * B_STAGE_BYTES);
          tma_load_2d(a_dst, &tmA, fb, kb * KB, mb * GEMM_BM);
          tma_load_2d(b_dst, &tmB, fb, kb * KB, wrow);
          if (++stage == GEMM_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // drain copies still in flight before the CTA exits
        for (int s = 0; s < GEMM_STAGES; ++s)
          if (armed & (1u << s))
            mbar_wait(smem_u32(&full[s]), (armed_par >> s) & 1u, nullptr, &never, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc =
          FP8 ? make_idesc_e4m3(GEMM_BM, GEMM_BN, false, false) : make_idesc_bf16(GEMM_BM, GEMM_BN, false, false);
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * GEMM_BN;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, p.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = make_sdesc(smem_u32(sA + stage * A_STAGE_BYTES), 16, 1024, SWZ_128B);
          const uint64_t bdesc = make_sdesc(smem_u32(sB + stage * B_STAGE_BYTES), 16, 1024, SWZ_128B);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
            if constexpr (FP8)
              mma_e4m3_ss(d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
            else
              mma_bf16_ss(d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&empty[stage]));
          if (++stage == GEMM_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&acc_full[acc]));
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      // all MMAs issued by this thread must finish before TMEM is released
      mma_commit(smem_u32(mma_done));
      mbar_wait(smem_u32(mma_done), 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ---------------------------------------------------------- epilogue warps
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const bool res = p.mode == EPI_GATE_RES && p.res_tma;
    ResStage rs{smem_u32(sR) + static_cast<uint32_t>(warp - 2) * 2 * RES_BOX_BYTES,
                smem_u32(&res_bar[2 * (warp - 2)]), 0, 0, abort_flag, false};
    uint32_t acc = 0, acc_phase = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, p.num_m_tiles, p.num_n_tiles, p.group_n, mb, nb);
      if (res) res_issue(rs, &tmO, nb * GEMM_BN, mb * GEMM_BM + quarter * 32, lane == 0);
      const bool got = mbar_wait(smem_u32(&acc_full[acc]), acc_phase, p.err, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + acc * GEMM_BN + (static_cast<uint32_t>(quarter * 32) << 16);
      epilogue_tile(p, tbase, mb * GEMM_BM, nb, row_in_tile, &rs, &tmO);
      if (rs.failed) break;
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[acc]));
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
    res_drain(rs, lane == 0);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------- CTA-pair variant
// Two CTAs of a cluster compute one 256 x 256 tile with tcgen05.mma.cta_group::2:
// each CTA loads its 128 rows of A and its 128-row half of the W tile (32 KB
// per stage instead of 48 KB for the same FLOPs per SM, so the TMA engine
// keeps up with the tensor core), the leader CTA issues the M = 256 MMAs
// and its commits arrive on both CTAs' barriers; each CTA's epilogue warps
// read the 128 x 256 accumulator half in their own TMEM.  The TMA loads of
// both CTAs complete on the leader's stage barrier; the follower's epilogue
// warps release the accumulator on the leader's barrier.
constexpr int G2_STAGES = 6;
constexpr uint32_t G2_A_BYTES = 128 * GEMM_BK * 2;  // 16 KB
constexpr uint32_t G2_B_BYTES = 128 * GEMM_BK * 2;  // 16 KB
constexpr int GEMM2_SMEM = G2_STAGES * (G2_A_BYTES + G2_B_BYTES) + GEMM_RES_BYTES + 1024 + 1024;

//
// Grouped mode: a second problem (tensor maps tmA1 / tmB1, parameters p1)
// with its own A, W, epilogue and output rides in the same persistent
// launch; its tiles follow the first problem's in the tile order (the joint
// block's text-stream projections after the image-stream ones, filling the
// image GEMM's last wave instead of a launch of their own).  p1.num_tiles = 0
// for a single problem, and GROUPED = false compiles the second problem out.
template <bool FP8, bool GROUPED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_tcgen05_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmA1,
                      const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmO1,
                      const __grid_constant__ GemmParams p, const __grid_constant__ GemmParams p1) {
  constexpr int KB = FP8 ? 2 * GEMM_BK : GEMM_BK;  // K elements per stage (128 bytes per row)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + G2_STAGES * G2_A_BYTES;
  uint8_t* sR = sB + G2_STAGES * G2_B_BYTES;     // residual boxes, 2 per epilogue warp
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + GEMM_RES_BYTES);
  uint64_t* full = bars;                         // [G2_STAGES], used in the leader
  uint64_t* empty = bars + G2_STAGES;            // [G2_STAGES], both CTAs
  uint64_t* acc_full = bars + 2 * G2_STAGES;     // [2], both CTAs
  uint64_t* acc_empty = acc_full + 2;            // [2], used in the leader
  uint64_t* mma_done = acc_empty + 2;
  uint64_t* res_bar = mma_done + 1;              // [epilogue warp][2], per CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_bar + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cl = blockIdx.x >> 1;
  const int ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G2_STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 8);  // 4 epilogue warps in each CTA
    }
    mbar_init(smem_u32(mma_done), 1);
    for (int i = 0; i < 8; ++i) mbar_init(smem_u32(&res_bar[i]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the partner's barriers exist before anything signals them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total_tiles = GROUPED ? p.num_tiles + p1.num_tiles : p.num_tiles;
  volatile int never = 0;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int t = cl; t < total_tiles && ok; t += ncl) {
        const bool second = GROUPED && t >= p.num_tiles;
        const GemmParams& q = second ? p1 : p;
        const CUtensorMap* ta = second ? &tmA1 : &tmA;
        const CUtensorMap* tb = second ? &tmB1 : &tmB;
        int mb, nb;
        tile_coords(second ? t - p.num_tiles : t, q.num_m_tiles, q.num_n_tiles, q.group_n, mb, nb);
        const int arow = mb * 256 + static_cast<int>(rank) * 128;
        const int wrow = nb * GEMM_BN + static_cast<int>(rank) * 128;
        const int num_k = (q.K + KB - 1) / KB;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.err, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_u32(&full[stage]);
          if (leader) mbar_arrive_expect_tx(fb_local, 2 * (G2_A_BYTES + G2_B_BYTES));
          const uint32_t fb = mapa_shared(fb_local, 0);
          tma_load_2d_pair(smem_u32(sA + stage * G2_A_BYTES), ta, fb, kb * KB, arow);
          tma_load_2d_pair(smem_u32(sB + stage * G2_B_BYTES), tb, fb, kb * KB, wrow);
          issued = true;
          if (++stage == G2_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && issued) {  // let copies still in flight land before the CTA leaves
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = FP8 ? make_idesc_e4m3(256, GEMM_BN, false, false) : make_idesc_bf16(256, GEMM_BN, false, false);
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int t = cl; t < total_tiles && ok; t += ncl) {
        if (!mbar_wait(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * GEMM_BN;
        const int num_k = (((GROUPED && t >= p.num_tiles) ? p1.K : p.K) + KB - 1) / KB;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, p.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = make_sdesc(smem_u32(sA + stage * G2_A_BYTES), 16, 1024, SWZ_128B);
          const uint64_t bdesc = make_sdesc(smem_u32(sB + stage * G2_B_BYTES), 16, 1024, SWZ_128B);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
            if constexpr (FP8)
              mma_e4m3_ss_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
            else
              mma_bf16_ss_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit_pair(smem_u32(&empty[stage]), 0x3);
          if (++stage == G2_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(smem_u32(&acc_full[acc]), 0x3);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      mma_commit_pair(smem_u32(mma_done), 0x1);
      mbar_wait(smem_u32(mma_done), 0, nullptr, &never, 100000000ull);
    }
  } else {
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    ResStage rs{smem_u32(sR) + static_cast<uint32_t>(warp - 2) * 2 * RES_BOX_BYTES,
                smem_u32(&res_bar[2 * (warp - 2)]), 0, 0, abort_flag, false};
    uint32_t acc = 0, acc_phase = 0;
    for (int t = cl; t < total_tiles; t += ncl) {
      const bool second = GROUPED && t >= p.num_tiles;
      const GemmParams& q = second ? p1 : p;
      const CUtensorMap* to = second ? &tmO1 : &tmO;
      int mb, nb;
      tile_coords(second ? t - p.num_tiles : t, q.num_m_tiles, q.num_n_tiles, q.group_n, mb, nb);
      const int m0 = mb * 256 + static_cast<int>(rank) * 128;
      if (q.mode == EPI_GATE_RES && q.res_tma) res_issue(rs, to, nb * GEMM_BN, m0 + quarter * 32, lane == 0);
      const bool got = mbar_wait(smem_u32(&acc_full[acc]), acc_phase, p.err, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + acc * GEMM_BN + (static_cast<uint32_t>(quarter * 32) << 16);
      epilogue_tile(q, tbase, m0, nb, row_in_tile, &rs, to);
      if (rs.failed) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(smem_u32(&acc_empty[acc]));
        else
          mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
      }
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
    res_drain(rs, lane == 0);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its partner may still signal it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ----------------------------------------------------------------- host launch

// Opt the kernels into their dynamic shared memory, once per device (a plain
// host call, never made while a stream is being captured after this ran).
cudaError_t gemm_set_attributes() {
  static uint64_t done = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if ((done >> dev) & 1u) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gemm_tcgen05<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tcgen05<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tcgen05_pair<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM2_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tcgen05_pair<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM2_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tcgen05_pair<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM2_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tcgen05_pair<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM2_SMEM);
  if (e != cudaSuccess) return e;
  done |= uint64_t(1) << dev;
  return cudaSuccess;
}

// Tensor maps and tile counts of one problem; pair = 256-row CTA-pair tiles.
// `to` maps the gated-residual output in 32 x 32 boxes (64-byte swizzle) when
// the residual can move by TMA; otherwise it is a copy of `ta` that no
// epilogue reads.
static cudaError_t prepare_gemm(GemmParams& p, const void* A, const void* W, int W_rows, bool pair, CUtensorMap* ta,
                                CUtensorMap* tb, CUtensorMap* to) {
  const bool fp8 = p.w_scale != nullptr;
  const int esz = fp8 ? 1 : 2;
  const int kb = fp8 ? 2 * GEMM_BK : GEMM_BK;  // 128-byte K boxes either way
  if (p.K <= 0 || (p.K * esz) % 16 != 0) return cudaErrorInvalidValue;
  if (fp8 && !p.a_scale) return cudaErrorInvalidValue;
  if (!encode_tmap_2d(ta, A, p.K, p.M, static_cast<uint64_t>(p.K) * esz, kb, GEMM_BM, fp8))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(tb, W, p.K, W_rows, static_cast<uint64_t>(p.K) * esz, kb, pair ? 128 : GEMM_BN, fp8))
    return cudaErrorInvalidValue;
  *to = *ta;
  p.res_tma = 0;
  if (p.mode == EPI_GATE_RES && p.out && (reinterpret_cast<uintptr_t>(p.out) & 15) == 0 &&
      (static_cast<uint64_t>(p.ldo) * 2) % 16 == 0 && p.ldo >= p.N && p.rows_per_batch == p.out_rows_per_batch &&
      p.out_row_off == 0) {
    if (encode_tmap_2d(to, p.out, p.N, p.M, static_cast<uint64_t>(p.ldo) * 2, 32, 32, false, 64)) p.res_tma = 1;
    else *to = *ta;
  }
  auto al16 = [](const void* a) { return (reinterpret_cast<uintptr_t>(a) & 15) == 0; };
  if (p.mode == EPI_SWIGLU && p.out && al16(p.out) && (static_cast<uint64_t>(p.ldo) * 2) % 16 == 0 &&
      p.ldo >= p.N && p.rows_per_batch == p.out_rows_per_batch && p.out_row_off == 0) {
    if (encode_tmap_2d(to, p.out, p.N, p.M, static_cast<uint64_t>(p.ldo) * 2, 32, 32, false, 64)) p.res_tma = 1;
    else *to = *ta;
  }
  if (p.mode == EPI_QKV && p.q && p.k && p.v && p.hd >= 32 && p.hd % 32 == 0 && p.rows_per_batch > 0 &&
      p.M % p.rows_per_batch == 0 && p.n_total >= p.qkv_row_off + p.rows_per_batch) {
    const char* q = reinterpret_cast<const char*>(p.q);
    const ptrdiff_t dk = reinterpret_cast<const char*>(p.k) - q, dv = reinterpret_cast<const char*>(p.v) - q;
    const uint64_t rows = static_cast<uint64_t>(p.M / p.rows_per_batch) * p.heads * p.n_total;
    if (al16(q) && dk > 0 && dv == 2 * dk && dk % 16 == 0 &&
        static_cast<uint64_t>(dk) >= rows * p.hd * 2 &&
        encode_tmap_3d(to, p.q, p.hd, rows, 3, static_cast<uint64_t>(p.hd) * 2, static_cast<uint64_t>(dk), 32, 32, 1,
                       64))
      p.res_tma = 1;
    else
      *to = *ta;
  }
  p.num_n_tiles = p.mode == EPI_SWIGLU ? (p.N + 127) / 128 : (p.N + GEMM_BN - 1) / GEMM_BN;
  p.group_n = p.num_n_tiles < 16 ? p.num_n_tiles : 16;
  p.num_m_tiles = pair ? (p.M + 255) / 256 : (p.M + GEMM_BM - 1) / GEMM_BM;
  p.num_tiles = p.num_m_tiles * p.num_n_tiles;
  return cudaSuccess;
}

static cudaError_t launch_pair(const GemmParams& p0, const CUtensorMap& ta0, const CUtensorMap& tb0,
                               const CUtensorMap& to0, const GemmParams& p1, const CUtensorMap& ta1,
                               const CUtensorMap& tb1, const CUtensorMap& to1, cudaStream_t stream, int num_sms) {
  const int total = p0.num_tiles + p1.num_tiles;
  const int pairs = num_sms / 2;
  const int grid = 2 * (total < pairs ? total : pairs);
  const bool grouped = p1.num_tiles > 0;
  if (p0.w_scale) {
    if (grouped)
      gemm_tcgen05_pair<true, true><<<grid, GEMM_THREADS, GEMM2_SMEM, stream>>>(ta0, tb0, to0, ta1, tb1, to1, p0, p1);
    else
      gemm_tcgen05_pair<true, false><<<grid, GEMM_THREADS, GEMM2_SMEM, stream>>>(ta0, tb0, to0, ta1, tb1, to1, p0, p1);
  } else {
    if (grouped)
      gemm_tcgen05_pair<false, true><<<grid, GEMM_THREADS, GEMM2_SMEM, stream>>>(ta0, tb0, to0, ta1, tb1, to1, p0, p1);
    else
      gemm_tcgen05_pair<false, false><<<grid, GEMM_THREADS, GEMM2_SMEM, stream>>>(ta0, tb0, to0, ta1, tb1, to1, p0, p1);
  }
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmParams& p_in, const void* A, const void* W, int W_rows, cudaStream_t stream,
                        int num_sms) {
  GemmParams p = p_in;
  if (p.M <= 0 || p.N <= 0) return cudaSuccess;
  const bool fp8 = p.w_scale != nullptr;
  const bool pair = p.M >= 1024 && num_sms >= 2;
  CUtensorMap ta, tb, to;
  cudaError_t e = prepare_gemm(p, A, W, W_rows, pair, &ta, &tb, &to);
  if (e != cudaSuccess) return e;
  e = gemm_set_attributes();
  if (e != cudaSuccess) return e;
  if (pair) {
    GemmParams none = p;
    none.num_tiles = 0;
    return launch_pair(p, ta, tb, to, none, ta, tb, to, stream, num_sms);
  }
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  if (fp8)
    gemm_tcgen05<true><<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, stream>>>(ta, tb, to, p);
  else
    gemm_tcgen05<false><<<grid, GEMM_THREADS, GEMM_SMEM_BYTES, stream>>>(ta, tb, to, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_grouped(const GemmParams& p0_in, const void* A0, const void* W0, int W0_rows,
                                const GemmParams& p1_in, const void* A1, const void* W1, int W1_rows,
                                cudaStream_t stream, int num_sms) {
  GemmParams p0 = p0_in, p1 = p1_in;
  if ((p0.w_scale != nullptr) != (p1.w_scale != nullptr)) return cudaErrorInvalidValue;
  const bool empty0 = p0.M <= 0 || p0.N <= 0, empty1 = p1.M <= 0 || p1.N <= 0;
  if (empty0 || empty1 || p0.M + p1.M < 1024 || num_sms < 2) {  // too small for pairs: one launch each
    cudaError_t e = empty0 ? cudaSuccess : launch_gemm(p0, A0, W0, W0_rows, stream, num_sms);
    if (e == cudaSuccess && !empty1) e = launch_gemm(p1, A1, W1, W1_rows, stream, num_sms);
    return e;
  }
  CUtensorMap ta0, tb0, to0, ta1, tb1, to1;
  cudaError_t e = prepare_gemm(p0, A0, W0, W0_rows, true, &ta0, &tb0, &to0);
  if (e == cudaSuccess) e = prepare_gemm(p1, A1, W1, W1_rows, true, &ta1, &tb1, &to1);
  if (e == cudaSuccess) e = gemm_set_attributes();
  if (e != cudaSuccess) return e;
  return launch_pair(p0, ta0, tb0, to0, p1, ta1, tb1, to1, stream, num_sms);
}

}  // namespace af
