// attention.cu -- joint / self attention of the AuraFlow blocks on sm_100a.
//
//   O = softmax(Q K^T * hd^-1/2) V   per (sample, head); non-causal, with an
//   optional per-sample masked key range (padded prompts)
//
// ("Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南",
// §注意力处理器与 QKV 融合: text and image tokens are concatenated and
// attended jointly with SDPA, dropout 0, is_causal False.)
//
// attn_hd256_online (any q, k) and attn_hd256_qknorm (per-head LayerNorm-ed
// q, k; see below): one CTA = 128 query rows of one (sample, head).
//   smem: Q 128x256 (64 KB, loaded once), K and V tiles of 64 keys x 256
//   double-buffered (2 x 32 KB each), P 128x64 bf16 (16 KB); all 128-byte
//   swizzled.  TMEM (512 columns): O 128x256 fp32 in columns [0,256), two
//   S buffers 128x64 fp32 in [256,384).
//   warp 0      TMA producer of Q (once) and the K tiles; warp 10 of the V
//               tiles (independent rings, so a K load never waits for a V
//               buffer release).
//   warp 1      one thread issues S_{j+1} = Q K_{j+1}^T (M=128, N=64, K=256)
//               before O += P_j V_j (M=128, N=256, K=64, V read MN-major),
//               so the tensor core works on the next scores while the
//               softmax warps handle the current ones.
//   warps 2..9  softmax, two warpgroups: warpgroup g owns key columns
//               [32g, 32g+32) of every S tile and O columns [128g, 128g+128);
//               thread = query row.  Partial row maxima (and at the end the
//               partial row sums) are exchanged through shared memory.  fp32
//               online softmax in the exp2 domain with a lazy running max
//               (O is rescaled only when the max grows by more than 2^8), P
//               written as bf16 into swizzled shared memory, O normalised at
//               the end.
// attn_small_simt: one thread per query row, for head_dim <= 64 (used by
//   small test models only).
#include "af_internal.h"
#include "ptx.cuh"

namespace af {

constexpr int AT_BM = 128;
constexpr int AT_BN = 64;
constexpr int AT_HD = 256;
constexpr uint32_t AT_Q_BYTES = AT_BM * AT_HD * 2;   // 64 KB
constexpr uint32_t AT_KV_BYTES = AT_BN * AT_HD * 2;  // 32 KB
constexpr uint32_t AT_P_BYTES = AT_BM * AT_BN * 2;   // 16 KB
constexpr int AT_SOFTMAX_WARPS = 8;
constexpr int AT_V_WARP = 2 + AT_SOFTMAX_WARPS;            // V producer (after the softmax warps)
constexpr int AT_THREADS = 32 * (AT_V_WARP + 1);
constexpr uint32_t AT_XCH_BYTES = 3 * 2 * AT_BM * 4;  // row-max slots [2][2][128] + row-sum [2][128]
constexpr int AT_SMEM = AT_Q_BYTES + 4 * AT_KV_BYTES + AT_P_BYTES + AT_XCH_BYTES + 512 + 1024;
constexpr float LAZY_RESCALE_LOG2 = 8.0f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Masked key range [lo, hi) of sample b (empty when the call has no mask).
__device__ __forceinline__ void key_mask_range(const AttnParams& p, int b, int& lo, int& hi) {
  lo = hi = 0;
  if (p.key_len) {
    const int n = min(max(p.key_len[b], 0), p.key_end - p.key_base);
    lo = p.key_base + n;
    hi = p.key_end;
  }
}

__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_hd256_online(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + AT_Q_BYTES;            // 2 buffers
  uint8_t* sV = sK + 2 * AT_KV_BYTES;       // 2 buffers
  uint8_t* sP = sV + 2 * AT_KV_BYTES;
  float* xmax = reinterpret_cast<float*>(sP + AT_P_BYTES);  // [slot 2][wg 2][row 128]
  float* xsum = xmax + 4 * AT_BM;                           // [wg 2][row 128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + AT_P_BYTES + AT_XCH_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* k_empty = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;   // [2]
  uint64_t* s_full = bars + 9;    // [2]
  uint64_t* s_empty = bars + 11;  // [2]
  uint64_t* p_full = bars + 13;
  uint64_t* o_done = bars + 14;
  uint64_t* mma_done = bars + 15;
  uint64_t* xbar = bars + 16;     // [2] row-max exchange
  uint64_t* lbar = bars + 18;     // row-sum exchange
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int q0 = qt * AT_BM;
  const int nkv = (p.N + AT_BN - 1) / AT_BN;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_empty[i]), 1);
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_empty[i]), AT_SOFTMAX_WARPS);
      mbar_init(smem_u32(&xbar[i]), AT_SOFTMAX_WARPS);
    }
    mbar_init(smem_u32(p_full), AT_SOFTMAX_WARPS);
    mbar_init(smem_u32(o_done), 1);
    mbar_init(smem_u32(mma_done), 1);
    mbar_init(smem_u32(lbar), AT_SOFTMAX_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem;
  const uint32_t tS = tmem + 256;
  volatile int never = 0;

  if (warp == 0 || warp == AT_V_WARP) {
    // warp 0 streams Q then the K tiles, the last warp streams the V tiles, so
    // neither ring waits behind the other's buffer release
    if (lane == 0) {
      const bool is_k = warp == 0;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const void* tm = is_k ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmV);
      uint8_t* buf = is_k ? sK : sV;
      uint32_t armed = 0, par = 0;
      bool ok = true;
      if (is_k) {
        mbar_arrive_expect_tx(smem_u32(q_full), AT_Q_BYTES);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(smem_u32(sQ + c * (AT_BM * 128)), &tmQ, smem_u32(q_full), c * 64, q0, bh);
      }
      for (int j = 0; j < nkv; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, p.err, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(smem_u32(&full[s]), AT_KV_BYTES);
        armed |= 1u << s; par = (par & ~(1u << s)) | (ph << s);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(smem_u32(buf + s * AT_KV_BYTES + c * (AT_BN * 128)), tm, smem_u32(&full[s]), c * 64,
                      j * AT_BN, bh);
      }
      if (!ok) {
        if (is_k) mbar_wait(smem_u32(q_full), 0, nullptr, &never, 100000000ull);
        for (int s = 0; s < 2; ++s)
          if (armed & (1u << s)) mbar_wait(smem_u32(&full[s]), (par >> s) & 1u, nullptr, &never, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(AT_BM, AT_BN, false, false);
      const uint32_t idesc_pv = make_idesc_bf16(AT_BM, AT_HD, false, true);
      const uint32_t qaddr = smem_u32(sQ);
      const uint32_t paddr = smem_u32(sP);
      bool ok = mbar_wait(smem_u32(q_full), 0, p.err, abort_flag);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(smem_u32(&k_full[s]), ph, p.err, abort_flag)) return false;
        if (!mbar_wait(smem_u32(&s_empty[s]), ph ^ 1u, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kaddr = smem_u32(sK + s * AT_KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < AT_HD / 16; ++kk) {
          const uint32_t c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t ad = make_sdesc(qaddr, 16, 1024, SWZ_128B) + static_cast<uint64_t>((c * (AT_BM * 128) + off) >> 4);
          const uint64_t bd = make_sdesc(kaddr, 16, 1024, SWZ_128B) + static_cast<uint64_t>((c * (AT_BN * 128) + off) >> 4);
          mma_bf16_ss(tS + s * AT_BN, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&s_full[s]));
        mma_commit(smem_u32(&k_empty[s]));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv && !issue_s(j + 1)) { ok = false; break; }
        const int s = j & 1;
        if (!mbar_wait(smem_u32(p_full), j & 1, p.err, abort_flag)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&v_full[s]), (j >> 1) & 1, p.err, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t vaddr = smem_u32(sV + s * AT_KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < AT_BN / 16; ++kk) {
          const uint64_t ad = make_sdesc(paddr, 16, 1024, SWZ_128B) + static_cast<uint64_t>((kk * 32) >> 4);
          const uint64_t bd = make_sdesc(vaddr, AT_BN * 128, 1024, SWZ_128B) + static_cast<uint64_t>((kk * (16 * 128)) >> 4);
          mma_bf16_ss(tO, ad, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(o_done));
        mma_commit(smem_u32(&v_empty[s]));
      }
      mma_commit(smem_u32(mma_done));
      mbar_wait(smem_u32(mma_done), 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    const int wg = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    int klo, khi;
    key_mask_range(p, b, klo, khi);
    bool ok = true;
    uint8_t* prow = sP + row * 128;
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      const bool got = mbar_wait(smem_u32(&s_full[s]), (j >> 1) & 1, p.err, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tS + s * AT_BN + 32 * wg + lane_off, r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s_empty[s]));
      float x[32];
      const int kvalid = p.N - j * AT_BN - 32 * wg;   // valid key columns in this half
      const int mlo = klo - j * AT_BN - 32 * wg, mhi = khi - j * AT_BN - 32 * wg;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        x[i] = (i < kvalid && (i < mlo || i >= mhi)) ? __uint_as_float(r[i]) : -INFINITY;
      float mr = x[0];
#pragma unroll
      for (int i = 1; i < 32; ++i) mr = fmaxf(mr, x[i]);
      // exchange the partial row max with the other warpgroup
      float* slot = xmax + (j & 1) * 2 * AT_BM;
      slot[wg * AT_BM + row] = mr * c;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&xbar[j & 1]));
      const bool gx = mbar_wait(smem_u32(&xbar[j & 1]), (j >> 1) & 1, p.err, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, gx)) { ok = false; break; }
      const float mt = fmaxf(mr * c, slot[(wg ^ 1) * AT_BM + row]);
      float m_new = m;
      bool rescale = false;
      if (j == 0) {
        m_new = mt == -INFINITY ? 0.f : mt;   // a fully masked first tile: any finite start
      } else if (mt > m + LAZY_RESCALE_LOG2) {
        m_new = mt;
        rescale = true;
      }
      float rs = 0.f;
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float e0 = ex2_approx(fmaf(x[2 * i], c, -m_new));
        const float e1 = ex2_approx(fmaf(x[2 * i + 1], c, -m_new));
        rs += e0 + e1;
        pk[i] = pack_bf16(e0, e1);
      }
      // PV_{j-1} must be complete before O is rescaled and P is overwritten
      if (j > 0) {
        const bool g2 = mbar_wait(smem_u32(o_done), (j - 1) & 1, p.err, abort_flag);
        __syncwarp();
        if (!__all_sync(0xffffffffu, g2)) { ok = false; break; }
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale)) {
        const float alpha = rescale ? ex2_approx(m - m_new) : 1.0f;
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t ta = tO + 128 * wg + cc * 32 + lane_off;
          uint32_t o[32];
          tmem_ld32(ta, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(ta, o);
        }
        tmem_wait_st();
        l *= alpha;
      }
      m = m_new;
      l += rs;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int chunk = 4 * wg + q;
        uint4 v = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        *reinterpret_cast<uint4*>(prow + ((chunk ^ (row & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(p_full));
    }
    if (ok) {
      // total row sum from both warpgroups
      xsum[wg * AT_BM + row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(lbar));
      const bool g3 = mbar_wait(smem_u32(lbar), 0, p.err, abort_flag) &&
                      mbar_wait(smem_u32(o_done), (nkv - 1) & 1, p.err, abort_flag);
      __syncwarp();
      if (__all_sync(0xffffffffu, g3)) {
        tc_fence_after();
        const float inv = 1.0f / (l + xsum[(wg ^ 1) * AT_BM + row]);
        const int qrow = q0 + row;
        const bool row_ok = qrow < p.N;
        uint16_t* dst = nullptr;
        if (row_ok) {
          if (qrow < p.split)
            dst = p.out_a + (static_cast<size_t>(b) * p.split + qrow) * p.ldo + h * AT_HD;
          else
            dst = p.out_b + (static_cast<size_t>(b) * (p.N - p.split) + (qrow - p.split)) * p.ldo + h * AT_HD;
          dst += 128 * wg;
        }
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + 128 * wg + cc * 32 + lane_off, o);
          tmem_wait_ld();
          if (row_ok) {
            uint4* d = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 u;
              u.x = pack_bf16(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
              u.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
              u.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
              u.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
              d[i] = u;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- QK-normalised inputs
// When every q and k row is a per-head LayerNorm output (||q||, ||k|| <=
// sqrt(hd), up to bf16 rounding), every logit satisfies
// |q.k| / sqrt(hd) <= sqrt(hd) * (1 + 2^-9)^2, i.e. <= 23.2 in log2 units
// for hd = 256.  Softmax is invariant to a common shift, so the fixed shift
// QKN_OFFSET_LOG2 = 24 replaces the running maximum exactly: probabilities
// lie in [2^-48, 1) (normal fp32/bf16 numbers) and no rescaling of O is ever
// needed.  The two softmax warpgroups then work on alternate KV tiles (group
// g takes tiles j = g mod 2, full 64-key rows) with one P buffer each, and
// their partial row sums are added at the end.
//
// Q is kept in TMEM (columns [384, 512), two bf16 per column) and S = Q K^T
// is issued with A read from TMEM, so the 16 K-steps of a tile only stream
// the K tile from shared memory (re-reading a 128 x 16 Q slice from shared
// memory for every step made the N = 64 product bandwidth-bound).  TMEM:
// O [0, 256), S0 [256, 320), S1 [320, 384), Q [384, 512).  The freed shared
// memory holds a third K and V stage.
//
// The CTAs of one (sample, head) all stream the same K and V; each starts its
// KV loop at a different tile (kv_tile(j) below) so that concurrently running
// CTAs request different lines instead of hammering the same L2 slices.
constexpr float QKN_OFFSET_LOG2 = 24.0f;
constexpr int QKN_THREADS = AT_THREADS;
constexpr int QKN_STAGES = 3;
constexpr uint32_t QKN_XCH_BYTES = 2 * AT_BM * 4;
constexpr int QKN_SMEM = 2 * QKN_STAGES * AT_KV_BYTES + 2 * AT_P_BYTES + QKN_XCH_BYTES + 256 + 1024;

__global__ void __launch_bounds__(QKN_THREADS, 1)
    attn_hd256_qknorm(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;                               // QKN_STAGES buffers
  uint8_t* sV = sK + QKN_STAGES * AT_KV_BYTES;      // QKN_STAGES buffers
  uint8_t* sP = sV + QKN_STAGES * AT_KV_BYTES;      // 2 buffers
  float* xsum = reinterpret_cast<float*>(sP + 2 * AT_P_BYTES);  // [wg 2][row 128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * AT_P_BYTES + QKN_XCH_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [QKN_STAGES]
  uint64_t* v_full = bars + 4;    // [QKN_STAGES]
  uint64_t* k_empty = bars + 7;   // [QKN_STAGES]
  uint64_t* v_empty = bars + 10;  // [QKN_STAGES]
  uint64_t* s_full = bars + 13;   // [2]
  uint64_t* s_empty = bars + 15;  // [2]
  uint64_t* p_full = bars + 17;   // [2]
  uint64_t* pv_done = bars + 19;  // [2]
  uint64_t* mma_done = bars + 21;
  uint64_t* lbar = bars + 22;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int q0 = qt * AT_BM;
  const int nkv = (p.N + AT_BN - 1) / AT_BN;
  const int kv0 = static_cast<int>((static_cast<long long>(qt) * nkv) / gridDim.x);
  auto kv_tile = [&](int j) { const int t = j + kv0; return t < nkv ? t : t - nkv; };

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 4);
    for (int i = 0; i < QKN_STAGES; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_empty[i]), 4);
      mbar_init(smem_u32(&p_full[i]), 4);
      mbar_init(smem_u32(&pv_done[i]), 1);
    }
    mbar_init(smem_u32(mma_done), 1);
    mbar_init(smem_u32(lbar), AT_SOFTMAX_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem;
  const uint32_t tS = tmem + 256;
  const uint32_t tQ = tmem + 384;
  volatile int never = 0;

  if (warp == 0 || warp == AT_V_WARP) {
    if (lane == 0) {
      const bool is_k = warp == 0;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const void* tm = is_k ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmV);
      uint8_t* buf = is_k ? sK : sV;
      uint32_t armed = 0, par = 0;
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % QKN_STAGES;
        const uint32_t ph = (j / QKN_STAGES) & 1;
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, p.err, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(smem_u32(&full[s]), AT_KV_BYTES);
        armed |= 1u << s; par = (par & ~(1u << s)) | (ph << s);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(smem_u32(buf + s * AT_KV_BYTES + c * (AT_BN * 128)), tm, smem_u32(&full[s]), c * 64,
                      kv_tile(j) * AT_BN, bh);
      }
      if (!ok) {
        for (int s = 0; s < QKN_STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(smem_u32(&full[s]), (par >> s) & 1u, nullptr, &never, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(AT_BM, AT_BN, false, false);
      const uint32_t idesc_pv = make_idesc_bf16(AT_BM, AT_HD, false, true);
      bool ok = mbar_wait(smem_u32(q_full), 0, p.err, abort_flag);
      tc_fence_after();
      auto issue_s = [&](int j) -> bool {
        const int kb = j % QKN_STAGES;
        const int s = j & 1;
        if (!mbar_wait(smem_u32(&k_full[kb]), (j / QKN_STAGES) & 1, p.err, abort_flag)) return false;
        if (!mbar_wait(smem_u32(&s_empty[s]), ((j >> 1) & 1) ^ 1u, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kaddr = smem_u32(sK + kb * AT_KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < AT_HD / 16; ++kk) {
          const uint32_t c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t bd = make_sdesc(kaddr, 16, 1024, SWZ_128B) + static_cast<uint64_t>((c * (AT_BN * 128) + off) >> 4);
          mma_bf16_ts(tS + s * AT_BN, tQ + kk * 8, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&s_full[s]));
        mma_commit(smem_u32(&k_empty[kb]));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv && !issue_s(j + 1)) { ok = false; break; }
        const int s = j & 1;
        const int vb = j % QKN_STAGES;
        if (!mbar_wait(smem_u32(&p_full[s]), (j >> 1) & 1, p.err, abort_flag)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&v_full[vb]), (j / QKN_STAGES) & 1, p.err, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t paddr = smem_u32(sP + s * AT_P_BYTES);
        const uint32_t vaddr = smem_u32(sV + vb * AT_KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < AT_BN / 16; ++kk) {
          const uint64_t ad = make_sdesc(paddr, 16, 1024, SWZ_128B) + static_cast<uint64_t>((kk * 32) >> 4);
          const uint64_t bd = make_sdesc(vaddr, AT_BN * 128, 1024, SWZ_128B) + static_cast<uint64_t>((kk * (16 * 128)) >> 4);
          mma_bf16_ss(tO, ad, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(&pv_done[s]));
        mma_commit(smem_u32(&v_empty[vb]));
      }
      mma_commit(smem_u32(mma_done));
      mbar_wait(smem_u32(mma_done), 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ---------------------------------------------------------------- softmax: group g takes tiles j = g (mod 2)
    const int wg = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    const float off = -QKN_OFFSET_LOG2;
    int klo, khi;
    key_mask_range(p, b, klo, khi);
    float l = 0.f;
    bool ok = true;
    uint8_t* prow = sP + wg * AT_P_BYTES + row * 128;
    if (wg == 0) {
      // this row of Q into TMEM (zeros beyond N), then release the MMA warp
      const int qrow = q0 + row;
      const uint4* src = reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(bh) * p.N + qrow) * AT_HD);
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t qv[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 u = qrow < p.N ? src[cc * 8 + i] : make_uint4(0, 0, 0, 0);
          qv[4 * i] = u.x;
          qv[4 * i + 1] = u.y;
          qv[4 * i + 2] = u.z;
          qv[4 * i + 3] = u.w;
        }
        tmem_st32(tQ + cc * 32 + lane_off, qv);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(q_full));
    }
    for (int j = wg; j < nkv; j += 2) {
      const uint32_t ph = (j >> 1) & 1;
      const bool got = mbar_wait(smem_u32(&s_full[wg]), ph, p.err, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tS + wg * AT_BN + lane_off, r0);
      tmem_ld32(tS + wg * AT_BN + 32 + lane_off, r1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s_empty[wg]));
      const int kbase = kv_tile(j) * AT_BN;
      const int kvalid = p.N - kbase, mlo = klo - kbase, mhi = khi - kbase;
      const bool partial = kvalid < AT_BN || (mlo < mhi && mlo < AT_BN && mhi > 0);
      auto dead = [&](int i) { return i >= kvalid || (i >= mlo && i < mhi); };
      uint32_t pk[32];
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float e0 = ex2_approx(fmaf(__uint_as_float(r0[2 * i]), c, off));
        float e1 = ex2_approx(fmaf(__uint_as_float(r0[2 * i + 1]), c, off));
        float e2 = ex2_approx(fmaf(__uint_as_float(r1[2 * i]), c, off));
        float e3 = ex2_approx(fmaf(__uint_as_float(r1[2 * i + 1]), c, off));
        if (partial) {
          if (dead(2 * i)) e0 = 0.f;
          if (dead(2 * i + 1)) e1 = 0.f;
          if (dead(32 + 2 * i)) e2 = 0.f;
          if (dead(32 + 2 * i + 1)) e3 = 0.f;
        }
        rs += (e0 + e1) + (e2 + e3);
        pk[i] = pack_bf16(e0, e1);
        pk[16 + i] = pack_bf16(e2, e3);
      }
      l += rs;
      // P buffer wg is free once PV_{j-2} has completed
      if (j >= 2) {
        const bool g2 = mbar_wait(smem_u32(&pv_done[wg]), ph ^ 1u, p.err, abort_flag);
        __syncwarp();
        if (!__all_sync(0xffffffffu, g2)) { ok = false; break; }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint4 v = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        *reinterpret_cast<uint4*>(prow + ((q ^ (row & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&p_full[wg]));
    }
    if (ok) {
      xsum[wg * AT_BM + row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(lbar));
      const int jl = nkv - 1;
      const bool g3 = mbar_wait(smem_u32(lbar), 0, p.err, abort_flag) &&
                      mbar_wait(smem_u32(&pv_done[jl & 1]), (jl >> 1) & 1, p.err, abort_flag);
      __syncwarp();
      if (__all_sync(0xffffffffu, g3)) {
        tc_fence_after();
        const float inv = 1.0f / (l + xsum[(wg ^ 1) * AT_BM + row]);
        const int qrow = q0 + row;
        const bool row_ok = qrow < p.N;
        uint16_t* dst = nullptr;
        if (row_ok) {
          if (qrow < p.split)
            dst = p.out_a + (static_cast<size_t>(b) * p.split + qrow) * p.ldo + h * AT_HD;
          else
            dst = p.out_b + (static_cast<size_t>(b) * (p.N - p.split) + (qrow - p.split)) * p.ldo + h * AT_HD;
          dst += 128 * wg;
        }
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + 128 * wg + cc * 32 + lane_off, o);
          tmem_wait_ld();
          if (row_ok) {
            uint4* d = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 u;
              u.x = pack_bf16(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
              u.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
              u.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
              u.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
              d[i] = u;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- QK-normalised inputs on CTA pairs
// attn_hd256_qknorm_pair: a cluster of two CTAs takes 256 query rows of one
// (sample, head), 128 per CTA, and walks the keys in tiles of 128 with
// tcgen05.mma.cta_group::2 issued from the leader CTA:
//   S = Q K^T   M = 256, N = 128, K = 256: A is each CTA's 128 Q rows, B half
//               of the K tile (64 keys), both from that CTA's shared memory;
//               each CTA's TMEM receives its 128 x 128 block of S.
//   O += P V    M = 256, N = 256, K = 128: A is each CTA's 128 rows of P, read
//               from its own TMEM; B is half of the V tile (128 head-dim
//               columns) from shared memory; each CTA's TMEM accumulates its
//               128 x 256 block of O.
// Per SM that is 64 KB of K/V per 128 keys instead of 128 KB, and every MMA
// has N >= 128 (full tensor-core rate).  Softmax (fixed shift, as for
// attn_hd256_qknorm): each softmax warpgroup owns a slice of the keys of
// every S tile; the partial row sums are added at the end.  S_{j+1} is
// issued as soon as both CTAs' softmax warps have read S_j out of TMEM,
// PV_j once P_j is published, so the tensor core computes the next scores
// while the softmax warps work.  Barriers that gather both CTAs live in the
// leader (TMA completions, S/P handshakes); commits are multicast to both
// CTAs.  The follower's softmax warps arrive directly on the leader's S/P
// barriers (CTA-scope release; a cluster-scope release there costs ~1.2k
// cycles).
// D (+)= A * B over the CTA pair with A in TMEM: each CTA's 128 rows of A are
// read from its own TMEM at a_tmem (two consecutive K elements per 32-bit
// column), B split along N between the two CTAs' shared memory.
__device__ __forceinline__ void mma_bf16_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

constexpr int AP_BN = 128;
constexpr uint32_t AP_KH_BYTES = 64 * AT_HD * 2;      // 32 KB: 64 keys x 256
constexpr uint32_t AP_VH_BYTES = AP_BN * 128 * 2;     // 32 KB: 128 keys x 128 columns
constexpr uint32_t AP_Q_BYTES = 128 * AT_HD * 2;      // 64 KB: 128 rows x 256

// Layout.  Q stays in shared memory for the S products, which leaves TMEM
// room for two P buffers: the softmax warps write P_j into TMEM with
// tcgen05.st (no shared-memory store, no proxy fence) and the PV product
// reads it from there.  TMEM per CTA: O [0, 256), S [256, 384), P_0
// [384, 448), P_1 [448, 512).  Shared memory per CTA: Q 64 KB, K 3 x 32 KB,
// V 2 x 32 KB (the row sums reuse a V stage after the last PV).  K has three
// stages (a K half takes ~900-4400 cycles from load to landing, and a stage
// is refilled only when the S product that read it completes), V two (a V
// stage is refilled when its PV completes and is next needed two tiles
// later).  Four softmax warpgroups of 32 keys each (TMEM lane quarters
// shared by warps w, w + 4, w + 8, w + 12); P buffer j & 1 is rewritten only
// after PV_{j-2} completes, so the softmax never waits for the PV product
// just before it.  Each softmax warp reads S_{j+1} out of TMEM before
// publishing P_j when S_{j+1} has already completed.  The S and PV products
// are issued by two threads: the barrier checks of one overlap the other's
// MMAs in the tensor pipe (one thread doing both left a gap of a few hundred
// cycles at every switch).  Earlier layouts, measured: Q in TMEM with P in
// shared memory (one or two P buffers, K and V stages 2 + 2, 3 + 3, 3 + 2 or
// a shared ring of 5) ran at ~2580-2870 cycles per tile, bound by the
// softmax warps' P store, proxy fence and arrival; this one runs ~2290.
// The epilogue stages the normalised O in the Q buffer (free once the last S
// product has completed) and writes it row-contiguously: with each thread
// storing its own row the stores of a CTA took ~4k cycles.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
constexpr int PAIR_NWG = 4;
constexpr int PAIR_SM_WARPS = 4 * PAIR_NWG;
constexpr int PAIR_V_WARP = 2 + PAIR_SM_WARPS;
constexpr int PAIR_PV_WARP = PAIR_V_WARP + 1;
constexpr int PAIR_THREADS = 32 * (PAIR_PV_WARP + 1);
constexpr int PAIR_KPW = AP_BN / PAIR_NWG;   // 32 keys per warpgroup
constexpr int PAIR_KST = 3;
constexpr int PAIR_VST = 2;
constexpr int PAIR_SMEM = AP_Q_BYTES + PAIR_KST * AP_KH_BYTES + PAIR_VST * AP_VH_BYTES + 256 + 1024;

// Non-suspending test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
    attn_hd256_qknorm_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                    // this CTA's 128 Q rows (64 KB)
  uint8_t* sK = sQ + AP_Q_BYTES;                     // PAIR_KST stages
  uint8_t* sV = sK + PAIR_KST * AP_KH_BYTES;              // PAIR_VST stages (row sums at the end)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + PAIR_VST * AP_VH_BYTES);
  uint64_t* q_full = bars + 0;                 // leader: both CTAs' Q tiles
  uint64_t* k_full = bars + 1;                 // [3] leader: both K halves
  uint64_t* k_empty = bars + 4;                // [3] both CTAs (multicast commit)
  uint64_t* v_full = bars + 7;                 // [2] leader: both V halves
  uint64_t* v_empty = bars + 9;                // [2] both CTAs
  uint64_t* s_full = bars + 11;                // both CTAs
  uint64_t* s_empty = bars + 12;               // leader: softmax warps of both CTAs
  uint64_t* p_full = bars + 13;                // [2] leader: softmax warps of both CTAs
  uint64_t* pv_done = bars + 15;               // [2] both CTAs
  uint64_t* mma_done = bars + 19;              // leader: the S issuer's MMAs
  uint64_t* lbar = bars + 20;                  // per CTA: row sums written
  uint64_t* mma_done_pv = bars + 21;           // leader: the PV issuer's MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 22);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int q0 = pair * 256 + static_cast<int>(rank) * 128;
  const int nkv = (p.N + AP_BN - 1) / AP_BN;
  const int kv0 = static_cast<int>((static_cast<long long>(pair) * nkv) / npairs);
  auto kv_tile = [&](int j) { const int t = j + kv0; return t < nkv ? t : t - nkv; };

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < PAIR_KST; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
    }
    for (int i = 0; i < PAIR_VST; ++i) {
      mbar_init(smem_u32(&v_full[i]), 1);
      mbar_init(smem_u32(&v_empty[i]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_empty), 2 * PAIR_SM_WARPS);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&p_full[i]), 2 * PAIR_SM_WARPS);
      mbar_init(smem_u32(&pv_done[i]), 1);
    }
    mbar_init(smem_u32(mma_done), 1);
    mbar_init(smem_u32(mma_done_pv), 1);
    mbar_init(smem_u32(lbar), PAIR_SM_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem;
  const uint32_t tS = tmem + 256;
  const uint32_t tP = tmem + 384;  // P buffer b at tP + 64 b
  volatile int never = 0;

  if (warp == 0 || warp == PAIR_V_WARP) {
    // warp 0: this CTA's Q tile, then the K halves (keys [64 rank, +64) of
    // each tile); the V warp: the V halves (head-dim columns [128 rank, +128))
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int nst = is_k ? PAIR_KST : PAIR_VST;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const uint32_t half = is_k ? AP_KH_BYTES : AP_VH_BYTES;
      uint8_t* buf = is_k ? sK : sV;
      bool ok = true;
      if (is_k) {
        // both CTAs' Q tiles complete on the leader's barrier
        if (leader) mbar_arrive_expect_tx(smem_u32(q_full), 2 * AP_Q_BYTES);
        const uint32_t qb = mapa_shared(smem_u32(q_full), 0);
        for (int c = 0; c < 4; ++c) tma_load_3d_pair(smem_u32(sQ + c * (128 * 128)), &tmQ, qb, c * 64, q0, bh);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j % nst;
        const uint32_t ph = (j / nst) & 1;
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, p.err, abort_flag)) { ok = false; break; }
        if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), 2 * half);
        const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
        const int key0 = kv_tile(j) * AP_BN;
        if (is_k) {
          for (int c = 0; c < 4; ++c)
            tma_load_3d_pair(smem_u32(buf + s * half + c * (64 * 128)), &tmK, fb, c * 64,
                             key0 + static_cast<int>(rank) * 64, bh);
        } else {
          for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(smem_u32(buf + s * half + c * (AP_BN * 128)), &tmV, fb,
                             static_cast<int>(rank) * 128 + c * 64, key0, bh);
        }
      }
      if (!ok) {  // let copies already in flight land before the CTA exits
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // S issuer: S_j into the single S buffer once K_j has landed and the
    // softmax warps of both CTAs have read S_{j-1}
    if (lane == 0 && leader) {
      const uint32_t idesc_qk = make_idesc_bf16(256, AP_BN, false, false);
      bool ok = mbar_wait(smem_u32(q_full), 0, p.err, abort_flag);
      const uint64_t qdesc = make_sdesc(smem_u32(sQ), 16, 1024, SWZ_128B);
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j % PAIR_KST;
        if (!mbar_wait(smem_u32(&k_full[s]), (j / PAIR_KST) & 1, p.err, abort_flag)) { ok = false; break; }
        if (j > 0 && !mbar_wait(smem_u32(s_empty), (j - 1) & 1, p.err, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kdesc = make_sdesc(smem_u32(sK + s * AP_KH_BYTES), 16, 1024, SWZ_128B);
#pragma unroll
        for (int kk = 0; kk < AT_HD / 16; ++kk) {
          const uint32_t c = kk >> 2, off = (kk & 3) * 32;
          const uint64_t ad = qdesc + static_cast<uint64_t>((c * (128 * 128) + off) >> 4);
          const uint64_t bd = kdesc + static_cast<uint64_t>((c * (64 * 128) + off) >> 4);
          mma_bf16_ss_pair(tS, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit_pair(smem_u32(s_full), 0x3);
        mma_commit_pair(smem_u32(&k_empty[s]), 0x3);
      }
      mma_commit_pair(smem_u32(mma_done), 0x1);
      mbar_wait(smem_u32(mma_done), 0, nullptr, &never, 100000000ull);
    }
  } else if (warp == PAIR_PV_WARP) {
    // PV issuer: O += P_j V_j once P_j is published (TMEM buffer j & 1, the A
    // operand) and V_j has landed
    if (lane == 0 && leader) {
      const uint32_t idesc_pv = make_idesc_bf16(256, AT_HD, false, true);
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j % PAIR_VST;
        // V first: it has normally landed long before P_j, so its check is
        // off the path from P_j's publication to the first PV instruction
        if (!mbar_wait(smem_u32(&v_full[s]), (j / PAIR_VST) & 1, p.err, abort_flag)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&p_full[j & 1]), (j >> 1) & 1, p.err, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t vdesc = make_sdesc(smem_u32(sV + s * AP_VH_BYTES), AP_BN * 128, 1024, SWZ_128B);
#pragma unroll
        for (int kk = 0; kk < AP_BN / 16; ++kk) {
          const uint64_t bd = vdesc + static_cast<uint64_t>((kk * (16 * 128)) >> 4);
          mma_bf16_ts_pair(tO, tP + 64 * (j & 1) + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_pair(smem_u32(&pv_done[j & 1]), 0x3);
        mma_commit_pair(smem_u32(&v_empty[s]), 0x3);
      }
      mma_commit_pair(smem_u32(mma_done_pv), 0x1);
      mbar_wait(smem_u32(mma_done_pv), 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ---------------------------------------------------------------- softmax: group g owns keys [32 g, 32 g + 32)
    const int wg = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    const float off = -QKN_OFFSET_LOG2;
    int klo, khi;
    key_mask_range(p, b, klo, khi);
    const uint32_t s_empty_l = mapa_shared(smem_u32(s_empty), 0);
    float l = 0.f;
    bool ok = true;
    // S_j out of TMEM into r (this group's 32 columns), then S is released
    uint32_t r[32];
    auto read_s = [&](int j) -> bool {
      const bool got = mbar_wait(smem_u32(s_full), j & 1, p.err, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) return false;
      tc_fence_after();
      tmem_ld32(tS + PAIR_KPW * wg + lane_off, r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(s_empty_l);
      return true;
    };
    if (ok && nkv > 0) ok = read_s(0);
    bool have_next = true;  // r holds S_j at the top of iteration j
    for (int j = 0; j < nkv && ok; ++j) {
      if (!have_next && !read_s(j)) { ok = false; break; }
      const int kbase = kv_tile(j) * AP_BN + PAIR_KPW * wg;
      const int kvalid = p.N - kbase, mlo = klo - kbase, mhi = khi - kbase;
      const bool partial = kvalid < PAIR_KPW || (mlo < mhi && mlo < PAIR_KPW && mhi > 0);
      auto dead = [&](int i) { return i >= kvalid || (i >= mlo && i < mhi); };
      uint32_t pk[16];
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float e0 = ex2_approx(fmaf(__uint_as_float(r[2 * i]), c, off));
        float e1 = ex2_approx(fmaf(__uint_as_float(r[2 * i + 1]), c, off));
        float e2 = ex2_approx(fmaf(__uint_as_float(r[16 + 2 * i]), c, off));
        float e3 = ex2_approx(fmaf(__uint_as_float(r[16 + 2 * i + 1]), c, off));
        if (partial) {
          if (dead(2 * i)) e0 = 0.f;
          if (dead(2 * i + 1)) e1 = 0.f;
          if (dead(16 + 2 * i)) e2 = 0.f;
          if (dead(16 + 2 * i + 1)) e3 = 0.f;
        }
        rs0 += e0 + e1;
        rs1 += e2 + e3;
        pk[i] = pack_bf16(e0, e1);
        pk[8 + i] = pack_bf16(e2, e3);
      }
      l += rs0 + rs1;
      // S_{j+1} now if it has completed (the S product after it can start
      // while P_j is stored), otherwise after P_j
      have_next = false;
      if (j + 1 < nkv && __all_sync(0xffffffffu, mbar_test(smem_u32(s_full), (j + 1) & 1))) {
        if (!read_s(j + 1)) { ok = false; break; }
        have_next = true;
      }
      // P buffer j & 1 is free once PV_{j-2} has completed
      if (j >= 2) {
        const bool g2 = mbar_wait(smem_u32(&pv_done[j & 1]), ((j - 2) >> 1) & 1, p.err, abort_flag);
        __syncwarp();
        if (!__all_sync(0xffffffffu, g2)) { ok = false; break; }
      }
      // this group's 32 keys of P_j (two per 32-bit column, in key order) into
      // columns [16 wg, 16 wg + 16) of TMEM buffer j & 1
      tmem_st16(tP + 64 * (j & 1) + 16 * wg + lane_off, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&p_full[j & 1]), 0));
    }
    if (ok) {
      // after the last PV no V stage is read any more: V stage 0 takes the row sums
      const int jl = nkv - 1;
      const bool g3 = mbar_wait(smem_u32(&pv_done[jl & 1]), (jl >> 1) & 1, p.err, abort_flag);
      __syncwarp();
      if (__all_sync(0xffffffffu, g3)) {
        float* xsum = reinterpret_cast<float*>(sV);  // [wg 4][row 128]
        xsum[wg * 128 + row] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(lbar));
        const bool g4 = mbar_wait(smem_u32(lbar), 0, p.err, abort_flag);
        __syncwarp();
        if (__all_sync(0xffffffffu, g4)) {
          tc_fence_after();
          const float tot = xsum[row] + xsum[128 + row] + xsum[256 + row] + xsum[384 + row];
          const float inv = 1.0f / tot;
          // this warp's 32 rows x 64 columns of O, normalised, through shared
          // memory (the Q tile's bytes: every S product has completed) so that
          // the global stores are row-contiguous: thread = row when reading
          // TMEM, 8 lanes per 128-byte row segment when writing out
          uint8_t* stage = sQ + wg * (128 * 128);  // [128 rows][128 bytes], 16-byte units XOR-swizzled
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 64 * wg + cc * 32 + lane_off, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 u;
              u.x = pack_bf16(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
              u.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
              u.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
              u.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
              const int unit = cc * 4 + i;
              *reinterpret_cast<uint4*>(stage + row * 128 + ((unit ^ (row & 7)) << 4)) = u;
            }
          }
          __syncwarp();
          const int unit = lane & 7;
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = quarter * 32 + it * 4 + (lane >> 3);  // a row of this warp
            const int qrow = q0 + rr;
            if (qrow < p.N) {
              uint16_t* dst =
                  qrow < p.split
                      ? p.out_a + (static_cast<size_t>(b) * p.split + qrow) * p.ldo
                      : p.out_b + (static_cast<size_t>(b) * (p.N - p.split) + (qrow - p.split)) * p.ldo;
              const uint4 u = *reinterpret_cast<const uint4*>(stage + rr * 128 + ((unit ^ (rr & 7)) << 4));
              *reinterpret_cast<uint4*>(dst + h * AT_HD + 64 * wg + unit * 8) = u;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------- small heads (SIMT)
template <int HD>
__global__ void attn_small_simt(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                const uint16_t* __restrict__ v, AttnParams p) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  if (i >= p.N) return;
  const size_t base = (static_cast<size_t>(b) * p.H + h) * p.N;
  float qv[HD], o[HD];
  for (int d = 0; d < HD; ++d) {
    qv[d] = __uint_as_float(static_cast<uint32_t>(q[(base + i) * HD + d]) << 16);
    o[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  int klo, khi;
  key_mask_range(p, b, klo, khi);
  for (int j = 0; j < p.N; ++j) {
    if (j >= klo && j < khi) continue;
    float s = 0.f;
    for (int d = 0; d < HD; ++d) s += qv[d] * __uint_as_float(static_cast<uint32_t>(k[(base + j) * HD + d]) << 16);
    s *= p.scale_log2;
    const float mn = fmaxf(m, s);
    const float a = exp2f(m - mn), e = exp2f(s - mn);
    l = l * a + e;
    for (int d = 0; d < HD; ++d)
      o[d] = o[d] * a + e * __uint_as_float(static_cast<uint32_t>(v[(base + j) * HD + d]) << 16);
    m = mn;
  }
  uint16_t* dst = i < p.split ? p.out_a + (static_cast<size_t>(b) * p.split + i) * p.ldo + h * HD
                              : p.out_b + (static_cast<size_t>(b) * (p.N - p.split) + (i - p.split)) * p.ldo + h * HD;
  for (int d = 0; d < HD; ++d) dst[d] = static_cast<uint16_t>(pack_bf16(o[d] / l, 0.f) & 0xFFFFu);
}

cudaError_t attention_set_attributes() {
  static uint64_t done = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if ((done >> dev) & 1u) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(attn_hd256_online, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_hd256_qknorm, cudaFuncAttributeMaxDynamicSharedMemorySize, QKN_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_hd256_qknorm_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, PAIR_SMEM);
  if (e != cudaSuccess) return e;
  done |= uint64_t(1) << dev;
  return cudaSuccess;
}

cudaError_t launch_attention(const AttnParams& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             cudaStream_t stream) {
  if (p.N <= 0 || p.B <= 0 || p.H <= 0) return cudaSuccess;
  if (p.hd == AT_HD) {
    CUtensorMap tq, tk, tv;
    const uint64_t rb = AT_HD * 2, sb = static_cast<uint64_t>(p.N) * AT_HD * 2;
    const uint64_t bh = static_cast<uint64_t>(p.B) * p.H;
    if (!encode_tmap_3d(&tq, q, AT_HD, p.N, bh, rb, sb, 64, AT_BM, 1)) return cudaErrorInvalidValue;
    if (!encode_tmap_3d(&tk, k, AT_HD, p.N, bh, rb, sb, 64, AT_BN, 1)) return cudaErrorInvalidValue;
    if (!encode_tmap_3d(&tv, v, AT_HD, p.N, bh, rb, sb, 64, AT_BN, 1)) return cudaErrorInvalidValue;
    {
      cudaError_t e = attention_set_attributes();
      if (e != cudaSuccess) return e;
    }
    if (p.qk_normalized && p.N >= 256) {
      CUtensorMap tv2;  // V halves: 128 keys x 64 columns per box
      if (!encode_tmap_3d(&tv2, v, AT_HD, p.N, bh, rb, sb, 64, AP_BN, 1)) return cudaErrorInvalidValue;
      dim3 grid2(2 * ((p.N + 255) / 256), p.H, p.B);
      attn_hd256_qknorm_pair<<<grid2, PAIR_THREADS, PAIR_SMEM, stream>>>(tq, tk, tv2, p);
      return cudaGetLastError();
    }
    dim3 grid((p.N + AT_BM - 1) / AT_BM, p.H, p.B);
    if (p.qk_normalized)
      attn_hd256_qknorm<<<grid, QKN_THREADS, QKN_SMEM, stream>>>(tq, tk, tv, p);
    else
      attn_hd256_online<<<grid, AT_THREADS, AT_SMEM, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
  }
  dim3 grid((p.N + 127) / 128, p.H, p.B);
  switch (p.hd) {
    case 8: attn_small_simt<8><<<grid, 128, 0, stream>>>(q, k, v, p); break;
    case 16: attn_small_simt<16><<<grid, 128, 0, stream>>>(q, k, v, p); break;
    case 32: attn_small_simt<32><<<grid, 128, 0, stream>>>(q, k, v, p); break;
    case 64: attn_small_simt<64><<<grid, 128, 0, stream>>>(q, k, v, p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace af
