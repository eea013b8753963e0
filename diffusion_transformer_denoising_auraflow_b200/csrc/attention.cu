// attention.cu -- joint / self attention of the AuraFlow blocks on sm_100a.
//
//   O = softmax(Q K^T * hd^-1/2) V   per (sample, head); non-causal, no mask
//
// ("Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南",
// §注意力处理器与 QKV 融合: text and image tokens are concatenated and
// attended jointly with SDPA, dropout 0, is_causal False.)
//
// attn_hd256_tcgen05: one CTA = 128 query rows of one (sample, head).
//   smem: Q 128x256 (64 KB, loaded once), K and V tiles of 64 keys x 256
//   double-buffered (2 x 32 KB each), P 128x64 bf16 (16 KB); all 128-byte
//   swizzled.  TMEM (512 columns): O 128x256 fp32 in columns [0,256), two
//   S buffers 128x64 fp32 in [256,384).
//   warp 0      TMA producer (Q once, then K_j, V_j).
//   warp 1      one thread issues S_{j+1} = Q K_{j+1}^T (M=128, N=64, K=256)
//               before O += P_j V_j (M=128, N=256, K=64, V read MN-major),
//               so the tensor core works on the next scores while the
//               softmax warps handle the current ones.
//   warps 2..5  softmax: thread = query row; loads its S row from TMEM,
//               masks keys >= N, fp32 online softmax in the exp2 domain with
//               a lazy running max (O is rescaled only when the max grows by
//               more than 2^8), writes P (bf16) into shared memory, and at the
//               end normalises O and stores it.
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
constexpr int AT_THREADS = 192;
constexpr int AT_SMEM = AT_Q_BYTES + 4 * AT_KV_BYTES + AT_P_BYTES + 512 + 1024;
constexpr float LAZY_RESCALE_LOG2 = 8.0f;

__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_hd256_tcgen05(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + AT_Q_BYTES;            // 2 buffers
  uint8_t* sV = sK + 2 * AT_KV_BYTES;       // 2 buffers
  uint8_t* sP = sV + 2 * AT_KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + AT_P_BYTES);
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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
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
      mbar_init(smem_u32(&s_empty[i]), 128);
    }
    mbar_init(smem_u32(p_full), 128);
    mbar_init(smem_u32(o_done), 1);
    mbar_init(smem_u32(mma_done), 1);
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

  if (warp == 0) {
    if (lane == 0) {
      uint32_t armedK = 0, armedV = 0, parK = 0, parV = 0;
      bool ok = true;
      mbar_arrive_expect_tx(smem_u32(q_full), AT_Q_BYTES);
      for (int c = 0; c < 4; ++c)
        tma_load_3d(smem_u32(sQ + c * (AT_BM * 128)), &tmQ, smem_u32(q_full), c * 64, q0, bh);
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(smem_u32(&k_empty[s]), ph ^ 1u, p.err, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(smem_u32(&k_full[s]), AT_KV_BYTES);
        armedK |= 1u << s; parK = (parK & ~(1u << s)) | (ph << s);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(smem_u32(sK + s * AT_KV_BYTES + c * (AT_BN * 128)), &tmK, smem_u32(&k_full[s]), c * 64,
                      j * AT_BN, bh);
        if (!mbar_wait(smem_u32(&v_empty[s]), ph ^ 1u, p.err, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(smem_u32(&v_full[s]), AT_KV_BYTES);
        armedV |= 1u << s; parV = (parV & ~(1u << s)) | (ph << s);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(smem_u32(sV + s * AT_KV_BYTES + c * (AT_BN * 128)), &tmV, smem_u32(&v_full[s]), c * 64,
                      j * AT_BN, bh);
      }
      if (!ok) {
        mbar_wait(smem_u32(q_full), 0, nullptr, &never, 100000000ull);
        for (int s = 0; s < 2; ++s) {
          if (armedK & (1u << s)) mbar_wait(smem_u32(&k_full[s]), (parK >> s) & 1u, nullptr, &never, 100000000ull);
          if (armedV & (1u << s)) mbar_wait(smem_u32(&v_full[s]), (parV >> s) & 1u, nullptr, &never, 100000000ull);
        }
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
          const uint64_t ad = make_sdesc(qaddr + c * (AT_BM * 128) + off, 16, 1024, SWZ_128B);
          const uint64_t bd = make_sdesc(kaddr + c * (AT_BN * 128) + off, 16, 1024, SWZ_128B);
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
          const uint64_t ad = make_sdesc(paddr + kk * 32, 16, 1024, SWZ_128B);
          const uint64_t bd = make_sdesc(vaddr + kk * (16 * 128), AT_BN * 128, 1024, SWZ_128B);
          mma_bf16_ss(tO, ad, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(o_done));
        mma_commit(smem_u32(&v_empty[s]));
      }
      mma_commit(smem_u32(mma_done));
      mbar_wait(smem_u32(mma_done), 0, nullptr, &never, 100000000ull);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    uint8_t* prow = sP + row * 128;
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      const bool got = mbar_wait(smem_u32(&s_full[s]), (j >> 1) & 1, p.err, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tS + s * AT_BN + lane_off, r0);
      tmem_ld32(tS + s * AT_BN + 32 + lane_off, r1);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&s_empty[s]));
      float x[64];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        x[i] = __uint_as_float(r0[i]) * p.scale_log2;
        x[32 + i] = __uint_as_float(r1[i]) * p.scale_log2;
      }
      const int kvalid = p.N - j * AT_BN;
      if (kvalid < AT_BN) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= kvalid) x[i] = -INFINITY;
      }
      float mt = x[0];
#pragma unroll
      for (int i = 1; i < 64; ++i) mt = fmaxf(mt, x[i]);
      float m_new = m;
      bool rescale = false;
      if (j == 0) {
        m_new = mt;
      } else if (mt > m + LAZY_RESCALE_LOG2) {
        m_new = mt;
        rescale = true;
      }
      float rs = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float e0 = exp2f(x[2 * i] - m_new);
        const float e1 = exp2f(x[2 * i + 1] - m_new);
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
        const float alpha = rescale ? exp2f(m - m_new) : 1.0f;
        for (int c = 0; c < AT_HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32 + lane_off, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + c * 32 + lane_off, o);
        }
        tmem_wait_st();
        l *= alpha;
      }
      m = m_new;
      l += rs;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(p_full));
    }
    if (ok) {
      const bool g3 = mbar_wait(smem_u32(o_done), (nkv - 1) & 1, p.err, abort_flag);
      __syncwarp();
      if (__all_sync(0xffffffffu, g3)) {
        tc_fence_after();
        const int qrow = q0 + row;
        const bool row_ok = qrow < p.N;
        uint16_t* dst = nullptr;
        if (row_ok) {
          if (qrow < p.split)
            dst = p.out_a + (static_cast<size_t>(b) * p.split + qrow) * p.ldo + h * AT_HD;
          else
            dst = p.out_b + (static_cast<size_t>(b) * (p.N - p.split) + (qrow - p.split)) * p.ldo + h * AT_HD;
        }
        const float inv = 1.0f / l;
        for (int c = 0; c < AT_HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32 + lane_off, o);
          tmem_wait_ld();
          if (row_ok) {
            uint4* d = reinterpret_cast<uint4*>(dst + c * 32);
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
  for (int j = 0; j < p.N; ++j) {
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
    static bool attr = false;
    if (!attr) {
      cudaError_t e = cudaFuncSetAttribute(attn_hd256_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
      if (e != cudaSuccess) return e;
      attr = true;
    }
    dim3 grid((p.N + AT_BM - 1) / AT_BM, p.H, p.B);
    attn_hd256_tcgen05<<<grid, AT_THREADS, AT_SMEM, stream>>>(tq, tk, tv, p);
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
