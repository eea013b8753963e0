// init.cu -- filling and converting the weight pack on the device.
//
//   init_normal_kernel   seeded N(0, std^2) values for one tensor of the pack:
//                        element j takes lane j % 4 of the Philox4x32-10
//                        block j / 4 (Salmon, Moraes, Dror, Shaw, "Parallel
//                        random numbers: as easy as 1, 2, 3", SC 2011) with
//                        key (seed lo, seed hi) and counter (block lo,
//                        block hi, crc32(tensor name), 0), turned into
//                        normals by the Box-Muller transform in fp64, then
//                        float32(z * std) and, for a bf16 pack, bf16 with
//                        round-to-nearest-even.  Every element is a function
//                        of its index only, so any host implementation of the
//                        same published definitions reproduces the pack.
//   convert_copy_kernel  a tensor given in bf16 or fp32 written into the pack
//                        in the pack's storage type (widening, or narrowing
//                        with round-to-nearest-even).
//
// Both honour the pack's FFN up-projection layout: linear_1 / linear_2 rows
// interleaved in 128-row groups (pair slot 1 = linear_1, 2 = linear_2).
// The architecture description gives the scales of the random
// initialisation of the position table (0.1) and the register tokens (0.02)
// ("Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南",
// §Patch Embedding, §Register Tokens); the host passes them per tensor.
#include "af_internal.h"

namespace af {

namespace {

struct Philox4 {
  uint32_t x[4];
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                                 uint32_t k1) {
  constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(M0, c0), lo0 = M0 * c0;
    const uint32_t hi1 = __umulhi(M1, c2), lo1 = M1 * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += W0;
    k1 += W1;
  }
  Philox4 o;
  o.x[0] = c0;
  o.x[1] = c1;
  o.x[2] = c2;
  o.x[3] = c3;
  return o;
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  const uint32_t u = __float_as_uint(f);
  return static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// Element j of a [rows, cols] tensor -> element offset in the pack region.
__device__ __forceinline__ size_t pack_offset(size_t j, int cols, int interleave) {
  if (interleave == 0) return j;
  const size_t row = j / static_cast<size_t>(cols), col = j - row * cols;
  const size_t prow = (row >> 7) * 256 + (interleave == 2 ? 128 : 0) + (row & 127);
  return prow * cols + col;
}

__global__ void init_normal_kernel(void* __restrict__ dst, int f32, size_t numel, int cols, int interleave,
                                   uint32_t key, uint64_t seed, float stdv) {
  const size_t nblocks = (numel + 3) / 4;
  const double s = static_cast<double>(stdv);
  for (size_t n = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; n < nblocks;
       n += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const Philox4 r = philox4x32_10(static_cast<uint32_t>(n), static_cast<uint32_t>(n >> 32), key, 0u,
                                    static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
    double z[4];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const double ua = (static_cast<double>(r.x[2 * p]) + 0.5) * 2.3283064365386963e-10;   // 2^-32
      const double ub = (static_cast<double>(r.x[2 * p + 1]) + 0.5) * 2.3283064365386963e-10;
      const double rad = sqrt(-2.0 * log(ua));
      const double th = 6.283185307179586476925286766559 * ub;
      z[2 * p] = rad * cos(th);
      z[2 * p + 1] = rad * sin(th);
    }
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const size_t j = 4 * n + l;
      if (j >= numel) break;
      const float v = __double2float_rn(z[l] * s);
      const size_t o = pack_offset(j, cols, interleave);
      if (f32)
        static_cast<float*>(dst)[o] = v;
      else
        static_cast<uint16_t*>(dst)[o] = f32_to_bf16_rne(v);
    }
  }
}

__global__ void convert_copy_kernel(const void* __restrict__ src, int src_f32, void* __restrict__ dst, int dst_f32,
                                    size_t numel, int cols, int interleave) {
  for (size_t j = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; j < numel;
       j += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float v = src_f32 ? static_cast<const float*>(src)[j]
                            : __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(src)[j]) << 16);
    const size_t o = pack_offset(j, cols, interleave);
    if (dst_f32)
      static_cast<float*>(dst)[o] = v;
    else
      static_cast<uint16_t*>(dst)[o] = f32_to_bf16_rne(v);
  }
}

int grid_for(size_t work) {
  static int sms = 0;
  if (!sms) sms = device_sm_count();
  const size_t want = (work + 255) / 256;
  const size_t cap = static_cast<size_t>(sms) * 16;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

}  // namespace

uint32_t crc32_ieee(const char* s) {
  uint32_t c = 0xFFFFFFFFu;
  for (const unsigned char* p = reinterpret_cast<const unsigned char*>(s); *p; ++p) {
    c ^= *p;
    for (int k = 0; k < 8; ++k) c = (c >> 1) ^ (0xEDB88320u & (0u - (c & 1u)));
  }
  return c ^ 0xFFFFFFFFu;
}

cudaError_t launch_init_normal(void* dst, bool f32, size_t numel, int cols, int interleave, uint32_t key,
                               uint64_t seed, float stdv, cudaStream_t s) {
  if (numel == 0) return cudaSuccess;
  init_normal_kernel<<<grid_for((numel + 3) / 4), 256, 0, s>>>(dst, f32 ? 1 : 0, numel, cols, interleave, key, seed,
                                                               stdv);
  return cudaGetLastError();
}

cudaError_t launch_convert_copy(const void* src, bool src_f32, void* dst, bool dst_f32, size_t numel, int cols,
                                int interleave, cudaStream_t s) {
  if (numel == 0) return cudaSuccess;
  convert_copy_kernel<<<grid_for(numel), 256, 0, s>>>(src, src_f32 ? 1 : 0, dst, dst_f32 ? 1 : 0, numel, cols,
                                                      interleave);
  return cudaGetLastError();
}

}  // namespace af
