// noalloc.cu -- a timestep-embedding entry point that never allocates.
//
// Some callers cannot allocate device memory at the point where they need a
// timestep embedding: a host process whose device memory is owned and
// budgeted by another framework's allocator, a latency-critical loop that
// must not pay for cudaMalloc / cudaFree (which may synchronise the device
// and stall unrelated streams), or a plug-in that is only allowed to
// allocate during its initialisation.  af_timestep_embed needs an
// af_scratch, which is created with cudaMalloc.  af_timestep_embed_noalloc
// computes the same result with the same kernels, but stages its
// intermediates (the 256-channel sinusoid and the SiLU hidden layer of the
// timestep MLP) in the fixed array below, which the CUDA runtime creates
// when the library is loaded.  The architecture description has no
// counterpart of this call; it exists only for such callers.
//
// Limits and sharing:
//   * The array holds kNoAllocFloats = 65536 floats (256 KB) and is held by
//     every GPU that loads this library until the process exits.
//   * A call needs B * (timestep_channels + inner_dim) floats of it; larger
//     requests are rejected with AF_ERR_SHAPE before anything is launched.
//   * All calls on a device share the one array and it keeps the contents
//     of the last call.  Nothing in it has to start at zero: both staged
//     buffers are fully written before they are read.  Calls that overlap on
//     the GPU (different streams, or host threads racing) overwrite each
//     other's intermediates; serialise them.
//   * The first call on each device resolves the array's device address
//     (cudaGetSymbolAddress, with that device made current); make that first
//     call before any stream capture.  A lookup that fails is not cached:
//     the next call tries again.
//   * Like every entry point taking a weight pack, it launches on the
//     current device, which must be the pack's (else AF_ERR_INVALID_ARG);
//     fp32 packs are not covered (AF_ERR_UNSUPPORTED).
#include <mutex>
#include <string>

#include "af.h"
#include "af_internal.h"

namespace {

constexpr int kNoAllocFloats = 65536;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocFloats];

constexpr int kMaxDevices = 64;
float* g_addr[kMaxDevices] = {};  // resolved device address per device, nullptr until a lookup succeeds
std::mutex g_addr_mutex;

// Device address of g_noalloc_scratch on `dev` (the host-side symbol is only
// a stand-in and must never be handed to a kernel).  Only a successful
// lookup is remembered.
cudaError_t scratch_address(int dev, float** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_addr_mutex);
  if (!g_addr[dev]) {
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e == cudaSuccess) e = cudaSetDevice(dev);
    if (e != cudaSuccess) return e;
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    cudaSetDevice(prev);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();  // leave no sticky error behind; the next call retries
      return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    }
    g_addr[dev] = static_cast<float*>(p);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" af_status af_timestep_embed_noalloc(const af_weights* w, const float* t, int B, float* temb,
                                               void* stream) {
  using namespace af;
  if (!w || !t || !temb || B <= 0) return AF_ERR_INVALID_ARG;
  if (weights_is_f32(w)) return AF_ERR_UNSUPPORTED;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    set_last_error(cudaGetErrorString(cudaGetLastError()));
    return AF_ERR_CUDA;
  }
  if (cur != weights_device(w)) {
    set_last_error("af_timestep_embed_noalloc: the current device (" + std::to_string(cur) +
                   ") is not the weight pack's device (" + std::to_string(weights_device(w)) + ")");
    return AF_ERR_INVALID_ARG;
  }
  const int C = weights_timestep_channels(w);
  const int D = weights_inner_dim(w);
  if (static_cast<long long>(B) * (C + D) > kNoAllocFloats) {
    set_last_error("af_timestep_embed_noalloc: B * (timestep_channels + inner_dim) = " +
                   std::to_string(static_cast<long long>(B) * (C + D)) + " floats exceeds the fixed " +
                   std::to_string(kNoAllocFloats) + "-float scratch");
    return AF_ERR_SHAPE;
  }
  float* scratch = nullptr;
  cudaError_t e = scratch_address(weights_device(w), &scratch);
  if (e != cudaSuccess) {
    set_last_error(std::string("af_timestep_embed_noalloc set-up: ") + cudaGetErrorString(e));
    return AF_ERR_CUDA;
  }
  float* feat = scratch;                               // [B, C]
  float* hidden = scratch + static_cast<size_t>(B) * C;  // [B, D]
  e = launch_timestep_mlp(t, B, weights_tensor(w, "time_step_proj.linear_1.weight"),
                          weights_tensor(w, "time_step_proj.linear_1.bias"),
                          weights_tensor(w, "time_step_proj.linear_2.weight"),
                          weights_tensor(w, "time_step_proj.linear_2.bias"), C, D, feat, hidden, temb,
                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return AF_ERR_CUDA;
  }
  return AF_OK;
}
