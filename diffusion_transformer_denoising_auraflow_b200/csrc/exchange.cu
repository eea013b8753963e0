// exchange.cu -- the two-GPU CFG split's velocity exchange, fused into the
// guidance + Euler update.
//
// The sampling loop's CFG batch is [uncond; text] and the two halves are
// independent forwards ("Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级
// 使用指南", §在 AuraFlowPipeline 中的实际调用: the latents are duplicated and
// the prediction chunked into the uncond and text halves; the guidance
// formula is in "Diffusers 中 AuraFlow 管线实战", §AuraFlowPipeline 核心参数详解).
// With one process per GPU, each writes its half of the velocity into an
// exchange buffer that the other process maps (CUDA IPC); the guidance +
// Euler kernel then reads its own half locally and the peer's half directly
// from the peer GPU's memory (NVLink), with no separate copy.  Plain loads
// only: no TMA, no multicast, nothing that waits on the other GPU.  Ordering
// is the caller's: a rank launches the update only after both halves of the
// step are complete (stream sync + host barrier), and a slot is not
// rewritten until the peer has passed the next barrier.
#include <cstring>
#include <string>

#include "af.h"
#include "af_internal.h"

struct af_exchange {
  int device = 0;
  size_t bytes = 0;
  void* local = nullptr;       // this process's buffer (cudaMalloc)
  void* peer = nullptr;        // the peer's buffer, mapped into this process
};

namespace {
af_status fail(cudaError_t e, const char* what) {
  af::set_last_error(std::string(what) + ": " + cudaGetErrorString(e));
  cudaGetLastError();
  return AF_ERR_CUDA;
}

af_status on_device(int dev) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return fail(cudaGetLastError(), "cudaGetDevice");
  if (cur != dev) {
    af::set_last_error("the current device (" + std::to_string(cur) + ") is not the exchange buffer's (" +
                       std::to_string(dev) + ")");
    return AF_ERR_INVALID_ARG;
  }
  return AF_OK;
}
}  // namespace

extern "C" {

af_status af_exchange_create(int device, size_t bytes, af_exchange** out) {
  if (!out || bytes == 0) return AF_ERR_INVALID_ARG;
  *out = nullptr;
  int prev = 0;
  cudaGetDevice(&prev);
  if (cudaSetDevice(device) != cudaSuccess) {
    cudaGetLastError();
    return AF_ERR_INVALID_ARG;
  }
  af_exchange* x = new af_exchange();
  x->device = device;
  x->bytes = bytes;
  cudaError_t e = cudaMalloc(&x->local, bytes);
  if (e == cudaSuccess) e = cudaMemset(x->local, 0, bytes);
  cudaSetDevice(prev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    if (x->local) cudaFree(x->local);
    delete x;
    return AF_ERR_OOM;
  }
  *out = x;
  return AF_OK;
}

af_status af_exchange_handle(const af_exchange* x, void* handle) {
  if (!x || !handle) return AF_ERR_INVALID_ARG;
  af_status st = on_device(x->device);
  if (st != AF_OK) return st;
  cudaIpcMemHandle_t h;
  const cudaError_t e = cudaIpcGetMemHandle(&h, x->local);
  if (e != cudaSuccess) return fail(e, "cudaIpcGetMemHandle");
  static_assert(sizeof(cudaIpcMemHandle_t) <= AF_IPC_HANDLE_BYTES, "IPC handle size");
  memset(handle, 0, AF_IPC_HANDLE_BYTES);
  memcpy(handle, &h, sizeof(h));
  return AF_OK;
}

af_status af_exchange_open_peer(af_exchange* x, const void* peer_handle) {
  if (!x || !peer_handle || x->peer) return AF_ERR_INVALID_ARG;
  af_status st = on_device(x->device);
  if (st != AF_OK) return st;
  cudaIpcMemHandle_t h;
  memcpy(&h, peer_handle, sizeof(h));
  void* p = nullptr;
  const cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return fail(e, "cudaIpcOpenMemHandle");
  x->peer = p;
  return AF_OK;
}

af_status af_exchange_ptrs(const af_exchange* x, void** local, void** peer) {
  if (!x) return AF_ERR_INVALID_ARG;
  if (local) *local = x->local;
  if (peer) *peer = x->peer;
  return AF_OK;
}

void af_exchange_destroy(af_exchange* x) {
  if (!x) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(x->device);
  if (x->peer) cudaIpcCloseMemHandle(x->peer);
  if (x->local) cudaFree(x->local);
  cudaSetDevice(prev);
  delete x;
}

af_status af_euler_cfg_step2(float* latents, const float* v_uncond, const float* v_text, int Bi, int C, int H, int W,
                             float guidance, float sigma, float sigma_next, void* stream) {
  if (!latents || !v_uncond || !v_text || Bi <= 0 || C <= 0 || H <= 0 || W <= 0) return AF_ERR_INVALID_ARG;
  const cudaError_t e = af::launch_euler_cfg2(latents, v_uncond, v_text, static_cast<int64_t>(Bi) * C * H * W,
                                              guidance, sigma, sigma_next, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(e, "euler_cfg");
  return AF_OK;
}

}  // extern "C"
