// The library's device error word: kernels with time-bounded waits write a
// code here (instead of hanging) when a wait gives up.
#include <mutex>

#include <cuda_runtime.h>

#include "launch.h"
#include "rtp.h"

namespace {
__device__ int g_rtp_error_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_word_ptr[kMaxDevices] = {};
}  // namespace

namespace rtp {
cudaError_t device_error_word(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_word_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_rtp_error_word);
    if (e != cudaSuccess) return e;
    g_word_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_word_ptr[dev];
  return cudaSuccess;
}
}  // namespace rtp

extern "C" rtp_status rtp_poll_device_error(int32_t* code) {
  if (!code) return RTP_ERR_INVALID_ARG;
  int* w = nullptr;
  cudaError_t e = rtp::device_error_word(&w);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  int v = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && v) e = cudaMemset(w, 0, sizeof(int));
  if (e != cudaSuccess) {
    rtp::set_last_cuda_error((int32_t)e);
    return RTP_ERR_CUDA;
  }
  *code = v;
  return RTP_OK;
}
