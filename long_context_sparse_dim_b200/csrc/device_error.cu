// The library's device error word (kernels with time-bounded waits write a
// code here instead of hanging when a wait gives up), the wait budget, and the
// lookup of file-scope device variables' addresses per CUDA context.
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "launch.h"
#include "rtp.h"

namespace {
__device__ int g_rtp_error_word;

std::atomic<long long> g_wait_budget{rtp::kDefaultWaitBudgetCycles};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// (context, symbol) -> device address; a small table, filled once per pair.
struct SymbolEntry {
  CUcontext ctx;
  const void* symbol;
  void* addr;
};
constexpr int kMaxEntries = 256;
std::mutex g_mu;
SymbolEntry g_entries[kMaxEntries];
int g_used = 0, g_next = 0;
}  // namespace

namespace rtp {

long long wait_budget_cycles() { return g_wait_budget.load(std::memory_order_relaxed); }

cudaError_t symbol_address(const void* symbol, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  if (!ctx) {  // no context yet on this thread: make the device's primary context current
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return e;
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_used; ++i)
    if (g_entries[i].ctx == ctx && g_entries[i].symbol == symbol) {
      *out = g_entries[i].addr;
      return cudaSuccess;
    }
  void* p = nullptr;
  if ((e = cudaGetSymbolAddress(&p, symbol)) != cudaSuccess) return e;
  const int slot = g_used < kMaxEntries ? g_used++ : (g_next++ % kMaxEntries);
  g_entries[slot] = SymbolEntry{ctx, symbol, p};
  *out = p;
  return cudaSuccess;
}

cudaError_t device_error_word(int** out) {
  void* p = nullptr;
  cudaError_t e = symbol_address(reinterpret_cast<const void*>(&g_rtp_error_word), &p);
  if (e == cudaSuccess) *out = static_cast<int*>(p);
  return e;
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

extern "C" rtp_status rtp_set_wait_budget_cycles(int64_t cycles) {
  if (cycles < 0) return RTP_ERR_INVALID_ARG;
  g_wait_budget.store(cycles == 0 ? rtp::kDefaultWaitBudgetCycles : (long long)cycles, std::memory_order_relaxed);
  return RTP_OK;
}
