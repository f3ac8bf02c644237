// rtp_sparse_attn_decode_noalloc: the decode sparse attention without a caller
// workspace, for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: a plugin loaded into a
// host framework that owns every device allocation and hands its plugins no
// allocator, or a serving runtime that reserves all device memory at start-up
// and forbids allocation afterwards.  Such a caller can pass its inputs and
// outputs but has nowhere to put the split-K scratch that
// rtp_sparse_attn_decode takes as a workspace.  This entry point keeps that
// scratch in a fixed file-scope device array instead.
//
// Costs and limits of that choice:
//   * every GPU that loads librtp.so holds RTP_NOALLOC_SCRATCH_BYTES of device
//     memory for this array until the process exits;
//   * shapes whose scratch would not fit are rejected (RTP_ERR_UNSUPPORTED);
//   * all calls on a device share the one array, so calls that overlap on the
//     GPU (different streams without ordering between them) race and give
//     wrong results; order them on one stream;
//   * the array's device address is looked up once per CUDA context, on the
//     first call made with that context current (cudaGetSymbolAddress); make
//     that first call before any stream capture.  A device reset or a second
//     context on the same device gets its own lookup.
// Every argument is checked before anything is enqueued, so a call that returns
// an error status has launched nothing and written nothing.  The array keeps
// whatever the previous call left in it; the only part that must start at zero
// (the per-group completion tickets) is cleared on the stream by every call.  No cudaMalloc, cudaFree or allocating library routine
// is called.
#include <cuda_runtime.h>

#include "launch.h"
#include "rtp.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[RTP_NOALLOC_SCRATCH_BYTES];

}  // namespace

extern "C" rtp_status rtp_sparse_attn_decode_noalloc(const rtp_tensor* q, const rtp_tensor* k,
                                                     const rtp_tensor* v, const int32_t* lens,
                                                     const rtp_selection* sel, float scale,
                                                     const rtp_tensor* o, rtp_stream_t stream) {
  // every argument check first: an invalid call launches and writes nothing
  rtp::LaunchAttnDecode a;
  const rtp_status s = rtp::check_sparse_attn_decode(q, k, v, lens, sel, scale, o, &a, false);
  if (s != RTP_OK) return s;
  const size_t need = rtp_sparse_attn_decode_workspace_size(a.B, a.Hq, a.Hk, a.N);
  if (need > (size_t)RTP_NOALLOC_SCRATCH_BYTES) return RTP_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  cudaError_t e = rtp::symbol_address(reinterpret_cast<const void*>(&g_noalloc_scratch), &scratch);
  if (e != cudaSuccess) {
    rtp::set_last_cuda_error((int32_t)e);
    return RTP_ERR_CUDA;
  }
  size_t t_off = 0, t_bytes = 0;
  rtp::attn_decode_ticket_range(a.B, a.Hk, a.N, 0, &t_off, &t_bytes);
  if (t_bytes) {
    e = cudaMemsetAsync(static_cast<unsigned char*>(scratch) + t_off, 0, t_bytes, (cudaStream_t)stream);
    if (e != cudaSuccess) {
      rtp::set_last_cuda_error((int32_t)e);
      return RTP_ERR_CUDA;
    }
  }
  a.ws = scratch;
  e = rtp::launch_attn_decode(a, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    rtp::set_last_cuda_error((int32_t)e);
    return RTP_ERR_CUDA;
  }
  return RTP_OK;
}
