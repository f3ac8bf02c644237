// Host-side launcher interfaces between the C ABI (rtp_api.cu) and the kernels.
// Arguments arrive here already validated.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace rtp {

// Launch `kern` with programmatic stream serialization (and an optional
// cluster shape), so it may be scheduled while the previous kernel of the
// stream drains; the kernel itself calls pdl_wait() before reading inputs.
template <typename K, typename... Args>
cudaError_t launch_pdl(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, unsigned cluster,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

struct LaunchIndexProject {
  View4 x;
  const float* P;
  MutView4 out;
  int64_t B, H, HP, N;
  bool in_bf16, out_bf16;
};
cudaError_t launch_index_project(const LaunchIndexProject& a, cudaStream_t stream);

// Top-p selection, decode form (one query per (b, h)).
struct LaunchToppDecode {
  View4 q_idx;   // [B, Hq, 1, 16]
  View4 k_idx;   // [B, Hk, N, 16]
  const int32_t* lens;
  int64_t B, Hq, Hk, N;
  float p;
  int32_t topk;  // > 0: keep the topk highest-scoring keys instead of the top-p mass
  bool bf16;
  uint32_t* tau_bits;
  int32_t* tiepos;
  int32_t* count;
  uint32_t* mask;
  int64_t mask_words;
  float* spill = nullptr;  // workspace: scores past the ones a CTA keeps on chip (long caches)
};
cudaError_t launch_topp_decode(const LaunchToppDecode& a, cudaStream_t stream);
bool topp_decode_supported(int64_t N);
size_t topp_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t N);

// Top-p selection, prefill form (T query tokens per sequence), tcgen05 score tiles.
struct LaunchToppPrefill {
  View4 q_idx;   // [B, Hq, T, 16] bf16
  View4 k_idx;   // [B, Hk, N, 16] bf16
  const int32_t* lens;
  int64_t B, Hq, Hk, T, N;
  float p;
  uint32_t* tau_bits;
  int32_t* tiepos;
  int32_t* count;
  uint32_t* mask;
  int64_t mask_words;
  int* err;      // device error word
};
cudaError_t launch_topp_prefill(const LaunchToppPrefill& a, cudaStream_t stream);

// Prefill kernels pack the G = Hq / Hk query heads of one KV head into a block
// of 128 rows: TB tokens per head, TB = 128 / G rounded down to a multiple of 8
// (the TMA swizzle atom); G must be at most 16.
inline int prefill_tokens_per_block(int G) { return (128 / G) & ~7; }
constexpr int kPrefillMaxGroup = 16;

// Prefill attention (T query tokens per sequence, bf16): sparse form (threshold
// selection + projected tiles) when W == 0, sliding window when W > 0.
struct LaunchAttnPrefill {
  View4 q, k, v;          // [B, Hq, T, 128], [B, Hk, N, 128]
  View4 q_idx, k_idx;     // sparse form: [B, Hq, T, 16], [B, Hk, N, 16]
  const int32_t* lens;
  const uint32_t* tau_bits;
  const int32_t* tiepos;
  int64_t B, Hq, Hk, T, N;
  int32_t W;
  float scale;
  MutView4 o;
  bool o_bf16;
  int* err;
};
cudaError_t launch_attn_prefill(const LaunchAttnPrefill& a, cudaStream_t stream);

// Device address of the library's error word in the current CUDA context.
cudaError_t device_error_word(int** out);
// Device address of a file-scope __device__ variable (given by its host-side
// name) in the current CUDA context, looked up once per context: a device
// reset or another context on the same device gets its own lookup.
cudaError_t symbol_address(const void* symbol, void** out);
// Cycles a device wait may take before it gives up (rtp_set_wait_budget_cycles).
constexpr long long kDefaultWaitBudgetCycles = 4000000000LL;  // ~2 s at 1.9 GHz
long long wait_budget_cycles();

// Decode attention: sparse (mask given) or sliding window (W > 0).
struct LaunchAttnDecode {
  View4 q;       // [B, Hq, 1, 128]
  View4 k, v;    // [B, Hk, N, 128]
  const int32_t* lens;
  const uint32_t* mask;  // sparse mode: [B*Hq, mask_words]
  int64_t mask_words;
  int64_t B, Hq, Hk, N;
  int32_t W;             // > 0: window mode
  float scale;
  bool bf16;             // q/k/v dtype
  MutView4 o;            // [B, Hq, 1, 128]
  bool o_bf16;
  void* ws;
  int64_t key_lo = 0;    // sparse mode: global position of key row 0 (multiple of 64)
  float* lse = nullptr;  // [B, Hq] (row stride lse_sb) or null: log-sum-exp of the attended scaled scores
  int64_t lse_sb = 0;
};
bool attn_decode_supported(int64_t B, int64_t Hk, int64_t N, int32_t W);
size_t attn_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t Hk, int64_t N, int32_t W);
cudaError_t launch_attn_decode(const LaunchAttnDecode& a, cudaStream_t stream);
// Every check rtp_sparse_attn_decode makes except the workspace's; on RTP_OK
// *a holds the launch arguments (a->ws still to be set).  Nothing is launched.
rtp_status check_sparse_attn_decode(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                    const int32_t* lens, const rtp_selection* sel, float scale,
                                    const rtp_tensor* o, LaunchAttnDecode* a, bool key_range);
// Byte range of the completion tickets inside a decode-attention workspace.
void attn_decode_ticket_range(int64_t B, int64_t Hk, int64_t N, int32_t W, size_t* offset, size_t* bytes);

// TMA descriptors: [B, H, R, 16] bf16 projected rows (box of box_rows rows,
// 32-byte swizzle), and [B, H, R, 128] bf16 K/V rows (box of box_rows rows x
// 64 columns, 128-byte swizzle).
bool make_idx_map(CUtensorMap* map, const View4& v, int64_t B, int64_t H, int64_t R, int box_rows);
bool make_row_map(CUtensorMap* map, const View4& v, int64_t B, int64_t H, int64_t R, int box_rows);

// Merge of key-range attention partials (rtp_attn_combine).
struct AttnCombineArgs {
  const float* o_parts;      // [S, B, Hq, 128] f32, strides ps, pb, ph (elements)
  int64_t ps, pb, ph;
  const float* lse;          // [S, B, Hq] f32, strides ls, lb, 1
  int64_t ls, lb;
  int S, B, Hq;
  MutView4 o;                // [B, Hq, 1, 128]
  int o_bf16;
};
cudaError_t launch_attn_combine(const AttnCombineArgs& a, cudaStream_t stream);

// Cache append (rtp_kv_append): the first R KV heads go to the full caches
// (and the projected-key cache), the others to W-row rings.
struct KvAppendArgs {
  View4 k_new, v_new;        // [B, H, T, 128]
  const int32_t* pos;        // [B] device: position of token 0
  const float* P;            // [R, 16, 128]
  MutView4 k_cache, v_cache; // [B, R, N, 128]
  MutView4 k_idx;            // [B, R, N, 16]
  MutView4 k_ring, v_ring;   // [B, H - R, W, 128]
  int32_t* lens_out;         // [B] or null: pos + T (clamped to [0, N] when R > 0)
  int32_t* ring_lens;        // [B] or null: min(pos + T, W)
  int B, H, T, R, N, W;
};
cudaError_t launch_kv_append(const KvAppendArgs& a, bool bf16, cudaStream_t stream);

// Records a CUDA error for rtp_last_cuda_error() on this thread.
void set_last_cuda_error(int32_t e);

}  // namespace rtp
