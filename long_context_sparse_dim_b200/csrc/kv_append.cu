// Cache maintenance around the path: appending the new tokens of a sequence.
//
// "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
// Hundred Training Steps", "Three Key Insights" 1: retrieval heads keep the
// full KV cache, local heads only a local window; "Full Attention Strikes Back
// ... (RTPurbo)", TL;DR: the lightweight token indexer keeps a projected key
// per cached token of the retrieval heads.
//
// One warp per new (sequence, KV head, token) row, in one pass over the row:
//   retrieval head (kv head < R): the K and V rows go to the full cache at the
//     token's position, and the projected key P k to the projected-key cache
//     (the arithmetic of rtp_index_project, so both give identical bits);
//   local head: the K and V rows go to a ring of W rows at position mod W, so
//     the ring always holds the last W tokens (every key a local query of the
//     newest token attends) in O(W) memory.
// Attention over a set of keys does not depend on their order, so the window
// attention of the newest token is the ordinary window attention over the
// min(n, W) stored ring rows; the kernel writes that length per sequence, and
// the sequence length after the append (the next append's position).
#include "common.cuh"
#include "launch.h"
#include "project.cuh"

namespace rtp {

namespace {

constexpr int kAppThreads = 256;

template <typename T>
RTP_DEVICE void copy_row(const T* src, T* dst, int lane) {
  // 128 elements: 8 (bf16) or 16 (f32) bytes per lane
  if constexpr (sizeof(T) == 2) {
    *reinterpret_cast<uint2*>(dst + 4 * lane) = __ldg(reinterpret_cast<const uint2*>(src + 4 * lane));
  } else {
    *reinterpret_cast<float4*>(dst + 4 * lane) = __ldg(reinterpret_cast<const float4*>(src + 4 * lane));
  }
}

template <typename T>
__global__ void __launch_bounds__(kAppThreads)
kv_append_kernel(KvAppendArgs A) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * kAppThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kAppThreads) >> 5;
  const int64_t rows = (int64_t)A.B * A.H * A.T;
  int cur_hp = -1;
  float Pl[kIdxDim][4];
  for (int64_t r = warp0; r < rows; r += nwarps) {
    const int t = (int)(r % A.T);
    const int64_t bh = r / A.T;
    const int h = (int)(bh % A.H), b = (int)(bh / A.H);
    const int p = A.pos[b] + t;  // position of this token in its sequence
    const T* kin = static_cast<const T*>(A.k_new.data) + b * A.k_new.sb + h * A.k_new.sh + (int64_t)t * A.k_new.sn;
    const T* vin = static_cast<const T*>(A.v_new.data) + b * A.v_new.sb + h * A.v_new.sh + (int64_t)t * A.v_new.sn;
    if (h < A.R) {
      if (p < 0 || p >= A.N) continue;  // outside the cache: nothing written
      copy_row<T>(kin, static_cast<T*>(A.k_cache.data) + b * A.k_cache.sb + h * A.k_cache.sh + (int64_t)p * A.k_cache.sn,
                  lane);
      copy_row<T>(vin, static_cast<T*>(A.v_cache.data) + b * A.v_cache.sb + h * A.v_cache.sh + (int64_t)p * A.v_cache.sn,
                  lane);
      if (h != cur_hp) {  // warp-uniform
        const float* Ph = A.P + (int64_t)h * kIdxDim * kHeadDim + 4 * lane;
#pragma unroll
        for (int j = 0; j < kIdxDim; ++j) {
          const float4 pv = __ldg(reinterpret_cast<const float4*>(Ph + j * kHeadDim));
          Pl[j][0] = pv.x;
          Pl[j][1] = pv.y;
          Pl[j][2] = pv.z;
          Pl[j][3] = pv.w;
        }
        cur_hp = h;
      }
      float xv[4];
      load4<T>(kin + 4 * lane, xv);
      project_row<T>(Pl, xv, lane,
                     static_cast<T*>(A.k_idx.data) + b * A.k_idx.sb + h * A.k_idx.sh + (int64_t)p * A.k_idx.sn);
    } else {
      // only the last W tokens of the append are kept (two tokens W apart share a slot)
      if (p < 0 || t < A.T - A.W) continue;
      const int l = h - A.R;
      const int slot = p % A.W;
      copy_row<T>(kin, static_cast<T*>(A.k_ring.data) + b * A.k_ring.sb + l * A.k_ring.sh + (int64_t)slot * A.k_ring.sn,
                  lane);
      copy_row<T>(vin, static_cast<T*>(A.v_ring.data) + b * A.v_ring.sb + l * A.v_ring.sh + (int64_t)slot * A.v_ring.sn,
                  lane);
    }
  }
  if (blockIdx.x == 0) {
    for (int b = threadIdx.x; b < A.B; b += kAppThreads) {
      const int end = A.pos[b] + A.T;  // one past the last appended position
      if (A.lens_out) A.lens_out[b] = A.R > 0 ? max(min(end, A.N), 0) : max(end, 0);
      if (A.ring_lens) A.ring_lens[b] = max(min(end, A.W), 0);
    }
  }
}

}  // namespace

cudaError_t launch_kv_append(const KvAppendArgs& a, bool bf16, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.B * a.H * a.T;
  if (rows == 0) return cudaSuccess;
  int64_t blocks = (rows + kAppThreads / 32 - 1) / (kAppThreads / 32);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (bf16)
    kv_append_kernel<__nv_bfloat16><<<(unsigned)blocks, kAppThreads, 0, stream>>>(a);
  else
    kv_append_kernel<float><<<(unsigned)blocks, kAppThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
